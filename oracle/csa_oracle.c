/*
 * csa_oracle.c -- plain CPU reference for CSA / HCA / window attention over an
 * MXFP4 KV cache. TEST INFRASTRUCTURE ONLY: see csa_oracle.h for the contract,
 * the sources and the precision rules. Written for a reader checking it
 * against the definitions, not for speed: no blocking, no fusion, one loop per
 * step of the method, every float step in double.
 */
#include "csa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ======================================================================
 * Number formats
 * ====================================================================== */

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double orc_bf16_decode(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a binary32 to the nearest bfloat16, ties to even (finite inputs). */
uint16_t orc_bf16_encode(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    uint32_t upper = u >> 16, lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
    return (uint16_t)upper;
}

/* E2M1 (OCP Microscaling Formats v1.0, FP4): bit 3 sign, bits 2..1 exponent
 * with bias 1, bit 0 mantissa. Exponent field 0 is subnormal: value = m/2. */
double orc_e2m1_decode(uint8_t code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Nearest representable magnitude among the 8 non-negative E2M1 codes, ties
 * to the code whose mantissa bit is 0, saturating to 6. The sign is kept, so
 * a negative value that rounds to zero gives code 0x8. */
uint8_t orc_e2m1_encode(double x) {
    uint8_t sign = signbit(x) ? 8 : 0;
    double a = fabs(x);
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - orc_e2m1_decode((uint8_t)c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* OCP FP8 E4M3: bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa.
 * Exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities. */
double orc_e4m3_decode(uint8_t code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest finite E4M3 magnitude (codes 0x00..0x7E are increasing), ties to
 * the even mantissa, saturating to 448. Sign kept. */
uint8_t orc_e4m3_encode(double x) {
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    int lo = 0, hi = 0x7E; /* find the largest code with magnitude <= a */
    if (a >= orc_e4m3_decode(0x7E)) return (uint8_t)(sign | 0x7E);
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (orc_e4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid - 1;
    }
    int below = lo, above = lo + 1;
    double db = a - orc_e4m3_decode((uint8_t)below);
    double da = orc_e4m3_decode((uint8_t)above) - a;
    int pick = (db < da) ? below : (da < db) ? above : ((below & 1) == 0 ? below : above);
    return (uint8_t)(sign | pick);
}

/* One MXFP4 block of 32 elements (OCP MX v1.0, section 6.3 conversion):
 * shared exponent X = floor(log2(amax)) - 2, where 2 is the exponent of the
 * largest E2M1 magnitude (6 = 1.5 * 2^2), clamped to the E8M0 range
 * [-127, 127]; a group whose amax is 0 takes X = -127 (the clamp of -inf).
 * Each element is v * 2^-X rounded to E2M1. Scaling by 2^-X is exact in
 * double, so the rounding decision is taken on the exact float32 input. */
void orc_mxfp4_quantize_group(const float *v, uint8_t *codes, uint8_t *scale_byte) {
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs((double)v[i]));
    int X;
    if (amax == 0.0) {
        X = -127;
    } else {
        int e;
        frexp(amax, &e); /* amax = f * 2^e, f in [0.5, 1): floor(log2 amax) = e-1 */
        X = (e - 1) - 2;
        if (X < -127) X = -127;
        if (X > 127) X = 127;
    }
    *scale_byte = (uint8_t)(X + 127);
    for (int i = 0; i < 32; ++i) codes[i] = orc_e2m1_encode(ldexp((double)v[i], -X));
}

/* One 16-element group of the E4M3-scaled variant (DeepSeek-V4.1-Flash podcast
 * transcript, cue 16: E2M1 elements, one E4M3 scale per sixteen channels, no
 * second-level global scale). The scale is the E4M3 rounding (nearest, ties to
 * even, saturating at 448) of amax / 6, so that the largest magnitude maps near
 * E2M1's largest value 6; each element is the E2M1 rounding of v / scale. A
 * scale that rounds to zero gives zero-magnitude codes that keep each
 * element's sign. Both quotients are taken in double; the rounding decision is
 * the one on the exact quotient (a rounded quotient of two floats never lands
 * on an E2M1 or E4M3 midpoint unless the exact one does), so it also matches a
 * correctly rounded float32 quotient or an exact threshold comparison. */
void orc_e4m3x16_quantize_group(const float *v, uint8_t *codes, uint8_t *scale_byte) {
    double amax = 0.0;
    for (int i = 0; i < 16; ++i) amax = fmax(amax, fabs((double)v[i]));
    uint8_t sb = orc_e4m3_encode(amax / 6.0);
    double s = orc_e4m3_decode(sb);
    *scale_byte = sb;
    for (int i = 0; i < 16; ++i) {
        if (s == 0.0)
            codes[i] = signbit(v[i]) ? 0x8 : 0x0;
        else
            codes[i] = orc_e2m1_encode((double)v[i] / s);
    }
}

/* Elements per scale byte: 32 for E8M0 scales (scale_fmt 0), 16 for E4M3 (1). */
static int group_size(int scale_fmt) { return scale_fmt == 0 ? 32 : 16; }

/* Element d of a stored row: E2M1(code) * 2^(byte - 127) (E8M0 scale) or
 * E2M1(code) * E4M3(byte) (E4M3 scale). */
static double fp4_element(const uint8_t *fp4_row, const uint8_t *scale_row, int d, int scale_fmt) {
    uint8_t byte = fp4_row[d / 2];
    uint8_t code = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    uint8_t sb = scale_row[d / group_size(scale_fmt)];
    if (scale_fmt == 0) return ldexp(orc_e2m1_decode(code), (int)sb - 127);
    return orc_e2m1_decode(code) * orc_e4m3_decode(sb);
}

/* Element c of one stored indexer key: bf16 (idx_dtype 0), e4m3 (1), or MXFP4
 * (2: codes two per byte, element 2i in the low nibble, and one E8M0 scale byte
 * per 32 elements in scale_row). */
static double idx_key_element(const uint8_t *key_row, const uint8_t *scale_row, int idx_dtype, int c) {
    if (idx_dtype == 0) {
        uint16_t bits;
        memcpy(&bits, key_row + 2 * c, 2);
        return orc_bf16_decode(bits);
    }
    if (idx_dtype == 2) {
        uint8_t byte = key_row[c / 2];
        uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        return ldexp(orc_e2m1_decode(code), (int)scale_row[c / 32] - 127);
    }
    return orc_e4m3_decode(key_row[c]);
}

/* Bytes of one stored indexer key (codes only for MXFP4; its scales are a plane of their own). */
static size_t idx_key_bytes(int idx_dtype, int dI) {
    return idx_dtype == 0 ? (size_t)dI * 2 : idx_dtype == 2 ? (size_t)dI / 2 : (size_t)dI;
}

/* ======================================================================
 * a1 + a2: gated block pooling, then quantization of the pooled block
 * ====================================================================== */
int orc_compress(int B, int D, int dI, int m, int idx_dtype, int scale_fmt, int cap,
                 const uint16_t *kv_tok, const uint16_t *idx_tok, const float *w_g,
                 const int32_t *tok_offsets, int32_t *n_blocks,
                 uint8_t *fp4, uint8_t *scale, uint8_t *idx_key, uint8_t *idx_key_scale, float *pooled_out,
                 float *pooled_idx_out) {
    int status = 0;
    for (int b = 0; b < B; ++b) {
        int count = tok_offsets[b + 1] - tok_offsets[b];
        if (count % m != 0 || n_blocks[b] + count / m > cap) {
            status = -1;
            continue;
        }
        int nb = count / m;
#pragma omp parallel for schedule(dynamic, 16)
        for (int jb = 0; jb < nb; ++jb) {
            int j = n_blocks[b] + jb;                        /* destination block */
            long t0 = (long)tok_offsets[b] + (long)jb * m;   /* first token of the block */
            double *g = malloc(sizeof(double) * m);
            double *alpha = malloc(sizeof(double) * m);
            float *e = malloc(sizeof(float) * D);
            /* gate logit of each token: g_t = sum_d kv_t[d] * w_g[d] */
            for (int t = 0; t < m; ++t) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d)
                    acc += orc_bf16_decode(kv_tok[(t0 + t) * D + d]) * (double)w_g[d];
                g[t] = acc;
            }
            /* softmax over the block's m tokens */
            double mu = g[0];
            for (int t = 1; t < m; ++t) mu = fmax(mu, g[t]);
            double den = 0.0;
            for (int t = 0; t < m; ++t) den += exp(g[t] - mu);
            for (int t = 0; t < m; ++t) alpha[t] = exp(g[t] - mu) / den;
            /* pooled main KV, rounded to float32 (the precision quantization decides in) */
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int t = 0; t < m; ++t) acc += alpha[t] * orc_bf16_decode(kv_tok[(t0 + t) * D + d]);
                e[d] = (float)acc;
            }
            size_t row = (size_t)b * cap + j;
            if (pooled_out) memcpy(pooled_out + row * D, e, sizeof(float) * D);
            /* FP4: one scale byte per group (E8M0 per 32 or E4M3 per 16), two codes per byte */
            int gs = group_size(scale_fmt);
            for (int grp = 0; grp < D / gs; ++grp) {
                uint8_t codes[32], sb;
                if (scale_fmt == 0)
                    orc_mxfp4_quantize_group(e + gs * grp, codes, &sb);
                else
                    orc_e4m3x16_quantize_group(e + gs * grp, codes, &sb);
                scale[row * (D / gs) + grp] = sb;
                for (int i = 0; i < gs / 2; ++i)
                    fp4[row * (D / 2) + (gs / 2) * grp + i] = (uint8_t)(codes[2 * i] | (codes[2 * i + 1] << 4));
            }
            /* pooled indexer key with the same gate, stored as bf16, e4m3, or MXFP4
             * (one E8M0 scale per 32 channels, the main KV's rule) */
            if (idx_key) {
                uint8_t *dst = idx_key + row * idx_key_bytes(idx_dtype, dI);
                float *kfs = malloc(sizeof(float) * dI);
                for (int c = 0; c < dI; ++c) {
                    double acc = 0.0;
                    for (int t = 0; t < m; ++t) acc += alpha[t] * orc_bf16_decode(idx_tok[(t0 + t) * dI + c]);
                    float kf = (float)acc;
                    kfs[c] = kf;
                    if (pooled_idx_out) pooled_idx_out[row * dI + c] = kf;
                    if (idx_dtype == 0) {
                        uint16_t bits = orc_bf16_encode(kf);
                        memcpy(dst + 2 * c, &bits, 2);
                    } else if (idx_dtype == 1) {
                        dst[c] = orc_e4m3_encode((double)kf);
                    }
                }
                if (idx_dtype == 2) {
                    for (int grp = 0; grp < dI / 32; ++grp) {
                        uint8_t codes[32], sb;
                        orc_mxfp4_quantize_group(kfs + 32 * grp, codes, &sb);
                        idx_key_scale[row * (dI / 32) + grp] = sb;
                        for (int i2 = 0; i2 < 16; ++i2)
                            dst[16 * grp + i2] = (uint8_t)(codes[2 * i2] | (codes[2 * i2 + 1] << 4));
                    }
                }
                free(kfs);
            }
            free(g);
            free(alpha);
            free(e);
        }
        n_blocks[b] += nb;
    }
    return status;
}

/* ======================================================================
 * a3: indexer scores
 * ====================================================================== */
static int request_of(const int32_t *q_offsets, int B, int i) {
    for (int b = 0; b < B; ++b)
        if (i >= q_offsets[b] && i < q_offsets[b + 1]) return b;
    return -1;
}

static int visible_blocks(int pos, int m, int filled) {
    long v = ((long)pos + 1) / m;
    if (v > filled) v = filled;
    if (v < 0) v = 0;
    return (int)v;
}

/* The indexer query as the scores use it: the bf16 value itself, or, with MXFP4
 * keys, its MXFP4 quantization per 32 channels of each head (the main KV's rule),
 * dequantized. qv: [H_I][dI] doubles of query i. */
static void index_query(int H_I, int dI, int idx_dtype, const uint16_t *q_row, double *qv) {
    for (int h = 0; h < H_I; ++h) {
        for (int c = 0; c < dI; ++c) qv[h * dI + c] = orc_bf16_decode(q_row[h * dI + c]);
        if (idx_dtype != 2) continue;
        for (int grp = 0; grp < dI / 32; ++grp) {
            float v[32];
            uint8_t codes[32], sb;
            for (int c = 0; c < 32; ++c) v[c] = (float)qv[h * dI + 32 * grp + c];
            orc_mxfp4_quantize_group(v, codes, &sb);
            for (int c = 0; c < 32; ++c) qv[h * dI + 32 * grp + c] = ldexp(orc_e2m1_decode(codes[c]), (int)sb - 127);
        }
    }
}

void orc_index_scores(int B, int Nq, int H_I, int dI, int idx_dtype, int m, int cap,
                      const uint8_t *idx_key, const uint8_t *idx_key_scale, const int32_t *n_blocks,
                      const int32_t *q_offsets, const int32_t *q_pos,
                      const uint16_t *q_idx, const float *w,
                      float *scores, int32_t *n_vis_out) {
    size_t kb = idx_key_bytes(idx_dtype, dI);
    double *qv = malloc(sizeof(double) * (size_t)H_I * dI);
    for (int i = 0; i < Nq; ++i) {
        int b = request_of(q_offsets, B, i);
        int n_vis = (b < 0) ? 0 : visible_blocks(q_pos[i], m, n_blocks[b]);
        if (n_vis_out) n_vis_out[i] = n_vis;
        index_query(H_I, dI, idx_dtype, q_idx + (size_t)i * H_I * dI, qv);
#pragma omp parallel for schedule(static)
        for (int j = 0; j < cap; ++j) {
            if (j >= n_vis) {
                scores[(size_t)i * cap + j] = -INFINITY;
                continue;
            }
            const uint8_t *key = idx_key + ((size_t)b * cap + j) * kb;
            const uint8_t *ksc = idx_dtype == 2 ? idx_key_scale + ((size_t)b * cap + j) * (dI / 32) : NULL;
            double s = 0.0;
            for (int h = 0; h < H_I; ++h) {
                double dot = 0.0;
                for (int c = 0; c < dI; ++c)
                    dot += qv[h * dI + c] * idx_key_element(key, ksc, idx_dtype, c);
                s += (double)w[(size_t)i * H_I + h] * fmax(dot, 0.0);
            }
            float sf = (float)s;
            if (sf == 0.0f) sf = 0.0f; /* -0 -> +0 */
            scores[(size_t)i * cap + j] = sf;
        }
    }
    free(qv);
}

/* ======================================================================
 * a4: top-k, ties to the lower block index, output ascending
 * ====================================================================== */
typedef struct { float s; int32_t j; } scored_t;

static int by_score_then_index(const void *pa, const void *pb) {
    const scored_t *a = pa, *b = pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

static int ascending_int(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

void orc_topk(int Nq, int cap, int k, const float *scores, const int32_t *n_vis, int32_t *sel_idx) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < Nq; ++i) {
        int n = n_vis[i];
        scored_t *list = malloc(sizeof(scored_t) * (n > 0 ? n : 1));
        for (int j = 0; j < n; ++j) {
            list[j].s = scores[(size_t)i * cap + j];
            list[j].j = j;
        }
        qsort(list, n, sizeof(scored_t), by_score_then_index);
        int take = n < k ? n : k;
        int32_t *row = sel_idx + (size_t)i * k;
        for (int r = 0; r < take; ++r) row[r] = list[r].j;
        qsort(row, take, sizeof(int32_t), ascending_int);
        for (int r = take; r < k; ++r) row[r] = -1;
        free(list);
    }
}

/* ======================================================================
 * Hierarchical indexer (DeepSeek-V4.1-Flash podcast transcript, cue 14) and
 * CSA2 Reindex mode (cue 12)
 * ====================================================================== */

/* First stage, run with the Full-mode layer's scores: group the visible
 * entries into blocks of G consecutive entries (block b holds entries
 * [G b, G b + G) below n_vis), score each block by the largest score of its
 * entries, and keep the P blocks with the largest block score, ties to the
 * lower block index; pool_blk[i] lists them ascending, padded with -1. */
void orc_index_pool(int Nq, int cap, int G, int P, const float *scores, const int32_t *n_vis, int32_t *pool_blk) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < Nq; ++i) {
        int n = n_vis[i];
        int nb = (n + G - 1) / G;
        scored_t *list = malloc(sizeof(scored_t) * (nb > 0 ? nb : 1));
        for (int b = 0; b < nb; ++b) {
            float best = -INFINITY;
            for (int j = G * b; j < G * b + G && j < n; ++j) best = fmaxf(best, scores[(size_t)i * cap + j]);
            list[b].s = best;
            list[b].j = b;
        }
        qsort(list, nb, sizeof(scored_t), by_score_then_index);
        int take = nb < P ? nb : P;
        int32_t *row = pool_blk + (size_t)i * P;
        for (int r = 0; r < take; ++r) row[r] = list[r].j;
        qsort(row, take, sizeof(int32_t), ascending_int);
        for (int r = take; r < P; ++r) row[r] = -1;
        free(list);
    }
}

/* Reindex-mode selection: the layer's own scores, restricted to the visible
 * entries of query i's pool blocks; the min(k, |pool entries|) largest, ties
 * to the lower entry index, ascending, padded with -1. */
void orc_reindex_topk(int Nq, int cap, int G, int P, int k, const float *scores, const int32_t *n_vis,
                      const int32_t *pool_blk, int32_t *sel_idx) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < Nq; ++i) {
        int n = n_vis[i];
        scored_t *list = malloc(sizeof(scored_t) * ((size_t)G * P + 1));
        int cnt = 0;
        for (int r = 0; r < P; ++r) {
            int b = pool_blk[(size_t)i * P + r];
            if (b < 0) continue;
            for (int j = G * b; j < G * b + G && j < n; ++j) {
                list[cnt].s = scores[(size_t)i * cap + j];
                list[cnt].j = j;
                ++cnt;
            }
        }
        qsort(list, cnt, sizeof(scored_t), by_score_then_index);
        int take = cnt < k ? cnt : k;
        int32_t *row = sel_idx + (size_t)i * k;
        for (int r = 0; r < take; ++r) row[r] = list[r].j;
        qsort(row, take, sizeof(int32_t), ascending_int);
        for (int r = take; r < k; ++r) row[r] = -1;
        free(list);
    }
}

/* ======================================================================
 * a5 + a6 (+ a7): one joint softmax over compressed entries and window rows
 * ====================================================================== */

/* Softmax attention of one query head over n entries given as rows of x
 * (n x D, double). Writes out[D] and returns the log-sum-exp. */
static double attend_rows(const double *qh, const double *x, int n, int D, double softmax_scale, double *out) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (n == 0) return -INFINITY;
    double *logit = malloc(sizeof(double) * n);
    double mu = -INFINITY;
    for (int r = 0; r < n; ++r) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qh[d] * x[(size_t)r * D + d];
        logit[r] = softmax_scale * dot;
        mu = fmax(mu, logit[r]);
    }
    double den = 0.0;
    for (int r = 0; r < n; ++r) den += exp(logit[r] - mu);
    for (int r = 0; r < n; ++r) {
        double p = exp(logit[r] - mu) / den;
        for (int d = 0; d < D; ++d) out[d] += p * x[(size_t)r * D + d];
    }
    free(logit);
    return mu + log(den);
}

/* Gather the entry rows of query i: compressed blocks (dequantized) then window rows. */
static int gather_entries(int D, int cap, int b, const int32_t *blocks, int nblk,
                          const uint8_t *fp4, const uint8_t *scale, int scale_fmt,
                          const uint16_t *win_kv, int64_t wstart, int wlen, double *x) {
    int n = 0;
    for (int r = 0; r < nblk; ++r) {
        int j = blocks[r];
        if (j < 0) continue;
        const uint8_t *frow = fp4 + ((size_t)b * cap + j) * (D / 2);
        const uint8_t *srow = scale + ((size_t)b * cap + j) * (D / group_size(scale_fmt));
        for (int d = 0; d < D; ++d) x[(size_t)n * D + d] = fp4_element(frow, srow, d, scale_fmt);
        ++n;
    }
    for (int t = 0; t < wlen; ++t) {
        for (int d = 0; d < D; ++d) x[(size_t)n * D + d] = orc_bf16_decode(win_kv[(wstart + t) * D + d]);
        ++n;
    }
    return n;
}

static void attend_query(int i, int H, int D, int n, const double *x, const uint16_t *q,
                         double softmax_scale, double *out, double *lse) {
    double *qh = malloc(sizeof(double) * D);
    for (int h = 0; h < H; ++h) {
        for (int d = 0; d < D; ++d) qh[d] = orc_bf16_decode(q[((size_t)i * H + h) * D + d]);
        double l = attend_rows(qh, x, n, D, softmax_scale, out + ((size_t)i * H + h) * D);
        if (lse) lse[(size_t)i * H + h] = l;
    }
    free(qh);
}

void orc_csa_attend(int B, int Nq, int H, int D, int cap, int k,
                    const uint8_t *fp4, const uint8_t *scale, int scale_fmt,
                    const int32_t *q_offsets, const uint16_t *q, const int32_t *sel_idx,
                    const uint16_t *win_kv, const int64_t *win_start, const int32_t *win_len,
                    double softmax_scale, double *out, double *lse) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < Nq; ++i) {
        int b = request_of(q_offsets, B, i);
        int wlen = win_len ? win_len[i] : 0;
        double *x = malloc(sizeof(double) * (size_t)(k + wlen + 1) * D);
        int n = gather_entries(D, cap, b, sel_idx + (size_t)i * k, b < 0 ? 0 : k, fp4, scale, scale_fmt,
                               win_kv, win_start ? win_start[i] : 0, wlen, x);
        attend_query(i, H, D, n, x, q, softmax_scale, out, lse);
        free(x);
    }
}

void orc_hca_attend(int B, int Nq, int H, int D, int m, int cap,
                    const uint8_t *fp4, const uint8_t *scale, int scale_fmt, const int32_t *n_blocks,
                    const int32_t *q_offsets, const int32_t *q_pos, const uint16_t *q,
                    const uint16_t *win_kv, const int64_t *win_start, const int32_t *win_len,
                    double softmax_scale, double *out, double *lse) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < Nq; ++i) {
        int b = request_of(q_offsets, B, i);
        int n_vis = (b < 0) ? 0 : visible_blocks(q_pos[i], m, n_blocks[b]);
        int wlen = win_len ? win_len[i] : 0;
        /* every visible block, in order: no indexer, no selection */
        int32_t *all = malloc(sizeof(int32_t) * (n_vis > 0 ? n_vis : 1));
        for (int j = 0; j < n_vis; ++j) all[j] = j;
        double *x = malloc(sizeof(double) * (size_t)(n_vis + wlen + 1) * D);
        int n = gather_entries(D, cap, b, all, n_vis, fp4, scale, scale_fmt, win_kv, win_start ? win_start[i] : 0, wlen, x);
        attend_query(i, H, D, n, x, q, softmax_scale, out, lse);
        free(x);
        free(all);
    }
}
