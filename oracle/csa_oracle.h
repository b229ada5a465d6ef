/*
 * csa_oracle.h -- plain CPU reference ("oracle") for compressed sparse attention
 * (CSA), heavily compressed attention (HCA) and the uncompressed sliding window,
 * over a KV cache stored as MXFP4.
 *
 * TEST INFRASTRUCTURE ONLY. This code exists to check the CUDA library against
 * the method's definition. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load it. It shares no code, header, table or constant
 * with the CUDA path, and the CUDA path never calls it.
 *
 * Sources (page title, section):
 *   "Frontier Architecture Decoding Notes (4): DeepSeek V4", section 1
 *       (CSA: 4-token blocks + top-k over blocks; HCA: compression up to 128x;
 *        128-token uncompressed window; "precise near, compressed far").
 *   DeepSeek-V4.1-Flash podcast transcript, cue 12 (indexer keys projected from
 *       the main KV, indexer query, top-k selection) and cue 16 (main KV in
 *       MXFP4, E2M1 elements, dequantized right before attention).
 *   Where the pages are silent the readings are the ones listed in the
 *   repository's design notes: softmax-gated pooling with a per-token scalar
 *   gate, score = sum_h w_h * ReLU(q_h . k), ties to the lower block index,
 *   one joint softmax over selected entries plus window, E8M0 scale per 32.
 *   The page's own scale format (one E4M3 scale per 16 elements, cue 16) is
 *   the second supported format.
 *
 * Precision: every floating-point step is carried out in double. Where a float
 * result decides an integer (an MXFP4 code or scale, an E4M3/BF16 byte pattern,
 * a top-k membership) the double result is first rounded to float32, the
 * precision the GPU kernels take that decision in.
 *
 * All bf16 tensors are passed as uint16_t bit patterns.
 */
#ifndef CSA_ORACLE_H
#define CSA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- number formats -------------------------------------------------- */
double   orc_bf16_decode(uint16_t bits);
uint16_t orc_bf16_encode(float x);            /* round to nearest even       */
double   orc_e2m1_decode(uint8_t code);       /* low 4 bits used              */
uint8_t  orc_e2m1_encode(double x);           /* RNE, saturate at +-6, keeps sign */
double   orc_e4m3_decode(uint8_t code);       /* OCP FP8 E4M3 (no inf)        */
uint8_t  orc_e4m3_encode(double x);           /* RNE, saturate at +-448       */
/* One 32-element MXFP4 group: codes[i] holds the E2M1 code of v[i] (one per
 * byte, not packed); *scale_byte is the E8M0 byte (exponent + 127). */
void     orc_mxfp4_quantize_group(const float *v, uint8_t *codes, uint8_t *scale_byte);
/* One 16-element group of the E4M3-scaled variant: *scale_byte is the E4M3
 * byte of amax/6 (RNE, saturating); codes[i] the E2M1 code of v[i] / scale. */
void     orc_e4m3x16_quantize_group(const float *v, uint8_t *codes, uint8_t *scale_byte);

/* ---- a1+a2: gated block pooling + quantization ------------------------ */
/* For each request b, tokens [tok_offsets[b], tok_offsets[b+1]) are pooled
 * m at a time into blocks appended at n_blocks[b] (n_blocks is updated).
 * kv_tok:  [T_total][D] bf16, idx_tok: [T_total][dI] bf16 (may be NULL when
 * idx_key is NULL), w_g: [D] float.
 * scale_fmt selects the scale format: 0 = one E8M0 byte per 32 elements
 * (OCP MXFP4), 1 = one E4M3 byte per 16 elements.
 * Output planes (per request stride = cap blocks):
 *   fp4   [B][cap][D/2]  two codes per byte, element 2i in the low nibble
 *   scale [B][cap][D/32] E8M0 bytes, or [B][cap][D/16] E4M3 bytes
 *   idx_key [B][cap][dI] bf16 (idx_dtype 0) or e4m3 (idx_dtype 1), or
 *           [B][cap][dI/2] MXFP4 codes (idx_dtype 2: the pooled key quantized
 *           like the main KV, one E8M0 scale per 32 channels, the scales in
 *           idx_key_scale [B][cap][dI/32]; NULL otherwise)
 * Optional pooled_out [B][cap][D] float and pooled_idx_out [B][cap][dI] float
 * receive the float32 pooled values before quantization (NULL to skip).
 * Returns 0, or -1 when a request's token count is not a multiple of m or
 * would overflow the capacity (nothing is written for that request). */
int orc_compress(int B, int D, int dI, int m, int idx_dtype, int scale_fmt, int cap,
                 const uint16_t *kv_tok, const uint16_t *idx_tok, const float *w_g,
                 const int32_t *tok_offsets, int32_t *n_blocks,
                 uint8_t *fp4, uint8_t *scale, uint8_t *idx_key, uint8_t *idx_key_scale, float *pooled_out,
                 float *pooled_idx_out);

/* ---- a3: indexer scores ---------------------------------------------- */
/* Query i belongs to request req(i) given by q_offsets [B+1]. Visible blocks:
 * n_vis = min(floor((q_pos[i]+1)/m), n_blocks[req]). scores[i][j] for
 * j < n_vis is the float32 rounding of
 *     sum_h w[i][h] * max(0, sum_c q_idx[i][h][c] * key_j[c]),
 * with -0 mapped to +0; entries j >= n_vis are set to -INFINITY.
 * With MXFP4 keys (idx_dtype 2, scales in idx_key_scale) the query is first
 * quantized the same way, per 32 channels of each head, and dequantized; the
 * product of two MXFP4 values is then exact and the sums run in double.
 * scores has row stride cap. n_vis_out[i] receives n_vis (may be NULL). */
void orc_index_scores(int B, int Nq, int H_I, int dI, int idx_dtype, int m, int cap,
                      const uint8_t *idx_key, const uint8_t *idx_key_scale, const int32_t *n_blocks,
                      const int32_t *q_offsets, const int32_t *q_pos,
                      const uint16_t *q_idx, const float *w,
                      float *scores, int32_t *n_vis_out);

/* ---- a4: top-k -------------------------------------------------------- */
/* Per query: the min(k, n_vis) blocks with the largest score, ties to the
 * lower block index, written in ascending block order, padded with -1. */
void orc_topk(int Nq, int cap, int k, const float *scores, const int32_t *n_vis,
              int32_t *sel_idx);

/* ---- hierarchical indexer pool and CSA2 Reindex selection -------------- */
/* Pool (Full-mode layer): blocks of G consecutive visible entries scored by
 * their largest score; the P best blocks (ties to the lower block index),
 * ascending, -1 padded, into pool_blk [Nq][P]. */
void orc_index_pool(int Nq, int cap, int G, int P, const float *scores, const int32_t *n_vis, int32_t *pool_blk);
/* Reindex: top-k (ties to the lower entry index) among the visible entries of
 * the pool blocks only, ascending, -1 padded, into sel_idx [Nq][k]. scores are
 * the Reindex layer's own scores (row stride cap). */
void orc_reindex_topk(int Nq, int cap, int G, int P, int k, const float *scores, const int32_t *n_vis,
                      const int32_t *pool_blk, int32_t *sel_idx);

/* ---- a5+a6: CSA joint attention --------------------------------------- */
/* For query i and head h, the entries are the dequantized cache blocks listed
 * in sel_idx[i][0..k) (negative entries ignored) followed by the window rows
 * win_kv[win_start[i] + t], t < win_len[i]. Logits are
 * softmax_scale * <q[i][h], x>; out[i][h] = sum softmax * x and
 * lse[i][h] = natural log of sum exp(logit). An empty entry set gives out = 0
 * and lse = -INFINITY. The cache planes are read in the scale format
 * scale_fmt (as for orc_compress). q: [Nq][H][D] bf16; out: [Nq][H][D] double;
 * lse: [Nq][H] double (may be NULL). */
void orc_csa_attend(int B, int Nq, int H, int D, int cap, int k,
                    const uint8_t *fp4, const uint8_t *scale, int scale_fmt,
                    const int32_t *q_offsets, const uint16_t *q, const int32_t *sel_idx,
                    const uint16_t *win_kv, const int64_t *win_start, const int32_t *win_len,
                    double softmax_scale, double *out, double *lse);

/* ---- a7: HCA dense attention ------------------------------------------ */
/* As orc_csa_attend, but the compressed entries are all visible blocks
 * j < min(floor((q_pos[i]+1)/m), n_blocks[req]) in order. */
void orc_hca_attend(int B, int Nq, int H, int D, int m, int cap,
                    const uint8_t *fp4, const uint8_t *scale, int scale_fmt, const int32_t *n_blocks,
                    const int32_t *q_offsets, const int32_t *q_pos, const uint16_t *q,
                    const uint16_t *win_kv, const int64_t *win_start, const int32_t *win_len,
                    double softmax_scale, double *out, double *lse);

/* Number of OpenMP threads the oracle's parallel loops use. */
int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
