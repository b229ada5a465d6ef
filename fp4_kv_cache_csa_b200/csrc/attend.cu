// attend.cu -- rows a5 + a6 + a7 + a8: dequantize the attended MXFP4 entries
// right before attention, one joint softmax over compressed entries and the
// uncompressed window, split over CTAs with a log-sum-exp merge.
//
// Sources: "Frontier Architecture Decoding Notes (4): DeepSeek V4", section 1
// (CSA attends the top-k compressed entries, HCA every entry of a 128x
// compressed cache, plus the latest 128 tokens uncompressed);
// DeepSeek-V4.1-Flash podcast transcript, cue 16 (MXFP4 main KV, dequantized
// right before attention). All heads share one latent vector per entry that is
// both key and value (cue 8: a shared latent), so the heads x D by D x entries
// products are dense contractions and run on the tcgen05 tensor cores.
//
// Design (one CTA per SM, 256 threads; entry j of a 128-entry tile belongs to
// threads j and j + 128, which take one half of its D channels each):
//   * Work = the flat list of 128-entry tiles of all queries (compressed tiles
//     first, then window tiles), cut into equal contiguous ranges, one per CTA.
//     A CTA whose range covers a whole query writes the output directly;
//     otherwise it writes an unnormalized partial, and attend_merge_kernel
//     (one CTA per query and 8-head slice) combines the partials.
//   * Operands are fp16 in shared memory. Entry j is stored as
//     E'_j = e_j * 2^-R_j with R_j the largest E8M0 exponent of the row (or the
//     exponent of max|x| for a window row): every E2M1 x 2^X value is exact in
//     fp16 within 2^24 of the row's largest group. With one E4M3 scale per 16
//     elements (the cache's other format) every E2M1 x E4M3 value is exact
//     in fp16 as it stands, so E'_j = e_j and R_j = 0. The query is stored as
//     q * 2^-sQ (exact for bf16 values within 2^31 of max|q|).
//   * S^T = E' Q'^T: M = 128 entries (TMEM lanes), N = 64 heads (columns).
//   * Softmax in the log2 domain, thread (j, half) holding 32 head logits of
//     entry j: u = log2(e) * scale * <q,e_j> + R_j. Each head h keeps a
//     reference rho_h, set from the first tile's maximum and raised (with the
//     TMEM accumulator rescaled) only when some logit exceeds it by more than
//     8, so the per-head maximum over entries (a cross-thread reduction) is
//     taken only then; P'_{j,h} = 2^(u - rho_h) <= 256 is stored in fp16,
//     folding the row factor 2^R_j back in. The row sums stay per thread and
//     are reduced once per segment.
//   * O^T += E'^T P': M = 128 latent channels per d-tile, N = 64 heads, K = 16
//     entries per MMA; O^T lives in TMEM for the whole segment. The PV MMAs of
//     the low and high channel halves complete on separate barriers, so each
//     half of the next tile is dequantized as soon as its channels are free.
//   * out = O / l and lse = ln 2 * (rho + log2 l), l = sum_j 2^(lambda_j - rho).
// Compressed rows are loaded into registers one tile ahead (their selected
// indices two tiles ahead); window tiles (bf16) are copied with cp.async into
// the operand buffer and converted in place.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "tc_util.cuh"

namespace csa {

namespace {

constexpr int kTile = 128;
constexpr int kSchedSmemQueries = 1024;  // the schedule searches its prefixes in shared memory up to here
constexpr int kMaxAttendCtas = 256;      // ... and the CTA ranges up to this many CTAs
constexpr int kHeads = 64;
constexpr int kThreads = 256;
// Relative cost of the work the CTAs share out (global-timer traces of every CTA on
// B200 at D = 512: a compressed tile ~5.2-6.3 us, a window tile ~12.4 us -- bf16 rows
// 4x the bytes, copied and converted in place -- and each query a CTA starts ~10 us:
// its Q' copy, the first tile's cold loads, the final PV wait, the output or partial
// write). The flat tile list is cut into equal shares of these units, not of tiles.
constexpr long long kCTileCost = 100;
constexpr long long kWTileCost = 220;
constexpr long long kStartCost = 170;

template <int D>
struct Cfg {
    static constexpr int DT = D / 128;                    // O^T d-tiles
    static constexpr int GPR = D / 32;                    // MXFP4 groups per row
    static constexpr int CODE_V = D / 32;                 // 16-byte code loads per row (D/2 bytes)
    static constexpr int HALF_V = CODE_V / 2;             // ... per half row
    static constexpr int E_BYTES = kTile * D * 2;
    static constexpr int Q_BYTES = kHeads * D * 2;
    static constexpr int P_BYTES = kTile * kHeads * 2;
    static constexpr int KREG = kTile * 128;              // bytes per k-chunk region of E'
    static constexpr int QREG = kHeads * 128;             // bytes per k-chunk region of Q'
    static constexpr int TMEM_USED = kHeads + DT * kHeads;
    static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static constexpr int MISC_BYTES = 4096;
    static constexpr int SMEM = 1024 + E_BYTES + Q_BYTES + P_BYTES + MISC_BYTES;
};

// ---------------------------------------------------------------- arguments
// Per-query schedule record (written by the schedule kernel's CTA 0).
struct QInfo {
    int4 a;        // request, entry slots, compressed tiles, window rows
    int4 b;        // filled blocks of the request, 0, 0, 0
    longlong2 t;   // the query's tiles [t0, t1) in the flat tile list
};

struct AttArgs {
    const uint8_t *fp4, *scale;      // cache planes
    const int32_t *sel_idx;          // CSA: [Nq][topk]; HCA: null
    const __nv_bfloat16 *win_kv;     // [rows][D] or null
    const int64_t *win_start;
    float *out, *lse;
    int32_t *status;
    // schedule (workspace)
    const QInfo *qinfo;              // [Nq]
    const long long *tprefix;        // [Nq+1]
    const int32_t *cta_q;            // [G] first query of each CTA's range
    const long long *cta_t;          // [G+1] first tile of each CTA's range
    const int32_t *sq;               // [Nq] query scale exponents
    const uint8_t *qimg;             // [Nq][Q_BYTES] Q' images
    float *part_o, *part_rho, *part_l;  // [2G][64][D], [2G][64], [2G][64]
    int Nq, H, cap, topk;
    float scale_log2;                // softmax_scale * log2(e)
};

// Scale formats of the cache (template argument SF of the kernel).
constexpr int kScaleE8M0x32 = 0;  // one E8M0 byte per 32 elements
constexpr int kScaleE4M3x16 = 1;  // one E4M3 byte per 16 elements

// Prefetch of this thread's half of one compressed entry: its codes and the
// scale bytes it needs -- for E8M0 scales all D/32 bytes of the row (R_j is
// the maximum over the whole row), for E4M3 scales the D/32 bytes of its half.
template <int D>
struct RowRegs {
    uint4 code[Cfg<D>::HALF_V];
    uint4 sc;
    int valid;
};

// Everything the tile loop needs about one tile, gathered ahead of time so
// that no dependent global load sits on the per-tile critical path.
struct TileRef {
    int i;             // query
    int lt;            // local tile index within the query
    int win;           // 1: window tile
    int b;             // request of the query
    int nent;          // compressed entry slots of the query
    int ctiles;        // compressed tiles of the query
    int wlen;          // window rows of the query
    int nblk;          // filled blocks of request b (bound of a selected index)
    long long t0, t1;  // the query's tiles [t0, t1) in the flat tile list
};

__device__ __forceinline__ TileRef query_ref(const AttArgs &a, int i, long long t) {
    const QInfo *qi = a.qinfo + i;
    const int4 x = qi->a;
    const int4 y = qi->b;
    const longlong2 z = qi->t;
    TileRef r;
    r.i = i;
    r.b = x.x;
    r.nent = x.y;
    r.ctiles = x.z;
    r.wlen = x.w;
    r.nblk = y.x;
    r.t0 = z.x;
    r.t1 = z.y;
    r.lt = (int)(t - r.t0);
    r.win = r.lt >= r.ctiles;
    return r;
}

// The tile after r (t_next = its flat index): the same query, or the next one with tiles.
__device__ __forceinline__ TileRef advance(const AttArgs &a, const TileRef &r, long long t_next) {
    if (t_next < r.t1) {
        TileRef n = r;
        n.lt += 1;
        n.win = n.lt >= n.ctiles;
        return n;
    }
    int i = r.i + 1;
    while (i < a.Nq - 1 && a.tprefix[i + 1] == a.tprefix[i]) ++i;  // skip queries without tiles
    return query_ref(a, i, t_next);
}

// This thread's row of a compressed tile: the raw selected index (CSA) or the
// slot itself (HCA); -1 for padding rows. Checked against the bound at use.
__device__ __forceinline__ int row_block_raw(const AttArgs &a, const TileRef &tr) {
    const int slot = tr.lt * kTile + (int)(threadIdx.x & (kTile - 1));
    if (tr.win || slot >= tr.nent) return -1;
    return a.sel_idx ? a.sel_idx[(size_t)tr.i * a.topk + slot] : slot;
}

// Issue the loads of this thread's row of a compressed tile.
template <int D, int SF>
__device__ __forceinline__ void prefetch_row(const AttArgs &a, const TileRef &tr, int blk, RowRegs<D> &rr) {
    rr.valid = 0;
    if (blk >= 0 && (blk >= tr.nblk || blk >= a.cap)) {
        flag(a.status, CSA_DEV_BAD_INDEX);
        blk = -1;
    }
    if (blk >= 0) {
        const size_t row = (size_t)tr.b * a.cap + blk;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.fp4 + row * (D / 2)) + (threadIdx.x >> 7) * Cfg<D>::HALF_V;
#pragma unroll
        for (int v = 0; v < Cfg<D>::HALF_V; ++v) rr.code[v] = __ldg(src + v);
        // D/32 scale bytes either way: the whole row (E8M0) or this half (E4M3, D/16 per row)
        const uint8_t *sp = SF == kScaleE4M3x16 ? a.scale + row * (D / 16) + (threadIdx.x >> 7) * (D / 32)
                                                : a.scale + row * (D / 32);
        if constexpr (D / 32 >= 16) {
            rr.sc = __ldg(reinterpret_cast<const uint4 *>(sp));
        } else {
            rr.sc = make_uint4(__ldg(reinterpret_cast<const uint32_t *>(sp)), 0, 0, 0);
        }
        rr.valid = 1;
    }
}

// Byte k of the row's scale bytes.
template <int D>
__device__ __forceinline__ int scale_byte(const RowRegs<D> &rr, int k) {
    const uint32_t w = k < 4 ? rr.sc.x : k < 8 ? rr.sc.y : k < 12 ? rr.sc.z : rr.sc.w;
    return (int)((w >> (8 * (k & 3))) & 0xFF);
}

// Swizzled byte offset of 16-byte chunk kc (channels 8kc..8kc+7) of row j of E'.
template <int D>
__device__ __forceinline__ uint32_t e_chunk_off(int j, int kc) {
    return (uint32_t)((kc >> 3) * Cfg<D>::KREG + (j >> 3) * 1024 + (j & 7) * 128 + (((kc & 7) ^ (j & 7)) << 4));
}

// Dequantize one quarter of this thread's prefetched row into E' (fp16): the
// first (part 0) or second (part 1) half of its channel half. Part 0 of all
// threads covers channels [0, D/4) and [D/2, 3D/4) -- the "low" channel set,
// which the S and PV products of a tile consume first; part 1 the rest.
// E8M0 scales: E'_j = e_j * 2^-R_j, and part 0 returns R_j (the row's largest
// E8M0 exponent). E4M3 scales: every E2M1 x E4M3 product is exact in fp16 (at
// most 6 significant bits, magnitudes 2^-10 .. 2688), so E' = e and R_j = 0.
// Invalid rows are zero.
template <int D, int SF>
__device__ __forceinline__ int dequant_part(const RowRegs<D> &rr, uint8_t *E, int part) {
    constexpr int GQ = Cfg<D>::GPR / 4;                     // 32-element groups per quarter row
    const int j = threadIdx.x & (kTile - 1);
    const int g0 = (threadIdx.x >> 7) * (Cfg<D>::GPR / 2);  // first 32-element group of this half
    if (!rr.valid) {
#pragma unroll
        for (int kc = 4 * (g0 + part * GQ); kc < 4 * (g0 + part * GQ + GQ); ++kc)
            *reinterpret_cast<uint4 *>(E + e_chunk_off<D>(j, kc)) = make_uint4(0, 0, 0, 0);
        return 0;
    }
    if constexpr (SF == kScaleE4M3x16) {
#pragma unroll
        for (int gq = 0; gq < GQ; ++gq) {
            const int gl = part * GQ + gq;
            const int g = g0 + gl;
            const uint32_t *w = reinterpret_cast<const uint32_t *>(&rr.code[gl]);
            // code bytes 0..7 of this uint4 are 16-element group 2 gl of the half, 8..15 group 2 gl + 1
            __half2 s2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __half_raw hr = __nv_cvt_fp8_to_halfraw(
                    (__nv_fp8_storage_t)scale_byte<D>(rr, 2 * gl + h), __NV_E4M3);
                s2[h] = __halves2half2(__half(hr), __half(hr));
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t outw[4];
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    __half2_raw hr =
                        __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((w[c] >> (8 * bb)) & 0xFF), __NV_E2M1);
                    __half2 h = __hmul2(*reinterpret_cast<__half2 *>(&hr), s2[c >> 1]);
                    outw[bb] = *reinterpret_cast<uint32_t *>(&h);
                }
                *reinterpret_cast<uint4 *>(E + e_chunk_off<D>(j, 4 * g + c)) =
                    make_uint4(outw[0], outw[1], outw[2], outw[3]);
            }
        }
        return 0;
    } else {
        int rmax = 0;
#pragma unroll
        for (int g = 0; g < Cfg<D>::GPR; ++g) rmax = max(rmax, scale_byte<D>(rr, g));
#pragma unroll
        for (int gq = 0; gq < GQ; ++gq) {
            const int gl = part * GQ + gq;
            const int g = g0 + gl;
            const int k = scale_byte<D>(rr, g) - rmax;  // <= 0
            // 2^k in fp16: normal for k >= -14, subnormal down to -24, else 0
            const uint16_t hb = k >= -14 ? (uint16_t)((k + 15) << 10) : k >= -24 ? (uint16_t)(1u << (k + 24)) : 0;
            __half2 s2 = __halves2half2(__ushort_as_half(hb), __ushort_as_half(hb));
            const uint32_t *w = reinterpret_cast<const uint32_t *>(&rr.code[gl]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // 4 bytes -> 8 channels -> one 16-byte chunk
                uint32_t outw[4];
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    __half2_raw hr =
                        __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((w[c] >> (8 * bb)) & 0xFF), __NV_E2M1);
                    __half2 h = __hmul2(*reinterpret_cast<__half2 *>(&hr), s2);
                    outw[bb] = *reinterpret_cast<uint32_t *>(&h);
                }
                *reinterpret_cast<uint4 *>(E + e_chunk_off<D>(j, 4 * g + c)) =
                    make_uint4(outw[0], outw[1], outw[2], outw[3]);
            }
        }
        return rmax - 127;
    }
}

// Whether K-chunk kk (channels 16 kk .. 16 kk + 15) / O^T d-tile dt lies in the low channel set.
template <int D>
__host__ __device__ constexpr bool low_chunk(int kk) {
    return ((16 * kk) % (D / 2)) < D / 4;
}
template <int D>
__host__ __device__ constexpr bool low_dtile(int dt) {
    return D == 128 || ((128 * dt) % (D / 2)) < D / 4;
}

// Window tile: cp.async this thread's half of the bf16 row into E' and convert
// it in place to fp16 scaled by 2^-R_j, R_j = exponent of the row's max |x|
// (the two halves exchange their maxima through xmax[256]). Called by all
// threads of the CTA together.
template <int D>
__device__ __forceinline__ int load_window_row(const AttArgs &a, const TileRef &tr, uint8_t *E, uint32_t E_s,
                                               float *xmax, bool &valid) {
    const int j = threadIdx.x & (kTile - 1);
    const int kc0 = (threadIdx.x >> 7) * (D / 16);
    const int r = (tr.lt - tr.ctiles) * kTile + j;
    valid = r < tr.wlen;
    float mx = 0.f;
    if (!valid) {
        for (int kc = kc0; kc < kc0 + D / 16; ++kc)
            *reinterpret_cast<uint4 *>(E + e_chunk_off<D>(j, kc)) = make_uint4(0, 0, 0, 0);
    } else {
        const __nv_bfloat16 *src = a.win_kv + ((size_t)a.win_start[tr.i] + r) * D;
#pragma unroll 8
        for (int kc = kc0; kc < kc0 + D / 16; ++kc) cp_async16(E_s + e_chunk_off<D>(j, kc), src + 8 * kc);
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
        for (int kc = kc0; kc < kc0 + D / 16; ++kc) {
            uint4 u = *reinterpret_cast<const uint4 *>(E + e_chunk_off<D>(j, kc));
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 f = __bfloat1622float2(h[k]);
                mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
    }
    xmax[threadIdx.x] = mx;
    __syncthreads();
    mx = fmaxf(xmax[j], xmax[j + kTile]);
    if (!valid) return 0;
    const int R = mx > 0.f ? (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127 : 0;
    const float inv = ldexpf(1.0f, -R);
    for (int kc = kc0; kc < kc0 + D / 16; ++kc) {
        uint4 u = *reinterpret_cast<const uint4 *>(E + e_chunk_off<D>(j, kc));
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 f = __bfloat1622float2(h[k]);
            __half2 hh = __floats2half2_rn(f.x * inv, f.y * inv);
            o[k] = *reinterpret_cast<uint32_t *>(&hh);
        }
        *reinterpret_cast<uint4 *>(E + e_chunk_off<D>(j, kc)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    return R;
}

// The CTA whose range holds flat tile t: the last c with cta_t[c] <= t.
__device__ __forceinline__ int cta_of_tile(const long long *cta_t, int G, long long t) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cta_t[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ---------------------------------------------------------------- schedule
// One CTA of 1024 threads per query: its query's scale exponent sq[i] (from
// max|q|), the Q' image (q * 2^-sq in fp16, in the swizzled K-major layout
// the MMA reads, heads >= H zero) and, when the query has no entry at all,
// out = 0 and lse = -inf. One more CTA, in parallel with those, writes the
// per-query records, the tile prefix and the first query of every attention
// CTA's range.
__device__ __forceinline__ void query_tiles(const int32_t *q_offsets, const int32_t *q_pos, const int32_t *n_blocks,
                                            const int32_t *win_len, int batch, int m, int cap, int topk, int max_win,
                                            int i, int32_t *status, int &b_out, int &ne, int &ct, int &wl) {
    const int b = request_of(q_offsets, batch, i);
    ne = 0;
    if (b >= 0) ne = (q_pos ? min(visible_blocks(q_pos[i], m, n_blocks[b]), cap) : topk);
    wl = win_len ? win_len[i] : 0;
    if (wl < 0 || wl > max_win) {
        if (status) atomicOr(status, CSA_DEV_BAD_WINDOW);
        wl = min(max(wl, 0), max_win);
    }
    if (b < 0) wl = 0;
    ct = (ne + kTile - 1) / kTile;
    b_out = b < 0 ? 0 : b;
}

template <int D>
__global__ void __launch_bounds__(1024) attend_schedule_kernel(
    const int32_t *q_offsets, const int32_t *q_pos, const int32_t *n_blocks, const int32_t *win_len, int batch,
    int Nq, int m, int cap, int topk, int max_win, const __nv_bfloat16 *q, int H, int G, QInfo *qinfo,
    long long *tprefix, int32_t *cta_q, long long *cta_t, long long *uprefix, int32_t *sq, uint8_t *qimg, float *out,
    float *lse, int32_t *status, int2 *qspan) {
    __shared__ long long red[32];
    __shared__ long long round_total;
    __shared__ float fred[32];
    __shared__ int sq_s;
    grid_dep_launch();  // the attention kernel may start its prologue; it waits for this grid's results
    const int qi = blockIdx.x;
    // ---- CTAs 0 .. Nq-1: one query each: scale exponent, Q' image and the empty case
    if (qi < Nq) {
        // the query is read once: chunk c = 8 channels (h = c / (D/8), kc = c % (D/8)), kept in registers
        constexpr int kPer = (kHeads * (D / 8) + 1023) / 1024;
        const __nv_bfloat16 *qp = q + (size_t)qi * H * D;
        const int nchunks = H * D / 8;
        uint4 u[kPer];
        float mx = 0.f;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int c = threadIdx.x + j * 1024;
            u[j] = c < nchunks ? __ldg(reinterpret_cast<const uint4 *>(qp) + c) : make_uint4(0, 0, 0, 0);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u[j]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 f = __bfloat1622float2(h2[k]);
                mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
        mx = warp_max(mx);
        if ((threadIdx.x & 31) == 0) fred[threadIdx.x >> 5] = mx;
        __syncthreads();
        if (threadIdx.x == 0) {
            float m8 = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m8 = fmaxf(m8, fred[w]);
            // 2^-sq puts max|q| in [2^14, 2^15): every bf16 value within 2^31 of it is exact in fp16
            sq_s = m8 > 0.f ? (int)((__float_as_uint(m8) >> 23) & 0xFF) - 127 - 14 : 0;
            sq[qi] = sq_s;
        }
        __syncthreads();
        const float inv = ldexpf(1.0f, -sq_s);
        uint8_t *img = qimg + (size_t)qi * Cfg<D>::Q_BYTES;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int c = threadIdx.x + j * 1024;
            if (c >= kHeads * (D / 8)) break;
            const int h = c / (D / 8);
            const int kc = c % (D / 8);
            uint32_t o[4];
            const __nv_bfloat162 *hh = reinterpret_cast<const __nv_bfloat162 *>(&u[j]);  // zero for h >= H
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 f = __bfloat1622float2(hh[k]);
                __half2 x = __floats2half2_rn(f.x * inv, f.y * inv);
                o[k] = *reinterpret_cast<uint32_t *>(&x);
            }
            const size_t off =
                (size_t)(kc >> 3) * Cfg<D>::QREG + (h >> 3) * 1024 + (h & 7) * 128 + (((kc & 7) ^ (h & 7)) << 4);
            *reinterpret_cast<uint4 *>(img + off) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        int b, ne, ct, wl;
        query_tiles(q_offsets, q_pos, n_blocks, win_len, batch, m, cap, topk, max_win, qi, nullptr, b, ne, ct, wl);
        if (ct + (wl + kTile - 1) / kTile == 0) {
            for (int k = threadIdx.x; k < H * D; k += blockDim.x) out[(size_t)qi * H * D + k] = 0.f;
            if (lse)
                for (int k = threadIdx.x; k < H; k += blockDim.x) lse[(size_t)qi * H + k] = -INFINITY;
        }
    }
    if (qi != Nq) return;
    // ---- CTA Nq (in parallel with the others): per-query records, tile prefix,
    // first query of every CTA range. The prefixes and the CTA ranges are searched
    // below; up to kSchedSmemQueries queries they are searched in shared memory.
    __shared__ long long s_tpre[kSchedSmemQueries + 1], s_upre[kSchedSmemQueries + 1], s_ctat[kMaxAttendCtas + 1];
    const bool in_smem = Nq <= kSchedSmemQueries && G <= kMaxAttendCtas;
    const long long *tpre = in_smem ? s_tpre : tprefix;
    const long long *upre = in_smem ? s_upre : uprefix;
    const long long *ctat = in_smem ? s_ctat : cta_t;
    long long carry = 0, ucarry = 0;
    for (int base = 0; base < Nq; base += blockDim.x) {
        const int i = base + threadIdx.x;
        long long tiles = 0, units = 0;
        int b = 0, ne = 0, ct = 0, wl = 0;
        if (i < Nq) {
            query_tiles(q_offsets, q_pos, n_blocks, win_len, batch, m, cap, topk, max_win, i, status, b, ne, ct, wl);
            const int wt = (wl + kTile - 1) / kTile;
            tiles = ct + wt;
            units = tiles > 0 ? kStartCost + kCTileCost * ct + kWTileCost * wt : 0;
        }
        const long long incl = block_inclusive_scan<long long>(tiles, red);
        if (i < Nq) {
            const long long t0 = carry + incl - tiles;
            tprefix[i + 1] = t0 + tiles;
            if (in_smem) s_tpre[i + 1] = t0 + tiles;
            QInfo r;
            r.a = make_int4(b, ne, ct, wl);
            r.b = make_int4(n_blocks[b], 0, 0, 0);
            r.t = make_longlong2(t0, t0 + tiles);
            qinfo[i] = r;
        }
        if (i == 0) {
            tprefix[0] = 0;
            if (in_smem) s_tpre[0] = 0;
        }
        if (threadIdx.x == blockDim.x - 1) round_total = incl;
        __syncthreads();
        carry += round_total;
        __syncthreads();
        const long long uincl = block_inclusive_scan<long long>(units, red);
        if (i < Nq) {
            uprefix[i + 1] = ucarry + uincl;
            if (in_smem) s_upre[i + 1] = ucarry + uincl;
        }
        if (i == 0) {
            uprefix[0] = 0;
            if (in_smem) s_upre[0] = 0;
        }
        if (threadIdx.x == blockDim.x - 1) round_total = uincl;
        __syncthreads();
        ucarry += round_total;
        __syncthreads();
    }
    __threadfence_block();
    __syncthreads();
    // CTA c's share starts at unit U c / G: its first tile is the first one of the
    // query holding that unit whose own units start at or after it; its first query
    // is the last i with tprefix[i] <= that tile
    const long long T = carry, U = ucarry;
    for (int c = threadIdx.x; c <= G; c += blockDim.x) {
        long long tb = T;
        if (c < G && U > 0) {
            const long long ub = U * c / G;
            int lo = 0, hi = Nq - 1;  // last i with uprefix[i] <= ub
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (upre[mid] <= ub) lo = mid; else hi = mid - 1;
            }
            const QInfo r = qinfo[lo];
            const long long ct = r.a.z, nt = r.t.y - r.t.x;
            const long long x = ub - upre[lo] - kStartCost;  // units into the query's tiles
            long long before = 0;                               // its tiles starting before ub
            if (x > 0) {  // the tile boundary nearest to ub (halves the overshoot of a CTA's share)
                if (x <= ct * kCTileCost) before = (x + kCTileCost / 2) / kCTileCost;
                else before = ct + (x - ct * kCTileCost + kWTileCost / 2) / kWTileCost;
            }
            tb = r.t.x + min(before, nt);
        }
        cta_t[c] = tb;
        if (in_smem) s_ctat[c] = tb;
        if (c < G) {
            int lo = 0, hi = Nq - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (tpre[mid] <= tb) lo = mid; else hi = mid - 1;
            }
            cta_q[c] = lo;
        }
    }
    __syncthreads();  // cta_t complete (global writes of this CTA, visible to its threads)
    // the first and last CTA holding each query's tiles, for the merge ((-1, -1): no tiles)
    for (int i = threadIdx.x; i < Nq; i += blockDim.x) {
        const long long t0 = tpre[i], t1 = tpre[i + 1];
        qspan[i] = t1 > t0 ? make_int2(cta_of_tile(ctat, G, t0), cta_of_tile(ctat, G, t1 - 1)) : make_int2(-1, -1);
    }
}

// ---------------------------------------------------------------- split merge
// Row a8: a query whose tiles were spread over several CTAs has one partial
// (unnormalized O, reference rho, row sum l) per CTA; combine them with the
// log-sum-exp rule. One CTA per (query, 8-head slice, 128 channels); queries that a single
// CTA covered were written directly by attend_kernel and are skipped.
constexpr int kMergeHeads = 8;

// by_boundary (calls with more queries than CTAs): blockIdx.x + 1 is a CTA
// index c; only a query that CTA c - 1 and CTA c both cover can need a merge,
// and the CTA for the first such boundary of a query merges it, so the grid
// has G - 1 columns instead of one per query.
__global__ void __launch_bounds__(256) attend_merge_kernel(const long long *tprefix, const long long *cta_t,
                                                           const int2 *qspan, int Nq, int H, int D, int G,
                                                           const float *part_o, const float *part_rho,
                                                           const float *part_l, float *out, float *lse,
                                                           int by_boundary) {
    __shared__ int slots[256];
    __shared__ float wts[256 * kMergeHeads];
    __shared__ float s_rho[256 * kMergeHeads], s_l[256 * kMergeHeads];
    __shared__ float inv_l[kMergeHeads];
    __shared__ int np_s;
    grid_dep_wait();
    const int h0 = blockIdx.y * kMergeHeads;
    if (h0 >= H) return;
    int i = blockIdx.x;
    if (by_boundary) {
        // the query holding tile rb = first tile of CTA c: largest i with tprefix[i] < rb
        const int c = blockIdx.x + 1;
        const long long rb = cta_t[c];
        int lo = 0, hi = Nq - 1;  // tprefix[0] = 0 < rb unless rb = 0 (then no query straddles)
        if (rb <= 0) return;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tprefix[mid] < rb) lo = mid; else hi = mid - 1;
        }
        i = lo;
        if (tprefix[i + 1] <= rb) return;      // the boundary is at the end of query i: nothing straddles
        if (qspan[i].x + 1 != c) return;        // not the query's first inner boundary
    }
    // the CTAs that hold the query's tiles (the schedule kernel found them)
    const int2 span = qspan[i];
    const int c_first = span.x, c_last = span.y;
    if (c_first < 0 || c_first == c_last) return;  // no entry (written by the schedule kernel) or one CTA wrote it
    // its partials, in CTA order, CTAs with an empty range skipped: warp 0, 32 CTAs per round
    if (threadIdx.x < 32) {
        int np = 0;
        for (int cc0 = c_first; cc0 <= c_last && np < 256; cc0 += 32) {
            const int cc = cc0 + (int)threadIdx.x;
            bool has = false;
            long long rb = 0;
            if (cc <= c_last) {
                rb = cta_t[cc];
                has = rb < cta_t[cc + 1];
            }
            const uint32_t m = __ballot_sync(0xffffffffu, has);
            const int pos = np + __popc(m & ((1u << threadIdx.x) - 1u));
            if (has && pos < 256) slots[pos] = 2 * cc + (rb >= tprefix[i] ? 0 : 1);
            np += __popc(m);
        }
        if (threadIdx.x == 0) np_s = min(np, 256);
    }
    __syncthreads();
    const int np = np_s;
    const int nh = min(kMergeHeads, H - h0);
    // every partial's (rho, l) of the slice's heads, one load per thread
    for (int k = threadIdx.x; k < np * kMergeHeads; k += blockDim.x) {
        const int p = k / kMergeHeads, hh = k % kMergeHeads;
        const size_t at = (size_t)slots[p] * kHeads + h0 + hh;
        s_rho[k] = hh < nh ? part_rho[at] : -INFINITY;
        s_l[k] = hh < nh ? part_l[at] : 0.f;
    }
    __syncthreads();
    if (threadIdx.x < nh) {
        const int h = h0 + threadIdx.x;
        float rmax = -INFINITY;
        for (int p = 0; p < np; ++p) rmax = fmaxf(rmax, s_rho[p * kMergeHeads + threadIdx.x]);
        float l = 0.f;
        for (int p = 0; p < np; ++p) {
            // rho = -inf: no entry of this head in that partial (or in any, if rmax is -inf)
            const float wgt = rmax == -INFINITY ? 0.f : exp2f(s_rho[p * kMergeHeads + threadIdx.x] - rmax);
            wts[p * kMergeHeads + threadIdx.x] = wgt;
            l += wgt * s_l[p * kMergeHeads + threadIdx.x];
        }
        inv_l[threadIdx.x] = l > 0.f ? 1.f / l : 0.f;
        if (lse && blockIdx.z == 0) lse[(size_t)i * H + h] = l > 0.f ? (rmax + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
    __syncthreads();
    // one float4 of one head per thread: this CTA's 8 heads x 128 channels (blockIdx.z);
    // eight partials in flight at a time
    const int hh = threadIdx.x >> 5, d4 = blockIdx.z * 32 + (threadIdx.x & 31);
    if (hh < nh && d4 < D / 4) {
        const float4 *src = reinterpret_cast<const float4 *>(part_o + (size_t)(h0 + hh) * D) + d4;
        const size_t slot_stride = (size_t)kHeads * D / 4;  // float4s per partial
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int p0 = 0; p0 < np; p0 += 8) {
            float4 o[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                o[k] = p0 + k < np ? __ldcg(src + (size_t)slots[p0 + k] * slot_stride) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float wgt = p0 + k < np ? wts[(p0 + k) * kMergeHeads + hh] : 0.f;
                acc.x = fmaf(wgt, o[k].x, acc.x);
                acc.y = fmaf(wgt, o[k].y, acc.y);
                acc.z = fmaf(wgt, o[k].z, acc.z);
                acc.w = fmaf(wgt, o[k].w, acc.w);
            }
        }
        const float il = inv_l[hh];
        reinterpret_cast<float4 *>(out + ((size_t)i * H + h0 + hh) * D)[d4] =
            make_float4(acc.x * il, acc.y * il, acc.z * il, acc.w * il);
    }
}

// ---------------------------------------------------------------- main kernel
template <int D, int SF>
__global__ void __launch_bounds__(kThreads, 1) attend_kernel(AttArgs a) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *E = smem;
    uint8_t *Q = E + C::E_BYTES;
    uint8_t *P = Q + C::Q_BYTES;
    uint8_t *misc = P + C::P_BYTES;
    // [0] S done, [1] PV of the low channel set done, [2] PV all done, [3] Q' loaded,
    // [4] / [5] low / high channel set of E' written (256 arrivals each), [6] drain on abort
    uint64_t *mbar = reinterpret_cast<uint64_t *>(misc);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 64);
    int *flags = reinterpret_cast<int *>(misc + 80);                // [0] rescale, [1] abort
    float *rho = reinterpret_cast<float *>(misc + 128);             // [64]
    float *alpha = rho + 64;                                        // [64]
    float *wred = alpha + 64;                                       // [4][64]
    float *xmax = wred + 4 * 64;                                    // [256]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hf = tid >> 7;               // channel half (dequant) = head half (softmax)
    grid_dep_wait();                       // the schedule kernel's records (programmatic launch)
    const int c = blockIdx.x;
    const long long t_begin = a.cta_t[c], t_end = a.cta_t[c + 1];
    if (t_begin >= t_end) return;

    const uint32_t E_s = smem_u32(E), Q_s = smem_u32(Q), P_s = smem_u32(P);
    const uint32_t mbar_s = smem_u32(&mbar[0]), mbar_lo = smem_u32(&mbar[1]), mbar_hi = smem_u32(&mbar[2]);
    const uint32_t mbar_q = smem_u32(&mbar[3]);
    const uint32_t mbar_elo = smem_u32(&mbar[4]), mbar_ehi = smem_u32(&mbar[5]);
    const uint32_t mbar_drain = smem_u32(&mbar[6]);
    if (tid == 0) {
        mbar_init(mbar_s, 1);
        mbar_init(mbar_lo, 1);
        mbar_init(mbar_hi, 1);
        mbar_init(mbar_q, 1);
        mbar_init(mbar_elo, kThreads);
        mbar_init(mbar_ehi, kThreads);
        mbar_init(mbar_drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 0;
        flags[1] = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM lanes: warp w reaches lanes 32 (w % 4) .. + 31; its thread takes
    // the 32 columns of head half hf of S^T (cols 0..63) and of every O^T d-tile
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tmem_s = tmem + lane_off + 32 * hf;               // S^T, this thread's 32 heads
    const uint32_t tmem_o = tmem + lane_off + kHeads + 32 * hf;      // O^T d-tile dt at + 64 dt
    uint32_t ph_s = 0, ph_e = 0;
    uint32_t n_pv = 0;          // PV groups committed so far (each completes both halves' barriers once)
    bool pv_pending = false;

    constexpr uint32_t IDESC_S = idesc_f16(kTile, kHeads, false, false);
    constexpr uint32_t IDESC_PV = idesc_f16(kTile, kHeads, true, true);

    RowRegs<D> rr;
    TileRef cur = query_ref(a, a.cta_q[c], t_begin);
    // the first query's Q' image: one bulk copy (the schedule kernel wrote it)
#ifndef CSA_TEST_UNSENT_Q_COPY
    if (tid == 0) {
        mbar_expect_tx(mbar_q, C::Q_BYTES);
        bulk_g2s(Q_s, a.qimg + (size_t)cur.i * C::Q_BYTES, C::Q_BYTES, mbar_q);
    }
    uint32_t n_q_issued = 1;    // Q' copies issued ...
#else
    // a test build of the library announces the copy's bytes but never sends it, so the
    // wait for it can only run out: the kernel's timeout path is what that test checks
    if (tid == 0) mbar_expect_tx(mbar_q, C::Q_BYTES);
    uint32_t n_q_issued = 0;
#endif
    uint32_t n_q = 0;           // ... and waited for
    prefetch_row<D, SF>(a, cur, row_block_raw(a, cur), rr);
    // the next tile and this thread's selected index in it (one tile ahead of its row loads)
    TileRef nxt = cur;
    int blk_nxt = -1;
    if (t_begin + 1 < t_end) {
        nxt = advance(a, cur, t_begin + 1);
        blk_nxt = row_block_raw(a, nxt);
    }

    long long t = t_begin;
    bool aborted = false;
    while (t < t_end && !aborted) {
        // ---------------- segment = the tiles of query cur.i inside [t, t_end)
        const int i = cur.i;
        const long long seg_begin = t;
        const long long seg_end = min(t_end, cur.t1);
        const bool whole = (seg_begin == cur.t0) && (seg_end == cur.t1);
        // the previous segment's PV must finish before Q' and O^T are reused
        if (pv_pending) {
            const bool ok = mbar_wait(mbar_lo, (n_pv - 1) & 1) && mbar_wait(mbar_hi, (n_pv - 1) & 1);
            pv_pending = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        const int sQ = a.sq[i];
        // the previous segment's output copy has read the E' buffer
        if (tid == 0 && seg_begin != t_begin) bulk_wait_read();
        // Q' of this query (issued at kernel start or in the previous segment's epilogue)
        if (__syncthreads_or(!mbar_wait(mbar_q, n_q & 1))) { aborted = true; break; }
        ++n_q;
        float lsum[32];         // row sums of this thread's 32 heads over its entries
#pragma unroll
        for (int k = 0; k < 32; ++k) lsum[k] = 0.f;
        bool first = true;

        for (; t < seg_end; ++t) {
            // ---- operand E' for this tile, low channel set first: its S MMAs run
            // while the high set is converted. Each set waits for the previous
            // tile's PV MMAs that read those channels.
            bool ok = true;
            int Rj;
            bool valid;
            if (pv_pending) ok = mbar_wait(mbar_lo, (n_pv - 1) & 1);
            if (cur.win) {
                if (pv_pending) ok = mbar_wait(mbar_hi, (n_pv - 1) & 1) && ok;
                Rj = load_window_row<D>(a, cur, E, E_s, xmax, valid);
            } else {
                valid = rr.valid;
                Rj = dequant_part<D, SF>(rr, E, 0);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(mbar_elo);
            if (warp == 0) {  // S^T = E' Q'^T over the low channel set
                ok = mbar_wait(mbar_elo, ph_e) && ok;
                tc_fence_after();
                if (lane == 0 && ok) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        if (!low_chunk<D>(kk)) continue;
                        const uint32_t koff = (uint32_t)((kk & 3) * 32);
                        const uint64_t da = desc_sw128(E_s + (kk >> 2) * C::KREG + koff, 16, 1024);
                        const uint64_t db = desc_sw128(Q_s + (kk >> 2) * C::QREG + koff, 16, 1024);
                        mma_f16(tmem, da, db, IDESC_S, kk > 0);
                    }
                }
                __syncwarp();
            }
            if (!cur.win) {
                if (pv_pending) ok = mbar_wait(mbar_hi, (n_pv - 1) & 1) && ok;
                dequant_part<D, SF>(rr, E, 1);
            }
            pv_pending = false;
            // next tile (possibly of the next query): start its row loads now,
            // and the selected index of the tile after it
            TileRef nxt2 = nxt;
            int blk_nxt2 = -1;
            if (t + 1 < t_end) {
                prefetch_row<D, SF>(a, nxt, blk_nxt, rr);
                if (t + 2 < t_end) {
                    nxt2 = advance(a, nxt, t + 2);
                    blk_nxt2 = row_block_raw(a, nxt2);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(mbar_ehi);
            if (warp == 0) {  // ... and the high set
                ok = mbar_wait(mbar_ehi, ph_e) && ok;
                tc_fence_after();
                if (lane == 0 && ok) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        if (low_chunk<D>(kk)) continue;
                        const uint32_t koff = (uint32_t)((kk & 3) * 32);
                        const uint64_t da = desc_sw128(E_s + (kk >> 2) * C::KREG + koff, 16, 1024);
                        const uint64_t db = desc_sw128(Q_s + (kk >> 2) * C::QREG + koff, 16, 1024);
                        mma_f16(tmem, da, db, IDESC_S, 1u);
                    }
                    mma_commit(mbar_s);
                }
                __syncwarp();
            }
            ph_e ^= 1;
            // a failed wait anywhere leaves S uncommitted: every thread's S wait then runs
            // out and the vote below aborts the CTA
            if (!ok) flags[1] = 1;
            if (!mbar_wait(mbar_s, ph_s)) flags[1] = 1;
            ph_s ^= 1;
            tc_fence_after();
            // u = log2(e) * scale * <q, e_j> + R_j, or -inf for an empty row
            const float cj = ldexpf(a.scale_log2, Rj + sQ);
            const float rjf = (float)Rj;
            float u[32];
            tmem_ld32(tmem_s, u);
#pragma unroll
            for (int k = 0; k < 32; ++k) u[k] = valid ? fmaf(u[k], cj, rjf) : -INFINITY;
            float rh[32];
#pragma unroll
            for (int k = 0; k < 32; k += 4) {
                const float4 r4 = *reinterpret_cast<const float4 *>(rho + 32 * hf + k);
                rh[k] = r4.x; rh[k + 1] = r4.y; rh[k + 2] = r4.z; rh[k + 3] = r4.w;
            }
            float over = -INFINITY;  // largest u - rho of this thread (rho stale on the first tile)
#pragma unroll
            for (int k = 0; k < 32; ++k) over = fmaxf(over, u[k] - rh[k]);
            const bool need = __syncthreads_or(first || over > 8.f);
            if (flags[1]) { aborted = true; break; }
            if (need) {
                // ---- per-head tile maximum -> reference update (first tile, or a logit > rho + 8)
                {
                    float m[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k) m[k] = u[k];
                    transpose_reduce32<true>(m);  // lane L: head 32 hf + L over this warp's 32 entries
                    wred[(warp & 3) * 64 + 32 * hf + lane] = m[0];
                }
                __syncthreads();
                if (tid < 64) {
                    const float M = fmaxf(fmaxf(wred[tid], wred[64 + tid]), fmaxf(wred[128 + tid], wred[192 + tid]));
                    float al = 1.f;
                    if (first) {
                        rho[tid] = M;  // may be -inf: no entry for this head yet
                    } else if (M > rho[tid] + 8.f) {
                        al = rho[tid] == -INFINITY ? 0.f : exp2f(rho[tid] - M);
                        rho[tid] = M;
                    }
                    alpha[tid] = al;
                    if (al != 1.f) flags[0] = 1;
                }
                __syncthreads();
                if (flags[0]) {  // rescale O^T columns and row sums (PV of the previous tile is complete)
#pragma unroll 1
                    for (int dt = 0; dt < C::DT; ++dt) {
                        float o[32];
                        tmem_ld32(tmem_o + 64 * dt, o);
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] *= alpha[32 * hf + k];
                        tmem_st32(tmem_o + 64 * dt, o);
                    }
#pragma unroll
                    for (int k = 0; k < 32; ++k) lsum[k] *= alpha[32 * hf + k];
                }
#pragma unroll
                for (int k = 0; k < 32; k += 4) {
                    const float4 r4 = *reinterpret_cast<const float4 *>(rho + 32 * hf + k);
                    rh[k] = r4.x; rh[k + 1] = r4.y; rh[k + 2] = r4.z; rh[k + 3] = r4.w;
                }
            }
            // ---- P' = 2^(u - rho) (fp16, 8 heads per 16-byte store) and row sums ----
            {
                const int j = tid & (kTile - 1);
                const float rj_inv = ldexpf(1.0f, -Rj);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t pk[4];
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const int k = 8 * cc + 2 * q2;
                        const float p0 = valid ? exp2f(u[k] - rh[k]) : 0.f;
                        const float p1 = valid ? exp2f(u[k + 1] - rh[k + 1]) : 0.f;
                        __half2 hh = __floats2half2_rn(p0, p1);
                        pk[q2] = *reinterpret_cast<uint32_t *>(&hh);
                        lsum[k] = fmaf(p0, rj_inv, lsum[k]);
                        lsum[k + 1] = fmaf(p1, rj_inv, lsum[k + 1]);
                    }
                    const int chunk = 4 * hf + cc;
                    const uint32_t off = (uint32_t)((j >> 3) * 1024 + (j & 7) * 128 + ((chunk ^ (j & 7)) << 4));
                    *reinterpret_cast<uint4 *>(P + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                flags[0] = 0;
                tc_fence_after();
#pragma unroll
                for (int pass = 0; pass < 2; ++pass) {  // low channel set, then the high one
#pragma unroll
                    for (int dt = 0; dt < C::DT; ++dt) {
                        if (low_dtile<D>(dt) != (pass == 0)) continue;
#pragma unroll
                        for (int kj = 0; kj < kTile / 16; ++kj) {
                            const uint64_t da = desc_sw128(E_s + (2 * dt) * C::KREG + kj * 2048, C::KREG, 1024);
                            const uint64_t db = desc_sw128(P_s + kj * 2048, 8192, 1024);
                            mma_f16(tmem + kHeads + 64 * dt, da, db, IDESC_PV, (first && kj == 0) ? 0u : 1u);
                        }
                    }
                    mma_commit(pass == 0 ? mbar_lo : mbar_hi);
                }
            }
            ++n_pv;
            pv_pending = true;
            first = false;
            if (t + 1 < t_end) {
                cur = nxt;
                nxt = nxt2;
                blk_nxt = blk_nxt2;
            }
        }
        if (aborted) break;

        // ---------------- segment epilogue
        {
            const bool ok = mbar_wait(mbar_lo, (n_pv - 1) & 1) && mbar_wait(mbar_hi, (n_pv - 1) & 1);
            pv_pending = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        tc_fence_after();
        if (t < t_end && tid == 0) {  // the next segment's Q' (this segment's S MMAs are complete)
            mbar_expect_tx(mbar_q, C::Q_BYTES);
            bulk_g2s(Q_s, a.qimg + (size_t)cur.i * C::Q_BYTES, C::Q_BYTES, mbar_q);
        }
        if (t < t_end) ++n_q_issued;
        transpose_reduce32<false>(lsum);  // lane L: head 32 hf + L over this warp's entries
        wred[(warp & 3) * 64 + 32 * hf + lane] = lsum[0];
        __syncthreads();
        if (tid < 64) {
            const float l = wred[tid] + wred[64 + tid] + wred[128 + tid] + wred[192 + tid];
            alpha[tid] = l;  // l_h
        }
        __syncthreads();
        const int b_slot = 2 * c + ((seg_begin == t_begin) ? 0 : 1);
        float *dst = whole ? a.out + (size_t)i * a.H * D : a.part_o + (size_t)b_slot * kHeads * D;
        // O^T (or O / l for a whole query) -> the E' buffer as [head][channel] fp32
        // (64 x D x 4 bytes = the buffer's size), then one bulk copy of the H used rows
        if (whole && tid < 64) {
            const float l = alpha[tid];
            xmax[tid] = l > 0.f ? 1.0f / l : 0.f;
        }
        __syncthreads();
        float *ostage = reinterpret_cast<float *>(E);
        for (int dt = 0; dt < C::DT; ++dt) {
            float o[32];
            tmem_ld32(tmem_o + 64 * dt, o);
            const int d = 128 * dt + 32 * (warp & 3) + lane;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const int h = 32 * hf + k;
                ostage[h * D + d] = whole ? o[k] * xmax[h] : o[k];
            }
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) bulk_s2g(dst, E_s, (uint32_t)(a.H * D * 4));
        if (whole) {
            if (a.lse && tid < a.H) {
                const float l = alpha[tid];
                a.lse[(size_t)i * a.H + tid] = l > 0.f ? (rho[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
            }
        } else if (tid < 64) {
            a.part_rho[(size_t)b_slot * kHeads + tid] = rho[tid];
            a.part_l[(size_t)b_slot * kHeads + tid] = alpha[tid];
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (aborted) {
        // nothing this CTA started may still run when it leaves: its Q' copy, and every MMA
        // thread 0 issued (one commit tracks them all), waited for with the long limit
        if (tid == 0) flag(a.status, CSA_DEV_TIMEOUT);
        if (n_q_issued > n_q) mbar_wait_for(mbar_q, n_q & 1, kDrainCycles);
        if (tid == 0) {
            mma_commit(mbar_drain);
            mbar_wait_for(mbar_drain, 0, kDrainCycles);
        }
    }
    if (tid == 0) bulk_wait_all();  // output copies complete before the CTA's shared memory goes away
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS) : "memory");
}

template <int D, int SF>
cudaError_t launch_main(const AttArgs &a, int num_ctas, cudaStream_t s) {
    cudaError_t err;
    const int smem = Cfg<D>::SMEM;
    if ((err = cudaFuncSetAttribute(attend_kernel<D, SF>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attend_kernel<D, SF>, a);
}

template <int D>
cudaError_t launch_schedule(const csa_cache &c, const AttArgs &a, const int32_t *q_offsets, const int32_t *q_pos,
                            const int32_t *win_len, int topk, int max_win, const void *q, int num_ctas, QInfo *qinfo,
                            long long *tprefix, int32_t *cta_q, long long *cta_t, long long *uprefix, int32_t *sq,
                            uint8_t *qimg, int2 *qspan, cudaStream_t s) {
    attend_schedule_kernel<D><<<a.Nq + 1, 1024, 0, s>>>(q_offsets, q_pos, c.n_blocks, win_len, c.batch, a.Nq, c.block,
                                                   c.capacity, topk, max_win, static_cast<const __nv_bfloat16 *>(q),
                                                   a.H, num_ctas, qinfo, tprefix, cta_q, cta_t, uprefix, sq, qimg, a.out, a.lse,
                                                   c.status, qspan);
    return cudaGetLastError();
}

}  // namespace

size_t attend_workspace_bytes(int Nq, int D, int num_ctas) {
    size_t off = 0;
    auto take = [&](size_t bytes) { off = (off + bytes + 255) & ~size_t(255); };
    take(sizeof(QInfo) * (size_t)Nq);                 // qinfo
    take(8 * (size_t)(Nq + 1));                       // tprefix
    take(4 * (size_t)num_ctas);                       // cta_q
    take(8 * (size_t)(num_ctas + 1));                 // cta_t
    take(8 * (size_t)(Nq + 1));                       // uprefix
    take(4 * (size_t)Nq);                             // sq
    take((size_t)Nq * kHeads * D * 2);                // qimg
    take(4 * (size_t)2 * num_ctas * kHeads * D);      // part_o
    take(4 * (size_t)2 * num_ctas * kHeads);          // part_rho
    take(4 * (size_t)2 * num_ctas * kHeads);          // part_l
    take(8 * (size_t)Nq);                             // qspan
    return off;
}

cudaError_t launch_attend(const csa_cache &c, const void *q, int Nq, int H, const int32_t *q_offsets,
                          const int32_t *q_pos, const int32_t *sel_idx, int topk, const void *win_kv,
                          const int64_t *win_start, const int32_t *win_len, int max_win, float softmax_scale,
                          float *out, float *lse, void *workspace, int num_ctas, cudaStream_t s) {
    const int D = c.dim;
    char *base = static_cast<char *>(workspace);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base + off;
        off = (off + bytes + 255) & ~size_t(255);
        return p;
    };
    AttArgs a;
    QInfo *qinfo = reinterpret_cast<QInfo *>(take(sizeof(QInfo) * (size_t)Nq));
    long long *tprefix = reinterpret_cast<long long *>(take(8 * (size_t)(Nq + 1)));
    int32_t *cta_q = reinterpret_cast<int32_t *>(take(4 * (size_t)num_ctas));
    long long *cta_t = reinterpret_cast<long long *>(take(8 * (size_t)(num_ctas + 1)));
    long long *uprefix = reinterpret_cast<long long *>(take(8 * (size_t)(Nq + 1)));
    int32_t *sq = reinterpret_cast<int32_t *>(take(4 * (size_t)Nq));
    uint8_t *qimg = reinterpret_cast<uint8_t *>(take((size_t)Nq * kHeads * D * 2));
    a.part_o = reinterpret_cast<float *>(take(4 * (size_t)2 * num_ctas * kHeads * D));
    a.part_rho = reinterpret_cast<float *>(take(4 * (size_t)2 * num_ctas * kHeads));
    a.part_l = reinterpret_cast<float *>(take(4 * (size_t)2 * num_ctas * kHeads));
    int2 *qspan = reinterpret_cast<int2 *>(take(8 * (size_t)Nq));
    a.fp4 = c.fp4;
    a.scale = c.scale;
    a.sel_idx = sel_idx;
    a.win_kv = static_cast<const __nv_bfloat16 *>(win_kv);
    a.win_start = win_start;
    a.out = out;
    a.lse = lse;
    a.status = c.status;
    a.qinfo = qinfo;
    a.tprefix = tprefix;
    a.cta_q = cta_q;
    a.cta_t = cta_t;
    a.sq = sq;
    a.qimg = qimg;
    a.Nq = Nq;
    a.H = H;
    a.cap = c.capacity;
    a.topk = topk;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;

    cudaError_t err;
    const int32_t *qp = sel_idx ? nullptr : q_pos;
    const int32_t *wl = win_kv ? win_len : nullptr;
    const int G = num_ctas;  // work ranges, one per CTA
    if (D == 512) {
        if ((err = launch_schedule<512>(c, a, q_offsets, qp, wl, topk, max_win, q, num_ctas, qinfo, tprefix, cta_q, cta_t,
                                        uprefix, sq, qimg, qspan, s)) != cudaSuccess)
            return err;
        err = c.scale_fmt == CSA_SCALE_E4M3_16 ? launch_main<512, kScaleE4M3x16>(a, num_ctas, s)
                                                : launch_main<512, kScaleE8M0x32>(a, num_ctas, s);
        if (err != cudaSuccess) return err;
    } else if (D == 128) {
        if ((err = launch_schedule<128>(c, a, q_offsets, qp, wl, topk, max_win, q, num_ctas, qinfo, tprefix, cta_q, cta_t,
                                        uprefix, sq, qimg, qspan, s)) != cudaSuccess)
            return err;
        err = c.scale_fmt == CSA_SCALE_E4M3_16 ? launch_main<128, kScaleE4M3x16>(a, num_ctas, s)
                                                : launch_main<128, kScaleE8M0x32>(a, num_ctas, s);
        if (err != cudaSuccess) return err;
    } else {
        return cudaErrorInvalidValue;
    }
    cudaLaunchConfig_t cfg = {};
    const int by_boundary = Nq > G ? 1 : 0;  // many queries: one column per CTA boundary
    cfg.gridDim = dim3(by_boundary ? max(1, G - 1) : Nq, (H + kMergeHeads - 1) / kMergeHeads, D / 128);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attend_merge_kernel, (const long long *)tprefix, (const long long *)cta_t,
                              (const int2 *)qspan, Nq, H, D, G,
                              (const float *)a.part_o, (const float *)a.part_rho, (const float *)a.part_l, out, lse,
                              by_boundary);
}

}  // namespace csa
