// prefill.cu -- row a3 when a request brings many queries (prefill): the
// indexer scores of every (query, visible block) pair as one tensor-core GEMM
// per request, instead of one key stream per query.
//
// Source: DeepSeek-V4.1-Flash podcast transcript, cue 12 (the indexer query
// scores the indexer keys; top-k over the scores) and cue 16 (MXFP4 = E2M1
// elements with a shared power-of-two scale per block); "Frontier Architecture
// Decoding Notes (4): DeepSeek V4", section 1 (top-k over 4-token blocks).
// Score form (the library's reading): s_j = sum_h w_h * ReLU(q_h . k_j).
//
// GEMM: rows (M) = 128 keys of one request per key stage (one key per TMEM
// lane), columns (N) = 128 (query, head) pairs of a query tile (128 / H_I
// consecutive queries, head-minor), K = d_I. An epilogue thread owns one key
// and reads whole queries' columns, so the weighted ReLU sum over a query's
// heads stays inside the thread, and one warp's 32 keys of one query form one
// 128-byte store of the score row. Two key formats:
//   * bf16 keys (CSA_IDX_BF16): kind::f16 MMAs on the cache's bf16 keys and the
//     bf16 query (exact products), 128-byte swizzled K regions of 64 channels;
//   * MXFP4 keys (CSA_IDX_MXFP4, d_I = 128): kind::mxf4 block-scaled MMAs, E2M1
//     operands with one E8M0 scale per 32 channels on both sides. The query is
//     quantized first (quantize_query_kernel, the same rule the streamed scan
//     applies to it); its codes arrive by TMA, its scales by one bulk copy of a
//     ready-made scale-factor block, while the producer warp transposes each key
//     stage's scale bytes into that block layout. tcgen05.cp moves both scale
//     blocks into tensor memory ahead of the MMAs that read them. The tensor
//     core accumulates a block-scaled product anchored at the largest block
//     scale taking part, also where that block's products cancel to zero: a
//     key whose 32-channel scales lie dozens of binades apart can lose the
//     small blocks' part of a score that fp32 arithmetic keeps.
// fp32 accumulators in TMEM, several accumulator buffers so that the epilogue of
// one key stage overlaps the MMAs of the next. Key stages are marked evict-last
// in L2, since every query tile of the request reads them again; the query tile
// stays resident while the request's keys stream past.
// Warp roles (320 threads, one CTA per SM, persistent over query tiles):
//   warps 0-7  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (its keys)
//              over half of the tile's columns; ReLU, head weight, head sum,
//              streaming stores to the score rows
//   warp 8     lane 0 issues the scale copies, the MMAs and their commits
//   warp 9     lane 0 issues the TMA loads; MXFP4: the warp writes key scales
// The score rows then go to the selection kernels.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "tc_util.cuh"

namespace csa {

namespace {

constexpr int kPfKeys = 128;     // MMA M: keys per stage
constexpr int kPfCols = 128;     // MMA N: (query, head) columns of a query tile
constexpr int kPfEpiWarps = 8;
constexpr int kPfThreads = 32 * (kPfEpiWarps + 2);
constexpr int kPfBf16 = 0;       // key formats of the kernel
constexpr int kPfMxfp4 = 1;
constexpr int kSfBlock = 512;    // scale-factor block: 128 rows x 4 E8M0 scales (d_I = 128)

template <int KF, int DI>
struct PfCfg {
    static constexpr bool MX = KF == kPfMxfp4;
    static constexpr int NREG = MX ? 1 : DI / 64;         // K regions of a row
    static constexpr int REG_ROW = MX ? DI / 2 : 128;     // bytes per row in a region
    static constexpr int A_CODES = NREG * kPfKeys * REG_ROW;  // one key stage's operand bytes
    static constexpr int B_CODES = NREG * kPfCols * REG_ROW;  // the query tile's operand bytes
    static constexpr int A_STAGE = MX ? A_CODES + 1024 : A_CODES;  // MXFP4: codes, then the scale block
    static constexpr int B_BYTES = MX ? B_CODES + 1024 : B_CODES;
    static constexpr int MISC = 4096;  // barriers, TMEM slot, flags; per-query arrays from + 512 to + 3072
    static constexpr int BUDGET = 232448 - 1024 - MISC - B_BYTES;  // opt-in shared memory per CTA
    static constexpr int STAGES = BUDGET / A_STAGE >= 8 ? 8 : BUDGET / A_STAGE;
    static constexpr int SMEM = 1024 + B_BYTES + STAGES * A_STAGE + MISC;
    static constexpr int NACC = MX ? 3 : 4;               // accumulator buffers of kPfCols columns
    static constexpr int SFA_COL = MX ? 384 : 0;          // MXFP4: key scales of accumulator buffer u at + 16 u
    static constexpr int SFB_COL = MX ? 448 : 0;          // MXFP4: query scales
    static constexpr int TMEM_COLS = 512;
    // tcgen05 smem descriptor: 128-byte swizzle (bf16, 128-byte rows) or 64-byte swizzle
    // (MXFP4 at d_I = 128: 64-byte rows); 8-row groups REG_ROW * 8 bytes apart
    static constexpr uint32_t LAYOUT = MX ? 4u : 2u;
    static constexpr uint32_t SBO = 8 * REG_ROW;
    static_assert(STAGES >= 2, "key ring needs two stages");
    static_assert(!MX || DI == 128, "MXFP4 GEMM path: d_I = 128");
    static_assert(!MX || (NACC * kPfCols <= SFA_COL && SFA_COL + 16 * NACC <= SFB_COL && SFB_COL + 4 <= TMEM_COLS),
                  "accumulator and scale-factor columns overlap");
    static_assert(MX || NACC * kPfCols <= TMEM_COLS, "accumulators exceed tensor memory");
};

struct PfArgs {
    CUtensorMap tm_keys;         // keys: bf16 [batch * cap][d_I] or MXFP4 codes [batch * cap][d_I / 2]
    CUtensorMap tm_q;            // query: bf16 [Nq * H_I][d_I] or MXFP4 codes [Nq * H_I][d_I / 2]
    const uint8_t *key_scales;   // MXFP4: [batch * cap][d_I / 32] E8M0
    const uint8_t *q_sf;         // MXFP4: per query tile one scale-factor block (kSfBlock bytes)
    const float *w;              // [Nq][H_I]
    const int32_t *req, *n_vis;  // [Nq], from the schedule kernel
    float *scores;               // [Nq][rows]
    int32_t *status;
    int Nq, cap, rows;
    long long key_rows;          // batch * cap
};

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 2-D tiled TMA load (no multicast) completing on mbar's transaction count.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *tm, int x, int y, uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap *tm, int x, int y, uint32_t mbar,
                                                 uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(mbar), "l"(pol)
        : "memory");
}

// Score rows are read once more, by the selection: stream them past L2.
__device__ __forceinline__ void st_score(float *p, float v) {
    asm volatile("st.global.cs.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// tcgen05 shared-memory matrix descriptor (start, LBO, SBO in 16-byte units,
// version 1 in bits 46-47, layout type in bits 61-63).
__device__ __forceinline__ uint64_t desc_smem(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// Instruction descriptor of kind::mxf4 (block-scaled): A and B E2M1 (format 1 in
// bits 7-9 and 10-12), both K-major, N >> 3 (bits 17-22), E8M0 scales (bit 23),
// M >> 4 (bits 24-28), dense K = 64; the scale-factor byte ids of A (bits 29-30)
// and B (bits 4-5) select which bytes of each 32-bit TMEM column the MMA reads.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, uint32_t a_sf_id, uint32_t b_sf_id) {
    return (b_sf_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
           ((uint32_t)(M >> 4) << 24) | (a_sf_id << 29);
}

__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                         uint32_t sfa, uint32_t sfb) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
}

// Copy one scale-factor block (32 rows of 16 bytes in shared memory) into four
// TMEM columns, replicated into all four lane quarters: lane r of every quarter,
// column a, byte k = the scale of row 32 a + r for channels 32 k .. 32 k + 31.
__device__ __forceinline__ void sf_copy(uint32_t taddr, uint32_t smem_addr) {
    const uint64_t d = desc_smem(smem_addr, 128, 128, 0);  // no swizzle, 8-row core matrices 128 bytes apart
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

// Byte offset of row m's scale for channel group k in a scale-factor block.
__host__ __device__ constexpr int sf_offset(int m, int k) { return 16 * (m & 31) + 4 * (m >> 5) + k; }

// MXFP4 indexer query: per (query, head) row and 32-channel group, E8M0 scale
// X = floor(log2 amax) - 2 and the E2M1 codes of q / 2^X (round to nearest even,
// saturating) -- the rule the streamed scan applies to the query. Codes go to
// [rows][d_I / 2] (element 2i in the low nibble), scales into one scale-factor
// block per 128 rows; rows past the last query get scale 1 and no codes (the
// TMA reads zeros there).
template <int DI>
__global__ void __launch_bounds__(256) quantize_query_kernel(const __nv_bfloat16 *q, int rows, int tiles,
                                                             uint8_t *codes, uint8_t *sf) {
    grid_dep_wait();
    grid_dep_launch();
    constexpr int G = DI / 32;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)tiles * kPfCols * G) return;
    const int row = (int)(t / G), grp = (int)(t % G);
    int xb = 127;
    if (row < rows) {
        const uint4 *src = reinterpret_cast<const uint4 *>(q + (size_t)row * DI + grp * 32);
        float v[32];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint4 x = __ldg(src + u);
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = __bfloat1622float2(h[k]);
                v[8 * u + 2 * k] = f.x;
                v[8 * u + 2 * k + 1] = f.y;
            }
        }
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(v[k]));
        xb = e8m0_byte(amax);
        const float inv = e8m0_inverse(xb);
        uint32_t cw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint32_t wv = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) wv |= e2m1_code(v[8 * u + e] * inv) << (4 * e);
            cw[u] = wv;
        }
        *reinterpret_cast<uint4 *>(codes + (size_t)row * (DI / 2) + grp * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    }
    sf[(size_t)(row >> 7) * kSfBlock + sf_offset(row & 127, grp)] = (uint8_t)xb;
}

template <int KF, int DI, int HI>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_score_kernel(const __grid_constant__ PfArgs a) {
    using C = PfCfg<KF, DI>;
    constexpr bool MX = C::MX;
    constexpr int ST = C::STAGES;
    constexpr int NACC = C::NACC;
    constexpr int QT = kPfCols / HI;      // queries per tile
    constexpr int QPT = 64 / HI;          // queries per epilogue thread (half of the tile's columns)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *Qs = smem;                   // query tile (+ its scale block at + B_CODES)
    uint8_t *Ks = Qs + C::B_BYTES;        // key stage s at Ks + s A_STAGE (+ its scale block at + A_CODES)
    uint8_t *misc = Ks + ST * C::A_STAGE;
    // barriers: query tile full / free, key stages full / free, accumulators full / free
    enum { B_QFULL = 0, B_QFREE = 1, B_KFULL = 2, B_KFREE = 2 + ST, B_CFULL = 2 + 2 * ST, B_CFREE = 2 + 2 * ST + NACC };
    uint64_t *mb = reinterpret_cast<uint64_t *>(misc);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 256);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 260);
    int *n_sub = reinterpret_cast<int *>(misc + 264);
    int *s_req = reinterpret_cast<int *>(misc + 512);        // [QT] request of each query of the tile (-1: none)
    int *s_nv = s_req + 128;                                  // [QT] its visible keys (<= cap)
    float *s_w = reinterpret_cast<float *>(s_nv + 128);      // [QT * HI] head weights
    int2 *s_sub = reinterpret_cast<int2 *>(s_w + 128);       // requests present: (request, largest n)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto bar = [&](int k) { return smem_u32(&mb[k]); };
    const uint32_t Q_s = smem_u32(Qs), K_s = smem_u32(Ks);
    if (tid == 0) {
        mbar_init(bar(B_QFULL), 1);
        mbar_init(bar(B_QFREE), 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar(B_KFULL + s), MX ? 2 : 1);  // MXFP4: the TMA, and the key scales written
            mbar_init(bar(B_KFREE + s), 1);
        }
        for (int u = 0; u < NACC; ++u) {
            mbar_init(bar(B_CFULL + u), 1);
            mbar_init(bar(B_CFREE + u), 32 * kPfEpiWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        *abort_flag = 0;
    }
    if (warp == 9 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tm_keys)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tm_q)) : "memory");
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
    grid_dep_wait();  // the schedule kernel's req / n_vis (and the quantized query)

    const int ntiles = (a.Nq + QT - 1) / QT;
    uint32_t gkt = 0;  // key stages of this CTA so far (ring slot, accumulator and phases)
    uint32_t ns = 0;   // (tile, request) items of this CTA so far
    bool ok = true;

    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int q0 = tile * QT;
        if (__syncthreads_or(!ok)) break;
        // per-query data of the tile, then the requests present in it (queries are
        // ordered by request: runs of one request), by one thread from shared memory
        if (tid < QT) {
            const int q = q0 + tid;
            s_req[tid] = q < a.Nq ? a.req[q] : -1;
            s_nv[tid] = q < a.Nq ? min(a.n_vis[q], a.cap) : 0;
        }
        if (tid < QT * HI) s_w[tid] = q0 + tid / HI < a.Nq ? a.w[(size_t)q0 * HI + tid] : 0.f;
        __syncthreads();
        if (tid == 0) {
            int cnt = 0;
            for (int qq = 0; qq < QT; ++qq) {
                const int r = s_req[qq];
                if (r < 0) continue;
                if (cnt == 0 || s_sub[cnt - 1].x != r) s_sub[cnt++] = make_int2(r, s_nv[qq]);
                else s_sub[cnt - 1].y = max(s_sub[cnt - 1].y, s_nv[qq]);
            }
            *n_sub = cnt;
        }
        __syncthreads();
        const int nsub = *n_sub;
        for (int si = 0; si < nsub && ok; ++si) {
            const int b = s_sub[si].x;
            const int maxn = s_sub[si].y;
            const int nkt = (maxn + kPfKeys - 1) / kPfKeys;
            if (nkt == 0) continue;
            if (warp == 9) {
                // ================= producer: TMA (lane 0); MXFP4 key scales (the warp)
                const uint64_t pol = policy_evict_last();
                if (lane == 0) {
                    if (ns >= 1) ok = mbar_wait_ab<false>(bar(B_QFREE), (ns - 1) & 1, abort_flag);
                    if (ok) {  // the query tile: rows (query, head) from q0 H_I; rows past the array read zeros
                        mbar_expect_tx(bar(B_QFULL), (uint32_t)(C::B_CODES + (MX ? kSfBlock : 0)));
#pragma unroll
                        for (int r = 0; r < C::NREG; ++r)
                            tma_load_2d(Q_s + r * kPfCols * C::REG_ROW, &a.tm_q, 64 * r, q0 * HI, bar(B_QFULL));
                        if constexpr (MX) bulk_g2s(Q_s + C::B_CODES, a.q_sf + (size_t)tile * kSfBlock, kSfBlock, bar(B_QFULL));
                    }
                }
                ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
                for (int kt = 0; kt < nkt && ok; ++kt) {
                    const uint32_t g = gkt + kt, s = g % ST;
                    const uint32_t stage = K_s + s * C::A_STAGE;
                    if (lane == 0 && g >= (uint32_t)ST)
                        ok = mbar_wait_ab<false>(bar(B_KFREE + s), ((g / ST) - 1) & 1, abort_flag);
                    ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
                    if (!ok) break;
                    // keys kt 128 .. + 127 of request b; columns past the visible ones are never stored
                    if (lane == 0) {
                        mbar_expect_tx(bar(B_KFULL + s), (uint32_t)C::A_CODES);
#pragma unroll
                        for (int r = 0; r < C::NREG; ++r)
                            tma_load_2d_hint(stage + r * kPfKeys * C::REG_ROW, &a.tm_keys, 64 * r,
                                             b * a.cap + kt * kPfKeys, bar(B_KFULL + s), pol);
                    }
                    if constexpr (MX) {
                        // the stage's key scales (4 bytes per key) into a scale-factor block:
                        // lane r writes the 16 bytes of keys r, 32 + r, 64 + r, 96 + r
                        const long long r0 = (long long)b * a.cap + kt * kPfKeys + lane;
                        uint32_t wv[4];
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const long long row = r0 + 32 * q4;
                            wv[q4] = row < a.key_rows
                                         ? __ldg(reinterpret_cast<const uint32_t *>(a.key_scales) + row)
                                         : 0x7F7F7F7Fu;
                        }
                        *reinterpret_cast<uint4 *>(Ks + s * C::A_STAGE + C::A_CODES + 16 * lane) =
                            make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        fence_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_KFULL + s));
                    }
                }
                if (lane == 0 && !ok) *abort_flag = 1;
            } else if (warp == 8) {
                // ================= MMA issue
                if (lane == 0) {
                    ok = mbar_wait_ab<false>(bar(B_QFULL), ns & 1, abort_flag);
                    if (ok && MX) {
                        tc_fence_after();
                        sf_copy(tmem + C::SFB_COL, Q_s + C::B_CODES);
                    }
                    for (int kt = 0; kt < nkt && ok; ++kt) {
                        const uint32_t g = gkt + kt, s = g % ST, u = g % NACC;
                        const uint32_t stage = K_s + s * C::A_STAGE;
                        ok = mbar_wait_ab<false>(bar(B_KFULL + s), (g / ST) & 1, abort_flag);
                        if (ok && g >= (uint32_t)NACC)
                            ok = mbar_wait_ab<false>(bar(B_CFREE + u), ((g / NACC) - 1) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t d = tmem + u * kPfCols;
                        if constexpr (MX) {
                            const uint32_t sfa = tmem + C::SFA_COL + 16 * u, sfb = tmem + C::SFB_COL;
                            sf_copy(sfa, stage + C::A_CODES);
#pragma unroll
                            for (int k = 0; k < DI / 64; ++k) {  // 64 channels = 32 bytes per MMA
                                const uint64_t da = desc_smem(stage + 32 * k, 16, C::SBO, C::LAYOUT);
                                const uint64_t db = desc_smem(Q_s + 32 * k, 16, C::SBO, C::LAYOUT);
                                const uint32_t id = (uint32_t)(2 * k);  // scale bytes 2k, 2k + 1 of each column
                                mma_mxf4(d, da, db, idesc_mxf4(kPfKeys, kPfCols, id, id), k > 0, sfa | (id << 30),
                                         sfb | (id << 30));
                            }
                        } else {
#pragma unroll
                            for (int kk = 0; kk < DI / 16; ++kk) {
                                const uint32_t koff = (uint32_t)((kk & 3) * 32);
                                const uint64_t da =
                                    desc_smem(stage + (kk >> 2) * kPfKeys * 128 + koff, 16, C::SBO, C::LAYOUT);
                                const uint64_t db =
                                    desc_smem(Q_s + (kk >> 2) * kPfCols * 128 + koff, 16, C::SBO, C::LAYOUT);
                                mma_f16(d, da, db, idesc_bf16(kPfKeys, kPfCols), kk > 0);
                            }
                        }
                        mma_commit(bar(B_KFREE + s));
                        mma_commit(bar(B_CFULL + u));
                    }
                    if (ok) mma_commit(bar(B_QFREE));
                    if (!ok) *abort_flag = 1;
                }
                ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
            } else {
                // ================= epilogue: TMEM lane = key, 64 columns = QPT whole queries
                const int qw = warp & 3, ch = warp >> 2;
                const uint32_t lane_off = (uint32_t)(32 * qw) << 16;
                // head weights and visible-key limits of the thread's queries (one or two heads:
                // the limits stay in shared memory, a broadcast read, to keep registers free)
                constexpr int NR = QPT <= 16 ? QPT : 1;
                float wr[64];
                int nr[NR];
#pragma unroll
                for (int e = 0; e < 64; ++e) wr[e] = s_w[64 * ch + e];
#pragma unroll
                for (int j = 0; j < NR; ++j) {
                    const int qq = QPT * ch + j;
                    nr[j] = s_req[qq] == b ? s_nv[qq] : 0;
                }
                float *const srow = a.scores + (size_t)(q0 + QPT * ch) * a.rows;
                for (int kt = 0; kt < nkt; ++kt) {
                    const uint32_t g = gkt + kt, u = g % NACC;
                    ok = mbar_wait_ab<false>(bar(B_CFULL + u), (g / NACC) & 1, abort_flag);
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    tc_fence_after();
                    const int key = kt * kPfKeys + 32 * qw + lane;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float v[32];
                        tmem_ld32(tmem + lane_off + u * kPfCols + 64 * ch + 32 * c, v);
#pragma unroll
                        for (int j = 0; j < 32 / HI; ++j) {
                            const int jq = (32 / HI) * c + j;  // query of the thread's QPT
                            float sc = 0.f;
#pragma unroll
                            for (int h = 0; h < HI; ++h) sc = fmaf(wr[HI * jq + h], fmaxf(v[HI * j + h], 0.f), sc);
                            const int lim = NR == QPT ? nr[jq % NR]
                                                      : (s_req[QPT * ch + jq] == b ? s_nv[QPT * ch + jq] : 0);
                            if (key < lim) st_score(srow + (size_t)jq * a.rows + key, sc);
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(bar(B_CFREE + u));
                }
                if (!ok) *abort_flag = 1;
            }
            gkt += nkt;
            ++ns;
        }
    }
    if (tid == 256 && ns >= 1 && ok) mbar_wait(bar(B_QFREE), (ns - 1) & 1);  // last commit landed
    if (__syncthreads_or(!ok) && tid == 0) flag(a.status, CSA_DEV_TIMEOUT);
    if (!ok && tid == 256) {  // let tensor-core and TMA work already issued finish before TMEM is released
        const long long t0 = clock64();
        while (clock64() - t0 < 2000000) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS) : "memory");
}

// Issue rate of the block-scaled MMA used above: one CTA per SM issues `iters`
// pairs of kind::mxf4 MMAs (M = 128, N = 256, K = 64 each) from resident shared-memory
// tiles (non-zero codes of alternating sign, so that every product toggles the
// datapath; unit scales) into one TMEM accumulator, with the same descriptor and
// scale-factor layout as the score GEMM. No data moves, so the time measures the
// tensor pipe alone; FLOPs = 2 * 128 * 256 * 128 * iters per CTA.
constexpr int kProbeN = 256;
__global__ void __launch_bounds__(128, 1) mxf4_probe_kernel(int iters, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *As = smem;                      // 128 rows x 64 B (K = 128 codes), 64-byte swizzle
    uint8_t *Bs = As + 128 * 64;             // 256 rows x 64 B
    uint8_t *SFa = Bs + kProbeN * 64;        // one scale-factor block (128 rows)
    uint8_t *SFb = SFa + 1024;               // two (256 rows)
    uint64_t *mb = reinterpret_cast<uint64_t *>(SFb + 2048);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mb + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int k = tid; k < (128 + kProbeN) * 64 / 16; k += blockDim.x)  // codes +1.5, -3, +6, -0.5, ...
        reinterpret_cast<uint4 *>(As)[k] = make_uint4(0xD37A9E15u, 0x6B2C5F91u, 0xA4E3172Du, 0x39C8B6F4u);
    for (int k = tid; k < 3 * 1024 / 4; k += blockDim.x) reinterpret_cast<uint32_t *>(SFa)[k] = 0x7F7F7F7Fu;
    if (tid == 0) {
        mbar_init(smem_u32(mb), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512u)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        const uint32_t sfa = tmem + 256, sfb = tmem + 272;  // accumulator in columns 0..255
        sf_copy(sfa, smem_u32(SFa));
        sf_copy(sfb, smem_u32(SFb));
        sf_copy(sfb + 4, smem_u32(SFb + 512));
        const uint32_t A_s = smem_u32(As), B_s = smem_u32(Bs);
        for (int it = 0; it < iters; ++it) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint64_t da = desc_smem(A_s + 32 * k, 16, 512, 4u);
                const uint64_t db = desc_smem(B_s + 32 * k, 16, 512, 4u);
                const uint32_t id = (uint32_t)(2 * k);
                mma_mxf4(tmem, da, db, idesc_mxf4(128, kProbeN, id, id), (it | k) != 0, sfa | (id << 30),
                         sfb | (id << 30));
            }
        }
        mma_commit(smem_u32(mb));
        if (!mbar_wait(smem_u32(mb), 0)) {  // flag it, and let the MMAs drain before TMEM is freed
            flag(status, CSA_DEV_TIMEOUT);
            mbar_wait_for(smem_u32(mb), 0, kDrainCycles);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u) : "memory");
}

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Row-major [rows][row_bytes] matrix in boxes of box_rows rows: bf16 in 64-channel
// boxes with a 128-byte swizzle, or MXFP4 codes (bytes) in whole-row boxes of
// row_bytes = 64 with a 64-byte swizzle.
bool encode_rows(CUtensorMap *tm, const void *base, uint64_t rows, int DI, bool mx, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
    const int row_bytes = mx ? DI / 2 : DI * 2;
    const cuuint64_t dims[2] = {(cuuint64_t)(mx ? row_bytes : DI), (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {mx ? (cuuint32_t)row_bytes : 64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(tm, mx ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               mx ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KF, int DI, int HI>
cudaError_t launch_pf(PfArgs &a, const void *keys, int batch, const void *q_rows, int num_sms, cudaStream_t s) {
    using C = PfCfg<KF, DI>;
    if (!encode_rows(&a.tm_keys, keys, (uint64_t)batch * a.cap, DI, C::MX, kPfKeys) ||
        !encode_rows(&a.tm_q, q_rows, (uint64_t)a.Nq * HI, DI, C::MX, kPfCols))
        return cudaErrorInvalidValue;
    cudaError_t err;
    if ((err = cudaFuncSetAttribute(prefill_score_kernel<KF, DI, HI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::SMEM)) != cudaSuccess)
        return err;
    const int ntiles = (a.Nq + kPfCols / HI - 1) / (kPfCols / HI);
    const int grid = max(1, min(num_sms, ntiles));
    return launch_pdl(prefill_score_kernel<KF, DI, HI>, dim3(grid), dim3(kPfThreads), (size_t)C::SMEM, s, a);
}

template <int KF, int DI>
cudaError_t launch_pf_heads(PfArgs &a, int H_I, const void *keys, int batch, const void *q_rows, int num_sms,
                            cudaStream_t s) {
    switch (H_I) {
        case 1: return launch_pf<KF, DI, 1>(a, keys, batch, q_rows, num_sms, s);
        case 2: return launch_pf<KF, DI, 2>(a, keys, batch, q_rows, num_sms, s);
        case 4: return launch_pf<KF, DI, 4>(a, keys, batch, q_rows, num_sms, s);
        case 8:
            if constexpr (KF == kPfBf16) return launch_pf<KF, DI, 8>(a, keys, batch, q_rows, num_sms, s);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

size_t align256_pf(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

bool prefill_scores_supported(int idx_dtype, int idx_dim, int H_I) {
    if (idx_dtype == CSA_IDX_BF16)
        return (idx_dim == 64 || idx_dim == 128 || idx_dim == 256) && (H_I == 1 || H_I == 2 || H_I == 4 || H_I == 8);
    if (idx_dtype == CSA_IDX_MXFP4) return idx_dim == 128 && (H_I == 1 || H_I == 2 || H_I == 4);
    return false;
}

// MXFP4 keys: scratch for the quantized query, codes [tiles * 128][d_I / 2] and its
// scale-factor blocks.
size_t prefill_query_scratch_bytes(int idx_dtype, int idx_dim, int Nq, int H_I) {
    if (idx_dtype != CSA_IDX_MXFP4) return 0;
    const size_t tiles = ((size_t)Nq * H_I + kPfCols - 1) / kPfCols;
    return align256_pf(tiles * kPfCols * (idx_dim / 2)) + tiles * kSfBlock;
}

// Score rows [Nq][rows] of every query's visible keys (bf16 or MXFP4 keys). MXFP4:
// q_scratch holds prefill_query_scratch_bytes() bytes (256-byte aligned).
cudaError_t launch_prefill_scores(const csa_cache &c, const void *q_idx, const float *w, int Nq, int H_I,
                                  const int32_t *req, const int32_t *n_vis, float *scores, int rows, void *q_scratch,
                                  int num_sms, cudaStream_t s) {
    PfArgs a;
    memset(&a, 0, sizeof(a));
    a.w = w;
    a.req = req;
    a.n_vis = n_vis;
    a.scores = scores;
    a.status = c.status;
    a.Nq = Nq;
    a.cap = c.capacity;
    a.rows = rows;
    a.key_rows = (long long)c.batch * c.capacity;
    if (c.idx_dtype == CSA_IDX_MXFP4) {
        if (c.idx_dim != 128 || (reinterpret_cast<uintptr_t>(c.idx_key_scale) & 3)) return cudaErrorInvalidValue;
        const int tiles = (int)(((long long)Nq * H_I + kPfCols - 1) / kPfCols);
        uint8_t *codes = static_cast<uint8_t *>(q_scratch);
        uint8_t *sf = codes + align256_pf((size_t)tiles * kPfCols * 64);
        const long long threads = (long long)tiles * kPfCols * 4;
        cudaError_t err = launch_pdl(quantize_query_kernel<128>, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0,
                                     s, static_cast<const __nv_bfloat16 *>(q_idx), Nq * H_I, tiles, codes, sf);
        if (err != cudaSuccess) return err;
        a.key_scales = c.idx_key_scale;
        a.q_sf = sf;
        return launch_pf_heads<kPfMxfp4, 128>(a, H_I, c.idx_key, c.batch, codes, num_sms, s);
    }
    switch (c.idx_dim) {
        case 64: return launch_pf_heads<kPfBf16, 64>(a, H_I, c.idx_key, c.batch, q_idx, num_sms, s);
        case 128: return launch_pf_heads<kPfBf16, 128>(a, H_I, c.idx_key, c.batch, q_idx, num_sms, s);
        case 256: return launch_pf_heads<kPfBf16, 256>(a, H_I, c.idx_key, c.batch, q_idx, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

// The MMA probe on every SM; FLOPs per launch = num_sms * iters * 2 * 128 * 256 * 128.
cudaError_t launch_mxf4_probe(int iters, int32_t *status, int num_sms, cudaStream_t s) {
    const int smem = 1024 + 128 * 64 + kProbeN * 64 + 1024 + 2048 + 64;
    cudaError_t err = cudaFuncSetAttribute(mxf4_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    mxf4_probe_kernel<<<num_sms, 128, smem, s>>>(iters, status);
    return cudaGetLastError();
}

}  // namespace csa
