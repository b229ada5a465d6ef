// prefill.cu -- row a3 when a request brings many queries (prefill): the
// indexer scores of every (query, visible block) pair as one tensor-core GEMM
// per request, instead of one key stream per query.
//
// Source: DeepSeek-V4.1-Flash podcast transcript, cue 12 (the indexer query
// scores the indexer keys; top-k over the scores); "Frontier Architecture
// Decoding Notes (4): DeepSeek V4", section 1 (top-k over 4-token blocks).
// Score form (the library's reading): s_j = sum_h w_h * ReLU(q_h . k_j).
//
// GEMM: rows (M) = (query, head) pairs, 128 per tile (128 / H_I consecutive
// queries of one request, head-minor so that a query's heads sit in adjacent
// TMEM lanes); columns (N) = the request's keys, 256 per key stage (128 for
// 256-channel keys); K = d_I. bf16 operands (the cache's bf16 keys and the bf16
// indexer query, exact products), fp32 accumulators in TMEM, two accumulator
// buffers so that the epilogue of one key stage overlaps the MMAs of the next.
// Operands arrive by TMA (tensor maps over the key plane and the query array,
// 128-byte swizzle; key stages are marked evict-last in L2, since every query
// tile of the request reads them again) into a ring of key stages; the query
// tile stays resident while the request's keys stream past.
// Warp roles (320 threads, one CTA per SM, persistent over query tiles):
//   warps 0-7  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (thread =
//              one (query, head) row) over half of the stage's columns; ReLU,
//              head weight, the sum over the query's H_I lanes (a transposing
//              butterfly: of every 32 columns each of those lanes ends with
//              32 / H_I finished scores), streaming stores to the score row
//   warp 8     lane 0 issues the MMAs and their commits
//   warp 9     lane 0 issues the TMA loads
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

constexpr int kPfRows = 128;     // MMA M: (query, head) rows of a tile
constexpr int kPfEpiWarps = 8;
constexpr int kPfThreads = 32 * (kPfEpiWarps + 2);

template <int DI>
struct PfCfg {
    static constexpr int NT = DI <= 128 ? 256 : 128;  // keys per stage (MMA N, TMA box height <= 256)
    static constexpr int A_REG = kPfRows * 128;        // one 64-channel K region of the query tile
    static constexpr int B_REG = NT * 128;             // ... of a key stage
    static constexpr int A_BYTES = (DI / 64) * A_REG;
    static constexpr int B_BYTES = (DI / 64) * B_REG;
    static constexpr int MISC = 1536;
    static constexpr int BUDGET = 232448 - 1024 - MISC - A_BYTES;  // opt-in shared memory per CTA
    static constexpr int STAGES = BUDGET / B_BYTES >= 4 ? 4 : BUDGET / B_BYTES;
    static constexpr int SMEM = 1024 + A_BYTES + STAGES * B_BYTES + MISC;
    static constexpr int TMEM_COLS = 2 * NT;
    static_assert(STAGES >= 2, "key ring needs two stages");
};

struct PfArgs {
    CUtensorMap tm_keys;         // [batch * cap][d_I] bf16, box 64 x NT
    CUtensorMap tm_q;            // [Nq * H_I][d_I] bf16, box 64 x 128
    const float *w;              // [Nq][H_I]
    const int32_t *req, *n_vis;  // [Nq], from the schedule kernel
    float *scores;               // [Nq][rows]
    int32_t *status;
    int Nq, cap, rows;
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
__device__ __forceinline__ void st_score4(float *p, float x, float y, float z, float w) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(x), "f"(y), "f"(z), "f"(w) : "memory");
}

template <int DI, int HI>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_score_kernel(const __grid_constant__ PfArgs a) {
    using C = PfCfg<DI>;
    constexpr int NT = C::NT;
    constexpr int ST = C::STAGES;
    constexpr int QT = kPfRows / HI;      // queries per tile
    constexpr int PER = 32 / HI;          // scores per lane per 32-column chunk
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *As = smem;
    uint8_t *Bs = As + C::A_BYTES;        // stage s at Bs + s B_BYTES
    uint8_t *misc = Bs + ST * C::B_BYTES;
    // barriers: query tile full / free, key stages full / free, accumulators full / free (2 buffers)
    enum { B_AFULL = 0, B_AFREE = 1, B_BFULL = 2, B_BFREE = 2 + ST, B_CFULL = 2 + 2 * ST, B_CFREE = 4 + 2 * ST };
    uint64_t *mb = reinterpret_cast<uint64_t *>(misc);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 128);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 132);
    int *n_sub = reinterpret_cast<int *>(misc + 136);
    // [QT <= 128] (request, visible blocks) of each query of the tile, then, in place, the
    // requests present in the tile with their largest visible-block count
    int2 *q_rn = reinterpret_cast<int2 *>(misc + 256);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto bar = [&](int k) { return smem_u32(&mb[k]); };
    const uint32_t A_s = smem_u32(As), B_s = smem_u32(Bs);
    if (tid == 0) {
        mbar_init(bar(B_AFULL), 1);
        mbar_init(bar(B_AFREE), 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar(B_BFULL + s), 1);
            mbar_init(bar(B_BFREE + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_CFULL + s), 1);
            mbar_init(bar(B_CFREE + s), 32 * kPfEpiWarps);
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
    grid_dep_wait();  // the schedule kernel's req / n_vis

    constexpr uint32_t IDESC = idesc_bf16(kPfRows, NT);
    const int ntiles = (a.Nq + QT - 1) / QT;
    uint32_t gkt = 0;  // key stages of this CTA so far (ring slot, accumulator and phases)
    uint32_t ns = 0;   // (tile, request) items of this CTA so far
    bool ok = true;

    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int q0 = tile * QT;
        if (__syncthreads_or(!ok)) break;
        // per-query data of the tile (in parallel), then the requests present in it
        // (queries are ordered by request: runs of one request), by one thread from shared memory
        if (tid < QT) {
            const int q = q0 + tid;
            q_rn[tid] = q < a.Nq ? make_int2(a.req[q], min(a.n_vis[q], a.cap)) : make_int2(-1, 0);
        }
        __syncthreads();
        if (tid == 0) {  // entry cnt - 1 <= qq: only entries already read are overwritten
            int cnt = 0;
            for (int qq = 0; qq < QT; ++qq) {
                const int2 rn = q_rn[qq];
                if (rn.x < 0) continue;
                if (cnt == 0 || q_rn[cnt - 1].x != rn.x) q_rn[cnt++] = rn;
                else q_rn[cnt - 1].y = max(q_rn[cnt - 1].y, rn.y);
            }
            *n_sub = cnt;
        }
        __syncthreads();
        const int nsub = *n_sub;
        for (int si = 0; si < nsub && ok; ++si) {
            const int b = q_rn[si].x;
            const int maxn = q_rn[si].y;
            const int nkt = (maxn + NT - 1) / NT;
            if (nkt == 0) continue;
            if (warp == 9) {
                // ================= TMA producer
                if (lane == 0) {
                    const uint64_t pol = policy_evict_last();
                    if (ns >= 1) ok = mbar_wait_ab<false>(bar(B_AFREE), (ns - 1) & 1, abort_flag);
                    if (ok) {  // the query tile: rows (query, head) from q0 H_I; rows past the array read zeros
                        mbar_expect_tx(bar(B_AFULL), (uint32_t)C::A_BYTES);
#pragma unroll
                        for (int r = 0; r < DI / 64; ++r)
                            tma_load_2d(A_s + r * C::A_REG, &a.tm_q, 64 * r, q0 * HI, bar(B_AFULL));
                    }
                    for (int kt = 0; kt < nkt && ok; ++kt) {
                        const uint32_t g = gkt + kt, s = g % ST;
                        if (g >= (uint32_t)ST) ok = mbar_wait_ab<false>(bar(B_BFREE + s), ((g / ST) - 1) & 1, abort_flag);
                        if (!ok) break;
                        // keys kt NT .. + NT - 1 of request b; columns past the visible ones are never stored
                        mbar_expect_tx(bar(B_BFULL + s), (uint32_t)C::B_BYTES);
#pragma unroll
                        for (int r = 0; r < DI / 64; ++r)
                            tma_load_2d_hint(B_s + s * C::B_BYTES + r * C::B_REG, &a.tm_keys, 64 * r,
                                             b * a.cap + kt * NT, bar(B_BFULL + s), pol);
                    }
                    if (!ok) *abort_flag = 1;
                }
                ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
            } else if (warp == 8) {
                // ================= MMA issue
                if (lane == 0) {
                    ok = mbar_wait_ab<false>(bar(B_AFULL), ns & 1, abort_flag);
                    for (int kt = 0; kt < nkt && ok; ++kt) {
                        const uint32_t g = gkt + kt, s = g % ST, acc = g & 1;
                        ok = mbar_wait_ab<false>(bar(B_BFULL + s), (g / ST) & 1, abort_flag);
                        if (ok && g >= 2) ok = mbar_wait_ab<false>(bar(B_CFREE + acc), ((g >> 1) - 1) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < DI / 16; ++kk) {
                            const uint32_t koff = (uint32_t)((kk & 3) * 32);
                            const uint64_t da = desc_sw128(A_s + (kk >> 2) * C::A_REG + koff, 16, 1024);
                            const uint64_t db = desc_sw128(B_s + s * C::B_BYTES + (kk >> 2) * C::B_REG + koff, 16, 1024);
                            mma_f16(tmem + acc * NT, da, db, IDESC, kk > 0);
                        }
                        mma_commit(bar(B_BFREE + s));
                        mma_commit(bar(B_CFULL + acc));
                    }
                    if (ok) mma_commit(bar(B_AFREE));
                    if (!ok) *abort_flag = 1;
                }
                ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
            } else {
                // ================= epilogue: TMEM lane r = (query, head), half of the columns
                const int r = 32 * (warp & 3) + lane;
                const int c0 = (warp >> 2) * (NT / 2);
                const int q = q0 + r / HI, h = r % HI;
                const bool live = q < a.Nq && a.req[q] == b;
                const float wv = live ? a.w[(size_t)q * HI + h] : 0.f;
                const int n = live ? min(a.n_vis[q], a.cap) : 0;
                float *srow = a.scores + (size_t)(live ? q : 0) * a.rows;
                const bool vec_ok = (a.rows & 3) == 0;  // 16-byte aligned row starts
                const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
                for (int kt = 0; kt < nkt; ++kt) {
                    const uint32_t g = gkt + kt, acc = g & 1;
                    ok = mbar_wait_ab<false>(bar(B_CFULL + acc), (g >> 1) & 1, abort_flag);
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < NT / 64; ++c) {
                        float v[32];
                        tmem_ld32(tmem + lane_off + acc * NT + c0 + 32 * c, v);
#pragma unroll
                        for (int k = 0; k < 32; ++k) v[k] = wv * fmaxf(v[k], 0.f);
                        // sum over the HI lanes of this query; lane h keeps columns h PER .. h PER + PER - 1
                        int m = 32;
#pragma unroll
                        for (int st = HI / 2; st >= 1; st >>= 1) {
                            const bool hi = (lane & st) != 0;
                            m >>= 1;
#pragma unroll
                            for (int k = 0; k < 16; ++k) {
                                if (k < m) {
                                    const float send = hi ? v[k] : v[k + m];
                                    const float keep = hi ? v[k + m] : v[k];
                                    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, st);
                                }
                            }
                        }
                        const int j0 = kt * NT + c0 + 32 * c + h * PER;
                        if (live && vec_ok && j0 + PER <= n) {
#pragma unroll
                            for (int e = 0; e < PER; e += 4) st_score4(srow + j0 + e, v[e], v[e + 1], v[e + 2], v[e + 3]);
                        } else if (live) {
#pragma unroll
                            for (int e = 0; e < PER; ++e)
                                if (j0 + e < n) st_score(srow + j0 + e, v[e]);
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(bar(B_CFREE + acc));
                }
                if (!ok) *abort_flag = 1;
            }
            gkt += nkt;
            ++ns;
        }
    }
    if (tid == 256 && ns >= 1 && ok) mbar_wait(bar(B_AFREE), (ns - 1) & 1);  // last commit landed
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

// Row-major bf16 [rows][DI] matrix, boxes of 64 channels x box_rows rows, 128-byte swizzle.
bool encode_rows(CUtensorMap *tm, const void *base, uint64_t rows, int DI, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)DI, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)DI * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DI, int HI>
cudaError_t launch_pf(PfArgs &a, const void *keys, int batch, const void *q_idx, int num_sms, cudaStream_t s) {
    using C = PfCfg<DI>;
    if (!encode_rows(&a.tm_keys, keys, (uint64_t)batch * a.cap, DI, C::NT) ||
        !encode_rows(&a.tm_q, q_idx, (uint64_t)a.Nq * HI, DI, kPfRows))
        return cudaErrorInvalidValue;
    cudaError_t err;
    if ((err = cudaFuncSetAttribute(prefill_score_kernel<DI, HI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::SMEM)) != cudaSuccess)
        return err;
    const int ntiles = (a.Nq + kPfRows / HI - 1) / (kPfRows / HI);
    const int grid = max(1, min(num_sms, ntiles));
    return launch_pdl(prefill_score_kernel<DI, HI>, dim3(grid), dim3(kPfThreads), (size_t)C::SMEM, s, a);
}

template <int DI>
cudaError_t launch_pf_heads(PfArgs &a, int H_I, const void *keys, int batch, const void *q_idx, int num_sms,
                            cudaStream_t s) {
    switch (H_I) {
        case 1: return launch_pf<DI, 1>(a, keys, batch, q_idx, num_sms, s);
        case 2: return launch_pf<DI, 2>(a, keys, batch, q_idx, num_sms, s);
        case 4: return launch_pf<DI, 4>(a, keys, batch, q_idx, num_sms, s);
        case 8: return launch_pf<DI, 8>(a, keys, batch, q_idx, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool prefill_scores_supported(int idx_dtype, int idx_dim, int H_I) {
    return idx_dtype == CSA_IDX_BF16 && (idx_dim == 64 || idx_dim == 128 || idx_dim == 256) &&
           (H_I == 1 || H_I == 2 || H_I == 4 || H_I == 8);
}

// Score rows [Nq][rows] of every query's visible keys, for bf16 keys.
cudaError_t launch_prefill_scores(const void *keys, int batch, int cap, int idx_dim, const void *q_idx, const float *w,
                                  int Nq, int H_I, const int32_t *req, const int32_t *n_vis, float *scores, int rows,
                                  int32_t *status, int num_sms, cudaStream_t s) {
    PfArgs a;
    memset(&a, 0, sizeof(a));
    a.w = w;
    a.req = req;
    a.n_vis = n_vis;
    a.scores = scores;
    a.status = status;
    a.Nq = Nq;
    a.cap = cap;
    a.rows = rows;
    switch (idx_dim) {
        case 64: return launch_pf_heads<64>(a, H_I, keys, batch, q_idx, num_sms, s);
        case 128: return launch_pf_heads<128>(a, H_I, keys, batch, q_idx, num_sms, s);
        case 256: return launch_pf_heads<256>(a, H_I, keys, batch, q_idx, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
