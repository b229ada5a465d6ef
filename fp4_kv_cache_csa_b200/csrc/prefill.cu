// prefill.cu -- row a3 when a request brings many queries (prefill): the
// indexer scores of every (query, visible block) pair as one tensor-core GEMM
// per request, instead of one key stream per query.
//
// Source: DeepSeek-V4.1-Flash podcast transcript, cue 12 (the indexer query
// scores the indexer keys; top-k over the scores); "Frontier Architecture
// Decoding Notes (4): DeepSeek V4", section 1 (top-k over 4-token blocks).
// Score form (the library's reading): s_j = sum_h w_h * ReLU(q_h . k_j).
//
// GEMM: rows = (query, head) pairs, 128 per tile (128 / H_I consecutive
// queries of one request, head-minor so that a query's heads sit in adjacent
// TMEM lanes); columns = the request's keys, NT per tile; K = d_I. bf16
// operands (the cache's bf16 keys and the bf16 indexer query, exact products),
// fp32 accumulators in TMEM, two accumulator buffers so that the epilogue of
// one key tile overlaps the MMAs of the next.
// Warp roles (288 threads, one CTA per SM, persistent over query tiles):
//   warps 0-3  epilogue: thread r owns TMEM lane r; ReLU, head weight, the sum
//              over the query's H_I lanes (a transposing butterfly: of every 32
//              columns each of those lanes ends with 32 / H_I finished scores),
//              stores to the score row
//   warps 4-7  loaders: the query tile (once per tile) and the key tiles (two
//              stages) with cp.async into the 128-byte-swizzled K-major layout
//   warp 8     lane 0 issues the MMAs and their commits
// The score rows, the per-query thresholds and the selection that follow are
// the same as for the key-stream scan, so the selection kernels are shared.
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_util.cuh"

namespace csa {

namespace {

constexpr int kPfRows = 128;     // MMA M: (query, head) rows of a tile
constexpr int kPfThreads = 288;  // epilogue warps 0-3, loader warps 4-7, MMA warp 8

template <int DI>
struct PfCfg {
    static constexpr int NT = DI <= 128 ? 256 : 128;  // keys per tile (MMA N)
    static constexpr int A_REG = kPfRows * 128;        // one 64-channel K region of the query tile
    static constexpr int B_REG = NT * 128;             // ... of a key tile
    static constexpr int A_BYTES = (DI / 64) * A_REG;
    static constexpr int B_BYTES = (DI / 64) * B_REG;
    static constexpr int MISC = 2048;
    static constexpr int SMEM = 1024 + A_BYTES + 2 * B_BYTES + MISC;
    static constexpr int TMEM_COLS = 2 * NT;
};

struct PfArgs {
    const __nv_bfloat16 *keys;   // [batch][cap][d_I]
    const __nv_bfloat16 *q_idx;  // [Nq][H_I][d_I]
    const float *w;              // [Nq][H_I]
    const int32_t *req, *n_vis;  // [Nq], from the schedule kernel
    float *scores;               // [Nq][rows]
    int32_t *status;
    int Nq, cap, rows;
};

// Swizzled byte offset of 16-byte chunk kc (channels 8 kc .. 8 kc + 7) of row r
// in a K-major operand of `reg` bytes per 64-channel region.
__device__ __forceinline__ uint32_t pf_chunk(int r, int kc, int reg) {
    return (uint32_t)((kc >> 3) * reg + (r >> 3) * 1024 + (r & 7) * 128 + (((kc & 7) ^ (r & 7)) << 4));
}

// Score rows are read again by the selection kernels: keep them in L2.
__device__ __forceinline__ uint64_t policy_keep() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void st_score(float *p, float v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_score4(float *p, float x, float y, float z, float w, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(x), "f"(y), "f"(z),
                 "f"(w), "l"(pol)
                 : "memory");
}

template <int DI, int HI>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_score_kernel(PfArgs a) {
    using C = PfCfg<DI>;
    constexpr int NT = C::NT;
    constexpr int QT = kPfRows / HI;      // queries per tile
    constexpr int PER = 32 / HI;          // scores per lane per 32-column chunk
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *As = smem;
    uint8_t *Bs = As + C::A_BYTES;        // stage s at Bs + s B_BYTES
    uint8_t *misc = Bs + 2 * C::B_BYTES;
    // barriers: A full / free, B full / free (2 stages), accumulator full / free (2 buffers)
    enum { B_AFULL = 0, B_AFREE = 1, B_BFULL = 2, B_BFREE = 4, B_CFULL = 6, B_CFREE = 8 };
    uint64_t *mb = reinterpret_cast<uint64_t *>(misc);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 128);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 132);
    int *n_sub = reinterpret_cast<int *>(misc + 136);
    int *sub_b = reinterpret_cast<int *>(misc + 512);      // [QT <= 128] requests present in the tile
    int *sub_n = reinterpret_cast<int *>(misc + 1024);     // [QT] their largest visible-block count

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto bar = [&](int k) { return smem_u32(&mb[k]); };
    const uint32_t A_s = smem_u32(As), B_s = smem_u32(Bs);
    if (tid == 0) {
        mbar_init(bar(B_AFULL), 128);
        mbar_init(bar(B_AFREE), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_BFULL + s), 128);
            mbar_init(bar(B_BFREE + s), 1);
            mbar_init(bar(B_CFULL + s), 1);
            mbar_init(bar(B_CFREE + s), 128);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        *abort_flag = 0;
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
    const uint64_t pol_keep = policy_keep();
    const int ntiles = (a.Nq + QT - 1) / QT;
    uint32_t gkt = 0;  // key tiles of this CTA so far (stage and accumulator index and phases)
    uint32_t ns = 0;   // (tile, request) items of this CTA so far
    bool ok = true;

    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int q0 = tile * QT;
        // the requests present in this tile (queries are ordered by request)
        if (__syncthreads_or(!ok)) break;
        if (tid == 0) {
            int cnt = 0;
            for (int qq = 0; qq < QT && q0 + qq < a.Nq; ++qq) {
                const int b = a.req[q0 + qq];
                const int n = a.n_vis[q0 + qq];
                if (b < 0) continue;
                if (cnt == 0 || sub_b[cnt - 1] != b) {
                    sub_b[cnt] = b;
                    sub_n[cnt] = 0;
                    ++cnt;
                }
                sub_n[cnt - 1] = max(sub_n[cnt - 1], n);
            }
            *n_sub = cnt;
        }
        __syncthreads();
        const int nsub = *n_sub;
        for (int si = 0; si < nsub && ok; ++si) {
            const int b = sub_b[si];
            const int maxn = min(sub_n[si], a.cap);
            const int nkt = (maxn + NT - 1) / NT;
            if (nkt == 0) continue;
            if (warp >= 4 && warp < 8) {
                // ================= loaders
                const int lt = tid - 128;
                if (ns >= 1) ok = mbar_wait_ab<false>(bar(B_AFREE), (ns - 1) & 1, abort_flag);
                if (ok) {  // query tile: row lt = (query q0 + lt / HI, head lt % HI)
                    const int q = q0 + lt / HI;
                    const bool live = q < a.Nq && a.req[q] == b;
                    const __nv_bfloat16 *src = a.q_idx + ((size_t)q * HI + lt % HI) * DI;
#pragma unroll
                    for (int kc = 0; kc < DI / 8; ++kc) {
                        if (live)
                            cp_async16(A_s + pf_chunk(lt, kc, C::A_REG), src + 8 * kc);
                        else
                            *reinterpret_cast<uint4 *>(As + pf_chunk(lt, kc, C::A_REG)) = make_uint4(0, 0, 0, 0);
                    }
                    asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
                    fence_async_smem();
                    mbar_arrive(bar(B_AFULL));
                }
                for (int kt = 0; kt < nkt && ok; ++kt) {
                    const uint32_t g = gkt + kt, s = g & 1;
                    if (g >= 2) ok = mbar_wait_ab<false>(bar(B_BFREE + s), ((g >> 1) - 1) & 1, abort_flag);
                    if (!ok) break;
                    uint8_t *Bst = Bs + s * C::B_BYTES;
                    const uint32_t Bst_s = B_s + s * C::B_BYTES;
#pragma unroll
                    for (int u = 0; u < NT / 128; ++u) {
                        const int jr = lt + 128 * u;
                        const int j = kt * NT + jr;
                        const __nv_bfloat16 *src = a.keys + ((size_t)b * a.cap + j) * DI;
#pragma unroll
                        for (int kc = 0; kc < DI / 8; ++kc) {
                            if (j < maxn)
                                cp_async16(Bst_s + pf_chunk(jr, kc, C::B_REG), src + 8 * kc);
                            else
                                *reinterpret_cast<uint4 *>(Bst + pf_chunk(jr, kc, C::B_REG)) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
                    fence_async_smem();
                    mbar_arrive(bar(B_BFULL + s));
                }
                if (!ok) *abort_flag = 1;
            } else if (warp == 8) {
                // ================= MMA issue
                if (lane == 0) {
                    ok = mbar_wait_ab<false>(bar(B_AFULL), ns & 1, abort_flag);
                    for (int kt = 0; kt < nkt && ok; ++kt) {
                        const uint32_t g = gkt + kt, s = g & 1;
                        ok = mbar_wait_ab<false>(bar(B_BFULL + s), (g >> 1) & 1, abort_flag);
                        if (ok && g >= 2) ok = mbar_wait_ab<false>(bar(B_CFREE + s), ((g >> 1) - 1) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < DI / 16; ++kk) {
                            const uint32_t koff = (uint32_t)((kk & 3) * 32);
                            const uint64_t da = desc_sw128(A_s + (kk >> 2) * C::A_REG + koff, 16, 1024);
                            const uint64_t db = desc_sw128(B_s + s * C::B_BYTES + (kk >> 2) * C::B_REG + koff, 16, 1024);
                            mma_f16(tmem + s * NT, da, db, IDESC, kk > 0);
                        }
                        mma_commit(bar(B_BFREE + s));
                        mma_commit(bar(B_CFULL + s));
                    }
                    if (ok) mma_commit(bar(B_AFREE));
                    if (!ok) *abort_flag = 1;
                }
                ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
            } else {
                // ================= epilogue: thread tid owns TMEM lane tid = (query, head)
                const int q = q0 + tid / HI, h = tid % HI;
                const bool live = q < a.Nq && a.req[q] == b;
                const float wv = live ? a.w[(size_t)q * HI + h] : 0.f;
                const int n = live ? min(a.n_vis[q], a.cap) : 0;
                float *srow = a.scores + (size_t)(live ? q : 0) * a.rows;
                const bool vec_ok = (a.rows & 3) == 0;  // 16-byte aligned row starts
                const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
                for (int kt = 0; kt < nkt; ++kt) {
                    const uint32_t g = gkt + kt, s = g & 1;
                    ok = mbar_wait_ab<false>(bar(B_CFULL + s), (g >> 1) & 1, abort_flag);
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < NT / 32; ++c) {
                        float v[32];
                        tmem_ld32(tmem + lane_off + s * NT + 32 * c, v);
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
                        const int j0 = kt * NT + 32 * c + h * PER;
                        if (live && vec_ok && j0 + PER <= n) {
#pragma unroll
                            for (int e = 0; e < PER; e += 4)
                                st_score4(srow + j0 + e, v[e], v[e + 1], v[e + 2], v[e + 3], pol_keep);
                        } else if (live) {
#pragma unroll
                            for (int e = 0; e < PER; ++e)
                                if (j0 + e < n) st_score(srow + j0 + e, v[e], pol_keep);
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(bar(B_CFREE + s));
                }
                if (!ok) *abort_flag = 1;
            }
            gkt += nkt;
            ++ns;
        }
    }
    if (tid == 256 && ns >= 1 && ok) mbar_wait(bar(B_AFREE), (ns - 1) & 1);  // last commit landed
    if (__syncthreads_or(!ok) && tid == 0) flag(a.status, CSA_DEV_TIMEOUT);
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok && tid == 256) {  // let tensor-core work already issued finish before TMEM is released
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

template <int DI, int HI>
cudaError_t launch_pf(const PfArgs &a, int num_sms, cudaStream_t s) {
    cudaError_t err;
    if ((err = cudaFuncSetAttribute(prefill_score_kernel<DI, HI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    PfCfg<DI>::SMEM)) != cudaSuccess)
        return err;
    const int ntiles = (a.Nq + kPfRows / HI - 1) / (kPfRows / HI);
    const int grid = max(1, min(num_sms, ntiles));
    return launch_pdl(prefill_score_kernel<DI, HI>, dim3(grid), dim3(kPfThreads), (size_t)PfCfg<DI>::SMEM, s, a);
}

template <int DI>
cudaError_t launch_pf_heads(const PfArgs &a, int H_I, int num_sms, cudaStream_t s) {
    switch (H_I) {
        case 1: return launch_pf<DI, 1>(a, num_sms, s);
        case 2: return launch_pf<DI, 2>(a, num_sms, s);
        case 4: return launch_pf<DI, 4>(a, num_sms, s);
        case 8: return launch_pf<DI, 8>(a, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool prefill_scores_supported(int idx_dtype, int idx_dim, int H_I) {
    return idx_dtype == CSA_IDX_BF16 && (idx_dim == 64 || idx_dim == 128 || idx_dim == 256) &&
           (H_I == 1 || H_I == 2 || H_I == 4 || H_I == 8);
}

// Score rows [Nq][rows] of every query's visible keys, for bf16 keys.
cudaError_t launch_prefill_scores(const void *keys, int cap, int idx_dim, const void *q_idx, const float *w, int Nq,
                                  int H_I, const int32_t *req, const int32_t *n_vis, float *scores, int rows,
                                  int32_t *status, int num_sms, cudaStream_t s) {
    PfArgs a;
    a.keys = static_cast<const __nv_bfloat16 *>(keys);
    a.q_idx = static_cast<const __nv_bfloat16 *>(q_idx);
    a.w = w;
    a.req = req;
    a.n_vis = n_vis;
    a.scores = scores;
    a.status = status;
    a.Nq = Nq;
    a.cap = cap;
    a.rows = rows;
    switch (idx_dim) {
        case 64: return launch_pf_heads<64>(a, H_I, num_sms, s);
        case 128: return launch_pf_heads<128>(a, H_I, num_sms, s);
        case 256: return launch_pf_heads<256>(a, H_I, num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
