// compress.cu -- rows a1 + a2: softmax-gated m-token pooling and MXFP4
// quantization of the pooled entry, plus the pooled indexer key.
//
// Source: "Frontier Architecture Decoding Notes (4): DeepSeek V4", section 1
// (KV of every 4 tokens compressed into one entry for CSA, up to 128 for HCA);
// DeepSeek-V4.1-Flash podcast transcript, cue 16 (main KV stored as MXFP4,
// E2M1 elements with one E4M3 scale per sixteen channels). Pooling form, gate
// and the E8M0/32 scale (the default format): the library's stated readings
// (see include/csa.h).
//
// One warp builds one block (eight warps share a block when m >= 32). Lane l
// owns E = D/32 consecutive channels [l*E, l*E+E) and EI = dI/32 consecutive
// indexer channels, so every token row is read as one coalesced warp-wide load;
// four tokens are loaded per step. The gate softmax is computed online
// (running max and rescaled sums) in a single pass over the m tokens. The
// kernel is HBM-bound: it reads m*(D+dI)*2 bytes and writes D/2 + D/32 + key
// bytes per block.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace csa {

namespace {

constexpr int kWarpsPerCta = 4;

// E2M1 code of v / s for a group scale s > 0 (E4M3 scales), from the rounding
// midpoints scaled by s: th[k] = mid_k * s is exact in float32 (a midpoint has
// at most 3 significant bits, an E4M3 value 4), so comparing |v| with th[k]
// takes the decision on the exact quotient, with no division. Same tie rule
// and saturation as e2m1_code. s = 0 is passed as +inf: every code is a zero
// magnitude with the element's sign.
__device__ __forceinline__ uint32_t e2m1_code_th(float v, const float (&th)[7]) {
    uint32_t sign = (__float_as_uint(v) >> 28) & 8u;
    float a = fabsf(v);
    uint32_t c = a <= th[0] ? 0u : a < th[1] ? 1u : a <= th[2] ? 2u : a < th[3] ? 3u
               : a <= th[4] ? 4u : a < th[5] ? 5u : a <= th[6] ? 6u : 7u;
    return sign | c;
}

// N consecutive bf16 values as N/2 raw 32-bit words (widest loads that fit).
template <int N>
__device__ __forceinline__ void load_raw(const __nv_bfloat16 *p, uint32_t (&w)[N / 2]) {
    static_assert(N % 2 == 0, "even channel count per lane");
    if constexpr (N % 8 == 0) {
#pragma unroll
        for (int v = 0; v < N / 8; ++v) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p) + v);
            w[4 * v] = u.x;
            w[4 * v + 1] = u.y;
            w[4 * v + 2] = u.z;
            w[4 * v + 3] = u.w;
        }
    } else if constexpr (N % 4 == 0) {
#pragma unroll
        for (int v = 0; v < N / 4; ++v) {
            const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p) + v);
            w[2 * v] = u.x;
            w[2 * v + 1] = u.y;
        }
    } else {
#pragma unroll
        for (int v = 0; v < N / 2; ++v) w[v] = __ldg(reinterpret_cast<const uint32_t *>(p) + v);
    }
}

template <int N>
__device__ __forceinline__ void unpack_bf16(const uint32_t (&w)[N / 2], float (&x)[N]) {
#pragma unroll
    for (int v = 0; v < N / 2; ++v) {
        __nv_bfloat162 h;
        *reinterpret_cast<uint32_t *>(&h) = w[v];
        const float2 f = __bfloat1622float2(h);
        x[2 * v] = f.x;
        x[2 * v + 1] = f.y;
    }
}

struct CompressArgs {
    const __nv_bfloat16 *kv_tok;   // [n_tokens][D]
    const __nv_bfloat16 *idx_tok;  // [n_tokens][dI] or null
    const float *gate_w;           // [D]
    const int32_t *tok_offsets;    // [B+1]
    const int32_t *n_blocks;       // [B]
    uint8_t *fp4;                  // [B][cap][D/2]
    uint8_t *scale;                // [B][cap][D/32] (E8M0) or [B][cap][D/16] (E4M3)
    uint8_t *idx_key;              // [B][cap][dI * esize], [B][cap][dI/2] (MXFP4 codes) or null
    uint8_t *idx_key_scale;        // [B][cap][dI/32] (MXFP4 keys) or null
    int32_t *status;
    int m, cap, D, dI;
    int idx_e4m3;
    int idx_mxfp4;
    int scale_e4m3;                // 1: one E4M3 scale per 16 elements, 0: one E8M0 scale per 32
    int batch;
    int flat;                      // 1: grid over all blocks of all requests (see below)
};

// Flat grid: the blocks of all requests in one list, request by request; a
// request whose token count is not a multiple of m has none. Every CTA builds
// the per-request block prefix in shared memory (s_pref[b] = blocks before
// request b, batch + 1 entries) and finds the request of its flat block by
// binary search, so no CTA is launched for a request's missing blocks.
constexpr int kFlatMaxBatch = 2047;

// E channels per lane (D = 32*E), EI indexer channels per lane (0 = no
// indexer keys), WPB warps per block: WPB = 1 puts four independent blocks in
// a CTA; WPB > 1 splits one block's tokens over WPB warps (large m), whose
// online-softmax states are then combined through shared memory. Each warp
// loads kChunk tokens at a time.
template <int E, int EI, int WPB>
__global__ void __launch_bounds__(WPB == 1 ? kWarpsPerCta * kWarp : WPB * kWarp)
pool_quantize_kernel(CompressArgs a) {
    constexpr int EK = EI > 0 ? EI : 2;
    // tokens in flight per warp step (fewer where 16 warps would run out of registers)
    constexpr int kChunk = WPB == 1 ? 4 : (WPB == 16 && E + EK >= 20) ? 4 : 8;
    // inputs may come from the previous kernel on the stream: wait for it, then
    // let the next kernel (the commit) begin launching
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int wib = WPB == 1 ? 0 : warp;  // warp index inside the block's team
    int b, jb;
    bool active;
    if (a.flat) {
        extern __shared__ int s_pref[];  // [batch + 1]
        __shared__ int scan_smem[32];
        __shared__ int round_total;
        int carry = 0;
        for (int r0 = 0; r0 < a.batch; r0 += blockDim.x) {
            const int r = r0 + (int)threadIdx.x;
            int nbr = 0;
            if (r < a.batch) {
                const int cnt = a.tok_offsets[r + 1] - a.tok_offsets[r];
                const bool ok = cnt >= 0 && cnt % a.m == 0;
                nbr = ok ? cnt / a.m : 0;
                if (!ok && blockIdx.x == 0) flag(a.status, CSA_DEV_TOKEN_COUNT);
            }
            const int incl = block_inclusive_scan<int>(nbr, scan_smem);
            if (r < a.batch) s_pref[r + 1] = carry + incl;
            if (threadIdx.x == blockDim.x - 1) round_total = incl;
            __syncthreads();
            carry += round_total;
            __syncthreads();
        }
        if (threadIdx.x == 0) s_pref[0] = 0;
        __syncthreads();
        const int gb = WPB == 1 ? blockIdx.x * kWarpsPerCta + warp : blockIdx.x;
        active = gb < s_pref[a.batch];  // CTA-uniform when WPB > 1
        b = 0;
        jb = 0;
        if (active) {
            int lo = 0, hi = a.batch - 1;  // last request with s_pref[b] <= gb
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_pref[mid] <= gb) lo = mid; else hi = mid - 1;
            }
            b = lo;
            jb = gb - s_pref[lo];
        }
    } else {
        b = blockIdx.y;
        jb = WPB == 1 ? blockIdx.x * kWarpsPerCta + warp : blockIdx.x;
        active = true;  // narrowed below
    }
    const int t_begin = a.tok_offsets[b];
    const int count = a.tok_offsets[b + 1] - t_begin;
    const bool count_ok = count >= 0 && count % a.m == 0;
    const int nb = count_ok ? count / a.m : 0;
    active = active && jb < nb;  // CTA-uniform when WPB > 1
    const int base = a.n_blocks[b];  // checked after the token loads are in flight

    float wg[E];
#pragma unroll
    for (int k = 0; k < E; ++k) wg[k] = __ldg(a.gate_w + lane * E + k);

    // Online softmax over this warp's tokens: mu = running max logit,
    // den = sum exp(g - mu), acc = sum exp(g - mu) * x.
    float acc[E], acck[EK];
    float mu = -INFINITY, den = 0.f;
#pragma unroll
    for (int k = 0; k < E; ++k) acc[k] = 0.f;
#pragma unroll
    for (int k = 0; k < EK; ++k) acck[k] = 0.f;

    const long long tok0 = (long long)t_begin + (long long)jb * a.m;
    for (int c0 = wib * kChunk; active && c0 < a.m; c0 += WPB * kChunk) {
        uint32_t xr[kChunk][E / 2], kr[kChunk][EK / 2];
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
            if (c0 + u < a.m) {
                load_raw<E>(a.kv_tok + (tok0 + c0 + u) * a.D + lane * E, xr[u]);
                if constexpr (EI > 0) load_raw<EI>(a.idx_tok + (tok0 + c0 + u) * a.dI + lane * EI, kr[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
            if (c0 + u < a.m) {
                float x[E];
                unpack_bf16<E>(xr[u], x);
                float part = 0.f;
#pragma unroll
                for (int k = 0; k < E; ++k) part = fmaf(x[k], wg[k], part);
                const float g = warp_sum(part);
                if (g > mu) {  // new maximum: rescale what has been accumulated
                    const float r = (mu == -INFINITY) ? 0.f : expf(mu - g);
                    den *= r;
#pragma unroll
                    for (int k = 0; k < E; ++k) acc[k] *= r;
#pragma unroll
                    for (int k = 0; k < EK; ++k) acck[k] *= r;
                    mu = g;
                }
                const float p = expf(g - mu);
                den += p;
#pragma unroll
                for (int k = 0; k < E; ++k) acc[k] = fmaf(p, x[k], acc[k]);
                if constexpr (EI > 0) {
                    float xk[EI];
                    unpack_bf16<EI>(kr[u], xk);
#pragma unroll
                    for (int k = 0; k < EI; ++k) acck[k] = fmaf(p, xk[k], acck[k]);
                }
            }
        }
    }

    if (!count_ok) {  // (flat grid: flagged above; only an idle CTA gets here)
        if (!a.flat && jb == 0 && threadIdx.x == 0) flag(a.status, CSA_DEV_TOKEN_COUNT);
        return;
    }
    if ((long long)base + nb > a.cap) {
        if (jb == 0 && threadIdx.x == 0) flag(a.status, CSA_DEV_CAPACITY);
        return;
    }
    if (!active) return;

    if constexpr (WPB > 1) {
        // combine the warps' partial softmax states; warp 0 finishes the block.
        // Channel k of lane l sits at [k][l]: consecutive lanes hit consecutive banks.
        __shared__ float s_mu[WPB], s_den[WPB];
        __shared__ float s_acc[WPB][E][32];
        __shared__ float s_acck[WPB][EK][32];
        if (lane == 0) {
            s_mu[warp] = mu;
            s_den[warp] = den;
        }
#pragma unroll
        for (int k = 0; k < E; ++k) s_acc[warp][k][lane] = acc[k];
#pragma unroll
        for (int k = 0; k < EK; ++k) s_acck[warp][k][lane] = acck[k];
        __syncthreads();
        if (warp != 0) return;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < WPB; ++w) M = fmaxf(M, s_mu[w]);
        den = 0.f;
#pragma unroll
        for (int k = 0; k < E; ++k) acc[k] = 0.f;
#pragma unroll
        for (int k = 0; k < EK; ++k) acck[k] = 0.f;
#pragma unroll
        for (int w = 0; w < WPB; ++w) {
            const float f = (s_mu[w] == -INFINITY) ? 0.f : expf(s_mu[w] - M);
            den = fmaf(s_den[w], f, den);
#pragma unroll
            for (int k = 0; k < E; ++k) acc[k] = fmaf(s_acc[w][k][lane], f, acc[k]);
#pragma unroll
            for (int k = 0; k < EK; ++k) acck[k] = fmaf(s_acck[w][k][lane], f, acck[k]);
        }
    }

    const size_t row = (size_t)b * a.cap + base + jb;
    // ---- main entry -> FP4 codes + one scale byte per group ----
    static_assert(E <= 16, "a lane's channels lie inside one 16-element group");
    float e[E];
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        e[k] = acc[k] / den;
        amax = fmaxf(amax, fabsf(e[k]));
    }
    uint32_t packed[E / 2 > 0 ? E / 2 : 1];
    if (a.scale_e4m3) {
        // a 16-element group spans 16/E lanes; s = E4M3(amax / 6), RNE, saturating
#pragma unroll
        for (int o = 1; o < 16 / E; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(__fdiv_rn(amax, 6.0f), __NV_SATFINITE, __NV_E4M3);
        const float sv = __half2float(__half(__nv_cvt_fp8_to_halfraw(sb, __NV_E4M3)));
        const float sc = sv > 0.f ? sv : INFINITY;
        const float th[7] = {0.25f * sc, 0.75f * sc, 1.25f * sc, 1.75f * sc, 2.5f * sc, 3.5f * sc, 5.0f * sc};
#pragma unroll
        for (int k = 0; k < E; k += 2) packed[k / 2] = e2m1_code_th(e[k], th) | (e2m1_code_th(e[k + 1], th) << 4);
        if (lane % (16 / E) == 0) a.scale[row * (a.D / 16) + lane / (16 / E)] = (uint8_t)sb;
    } else {
        // a 32-element group spans 32/E lanes
#pragma unroll
        for (int o = 1; o < 32 / E; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        // X = floor(log2 amax) - 2 from the exponent field, clamped to >= -127
        // (zero and subnormal amax land on the clamp); byte = X + 127.
        const int expbits = (int)((__float_as_uint(amax) >> 23) & 0xFF);
        const int sbyte = max(expbits - 2, 0);
        const float inv = __uint_as_float((uint32_t)(254 - sbyte) << 23);  // 2^-X, X = sbyte-127
#pragma unroll
        for (int k = 0; k < E; k += 2)
            packed[k / 2] = e2m1_code(e[k] * inv) | (e2m1_code(e[k + 1] * inv) << 4);
        if (lane % (32 / E) == 0) a.scale[row * (a.D / 32) + lane / (32 / E)] = (uint8_t)sbyte;
    }
    uint8_t *dst = a.fp4 + row * (a.D / 2) + lane * (E / 2);
    if constexpr (E == 16) {
        uint2 w;
        w.x = packed[0] | (packed[1] << 8) | (packed[2] << 16) | (packed[3] << 24);
        w.y = packed[4] | (packed[5] << 8) | (packed[6] << 16) | (packed[7] << 24);
        *reinterpret_cast<uint2 *>(dst) = w;
    } else if constexpr (E == 8) {
        *reinterpret_cast<uint32_t *>(dst) = packed[0] | (packed[1] << 8) | (packed[2] << 16) | (packed[3] << 24);
    } else if constexpr (E == 4) {
        *reinterpret_cast<uint16_t *>(dst) = (uint16_t)(packed[0] | (packed[1] << 8));
    } else {
        dst[0] = (uint8_t)packed[0];
    }

    // ---- pooled indexer key -> bf16, e4m3 or MXFP4 ----
    if constexpr (EI > 0) {
        if (a.idx_mxfp4) {
            // the main KV's E8M0 rule per 32 channels; a group spans 32/EI lanes
            float kv[EI];
            float kmax = 0.f;
#pragma unroll
            for (int k = 0; k < EI; ++k) {
                kv[k] = acck[k] / den;
                kmax = fmaxf(kmax, fabsf(kv[k]));
            }
#pragma unroll
            for (int o = 1; o < 32 / EI; o <<= 1) kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
            const int kbyte = max((int)((__float_as_uint(kmax) >> 23) & 0xFF) - 2, 0);
            const float kinv = __uint_as_float((uint32_t)(254 - kbyte) << 23);
            uint8_t *kd = a.idx_key + row * (a.dI / 2) + lane * (EI / 2);
#pragma unroll
            for (int k = 0; k < EI; k += 2)
                kd[k / 2] = (uint8_t)(e2m1_code(kv[k] * kinv) | (e2m1_code(kv[k + 1] * kinv) << 4));
            if (lane % (32 / EI) == 0) a.idx_key_scale[row * (a.dI / 32) + lane / (32 / EI)] = (uint8_t)kbyte;
        } else if (a.idx_e4m3) {
            uint8_t *kd = a.idx_key + row * a.dI + lane * EI;
#pragma unroll
            for (int k = 0; k < EI; ++k)
                kd[k] = (uint8_t)__nv_cvt_float_to_fp8(acck[k] / den, __NV_SATFINITE, __NV_E4M3);
        } else {
            __nv_bfloat16 *kd = reinterpret_cast<__nv_bfloat16 *>(a.idx_key + row * a.dI * 2) + lane * EI;
#pragma unroll
            for (int k = 0; k < EI; ++k) kd[k] = __float2bfloat16_rn(acck[k] / den);
        }
    }
}

// Advance n_blocks after the pooling kernel has read the old values; applies
// the same checks, so a rejected request is left untouched.
__global__ void commit_kernel(const int32_t *tok_offsets, int32_t *n_blocks, int batch, int m, int cap) {
    grid_dep_wait();
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
        const int count = tok_offsets[b + 1] - tok_offsets[b];
        if (count < 0 || count % m != 0) continue;
        if ((long long)n_blocks[b] + count / m > cap) continue;
        n_blocks[b] += count / m;
    }
}

// Warps of a block team: 16, or 8 when the team's combine buffers would not
// fit the 48 KB of static shared memory.
template <int E, int EI>
constexpr int team_warps() {
    return (E + (EI > 0 ? EI : 2)) * kWarp * 4 * 16 <= 40 * 1024 ? 16 : 8;
}

template <int E, int EI, int WPB>
cudaError_t launch_one(const CompressArgs &a, dim3 grid, cudaStream_t s) {
    constexpr int W = WPB == 1 ? 1 : team_warps<E, EI>();
    const dim3 block(W == 1 ? kWarpsPerCta * kWarp : W * kWarp);
    const size_t dyn = a.flat ? sizeof(int) * (size_t)(a.batch + 1) : 0;
    return launch_pdl(pool_quantize_kernel<E, EI, W>, grid, block, dyn, s, a);
}

template <int E, int WPB>
cudaError_t launch_ew(const CompressArgs &a, dim3 grid, cudaStream_t s) {
    switch (a.idx_key ? a.dI / 32 : 0) {
        case 0: return launch_one<E, 0, WPB>(a, grid, s);
        case 2: return launch_one<E, 2, WPB>(a, grid, s);
        case 4: return launch_one<E, 4, WPB>(a, grid, s);
        case 8: return launch_one<E, 8, WPB>(a, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

// m >= 32: a team of warps per block; otherwise four blocks per CTA, one warp each
template <int E>
cudaError_t launch_e(const CompressArgs &a, int max_blocks, int batch, cudaStream_t s) {
    // flat grid: max_blocks bounds the blocks of all requests together
    const int gy = a.flat ? 1 : batch;
    if (a.m >= 32) return launch_ew<E, 2>(a, dim3(max_blocks, gy), s);
    return launch_ew<E, 1>(a, dim3((max_blocks + kWarpsPerCta - 1) / kWarpsPerCta, gy), s);
}

}  // namespace

// Host launcher; arguments already validated by the C-ABI layer.
cudaError_t launch_compress(const csa_cache &c, const void *kv_tok, const void *idx_tok, const float *gate_w,
                            const int32_t *tok_offsets, int32_t n_tokens, cudaStream_t s) {
    CompressArgs a;
    a.kv_tok = static_cast<const __nv_bfloat16 *>(kv_tok);
    a.idx_tok = static_cast<const __nv_bfloat16 *>(idx_tok);
    a.gate_w = gate_w;
    a.tok_offsets = tok_offsets;
    a.n_blocks = c.n_blocks;
    a.fp4 = c.fp4;
    a.scale = c.scale;
    a.idx_key = static_cast<uint8_t *>(c.idx_key);
    a.status = c.status;
    a.m = c.block;
    a.cap = c.capacity;
    a.D = c.dim;
    a.dI = c.idx_key ? c.idx_dim : 0;
    a.idx_e4m3 = c.idx_dtype == CSA_IDX_E4M3;
    a.idx_mxfp4 = c.idx_dtype == CSA_IDX_MXFP4;
    a.idx_key_scale = c.idx_key_scale;
    a.scale_e4m3 = c.scale_fmt == CSA_SCALE_E4M3_16;
    a.batch = c.batch;
    a.flat = c.batch <= kFlatMaxBatch;
    const int max_blocks = (n_tokens + c.block - 1) / c.block;
    if (max_blocks > 0) {
        cudaError_t err;
        switch (c.dim / 32) {
            case 2: err = launch_e<2>(a, max_blocks, c.batch, s); break;
            case 4: err = launch_e<4>(a, max_blocks, c.batch, s); break;
            case 8: err = launch_e<8>(a, max_blocks, c.batch, s); break;
            case 16: err = launch_e<16>(a, max_blocks, c.batch, s); break;
            default: return cudaErrorInvalidValue;
        }
        if (err != cudaSuccess) return err;
    }
    return launch_pdl(commit_kernel, dim3((c.batch + 255) / 256), dim3(256), 0, s, tok_offsets, c.n_blocks, c.batch,
                      c.block, c.capacity);
}

}  // namespace csa
