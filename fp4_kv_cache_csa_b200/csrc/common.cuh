// common.cuh -- small device helpers shared by the libcsa kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/csa.h"

namespace csa {

constexpr int kWarp = 32;

// Programmatic dependent launch: a kernel launched with launch_pdl() may start
// while the previous kernel on the stream finishes; grid_dep_wait() blocks until
// that kernel has completed and its writes are visible, grid_dep_launch() lets
// the next kernel begin its launch early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch kern<<<grid, block, smem, s>>>(args...) with programmatic stream serialization.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

__device__ __forceinline__ void flag(int32_t *status, int32_t bits) {
    if (status) atomicOr(status, bits);
}

// Order-preserving map from float32 to uint32: a larger score gives a larger
// key. -0 is folded into +0 first, so the two compare equal.
__device__ __forceinline__ uint32_t ordered_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// E2M1 code of a scaled value s (|s| < 8), round to nearest with ties to the
// even code, saturating at 6; the sign bit is kept even when the magnitude
// rounds to zero. Thresholds are the midpoints between neighbouring
// magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6; "<=" sends a tie to the lower (even)
// code, "<" sends it to the upper (even) code.
__device__ __forceinline__ uint32_t e2m1_code(float s) {
    uint32_t sign = (__float_as_uint(s) >> 28) & 8u;
    float a = fabsf(s);
    uint32_t c = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
               : a <= 2.5f ? 4u : a < 3.5f ? 5u : a <= 5.0f ? 6u : 7u;
    return sign | c;
}

// E8M0 byte of a 32-element group with largest magnitude amax (X = floor(log2 amax) - 2,
// clamped to >= -127: zero and subnormal amax land on the clamp; byte = X + 127), and
// 2^-X as a float, the factor that maps the group onto E2M1's range.
__device__ __forceinline__ int e8m0_byte(float amax) {
    return max((int)((__float_as_uint(amax) >> 23) & 0xFF) - 2, 0);
}
__device__ __forceinline__ float e8m0_inverse(int byte) { return __uint_as_float((uint32_t)(254 - byte) << 23); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Index of the request that owns query i: the b with q_offsets[b] <= i < q_offsets[b+1]
// (binary search; -1 when i is outside [q_offsets[0], q_offsets[batch])).
__device__ __forceinline__ int request_of(const int32_t *q_offsets, int batch, int i) {
    if (i < q_offsets[0] || i >= q_offsets[batch]) return -1;
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (q_offsets[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Blocks visible to a query at absolute position pos: causal at block
// granularity and no more than the filled blocks.
__device__ __forceinline__ int visible_blocks(int pos, int m, int filled) {
    long long v = ((long long)pos + 1) / m;
    if (v > filled) v = filled;
    if (v < 0) v = 0;
    return (int)v;
}

// Inclusive prefix sum over the threads of a block (blockDim.x multiple of 32).
template <typename T>
__device__ T block_inclusive_scan(T v, T *smem /* >= 32 entries */) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) smem[warp] = v;
    __syncthreads();
    if (warp == 0) {
        T s = lane < nw ? smem[lane] : T(0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            T y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < nw) smem[lane] = s;
    }
    __syncthreads();
    if (warp > 0) v += smem[warp - 1];
    __syncthreads();
    return v;
}

}  // namespace csa
