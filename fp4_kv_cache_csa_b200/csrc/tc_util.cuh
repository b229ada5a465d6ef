// tc_util.cuh -- inline-PTX helpers for the sm_100a kernels that use the
// tensor memory and the fifth-generation tensor cores: shared-memory matrix
// and instruction descriptors, tcgen05.mma / commit / ld / st, mbarriers with
// bounded waits, bulk copies, cp.async, and the two-CTA cluster primitives.
// Internal to the library (each translation unit gets its own copies).
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace csa {

namespace {

// Bounded mbarrier waits: a wait that runs out makes the kernel flag
// CSA_DEV_TIMEOUT and leave. A test build of the library shortens the limit
// (-DCSA_WAIT_CYCLES=...) so that the first wait of a call runs out; the waits
// a kernel makes for its own copies and MMAs before it exits always use the
// long limit, so that nothing it started is still running when it leaves.
#ifndef CSA_WAIT_CYCLES
#define CSA_WAIT_CYCLES 2000000000LL
#endif
constexpr long long kWaitCycles = CSA_WAIT_CYCLES;  // ~1 s at the shipped value
constexpr long long kDrainCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    // tcgen05 shared-memory matrix descriptor: start >> 4, LBO >> 4, SBO >> 4,
    // version 1 (bits 46-47), 128-byte swizzle (layout type 2, bits 61-63).
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: D f32 (bits 4-5 = 1), A/B f16 (0),
// A/B major (bits 15/16), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// The same with bf16 A and B (formats 1 in bits 7-9 and 10-12), both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return idesc_f16(M, N, false, false) | (1u << 7) | (1u << 10);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

// Wait for the phase with this parity to complete; gives up after `limit` cycles.
__device__ __forceinline__ bool mbar_wait_for(uint32_t mbar, uint32_t parity, long long limit) {
    const long long t0 = clock64();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// Wait for the phase with this parity to complete; gives up after kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
    const long long t0 = clock64();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}

// Bulk copy (no tensor map, no multicast) of `bytes` from global memory to this
// CTA's shared memory, completing on mbar's transaction count.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

// Bulk copy of `bytes` from this CTA's shared memory to global memory (one
// bulk-async group per call); bulk_wait_read() returns once every issued
// group has finished reading shared memory, bulk_wait_all() once it has
// also written global memory.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n\t"
                 "cp.async.bulk.commit_group;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

#define CSA_LD16(base, r)                                                                                    \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];" \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), \
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),       \
                   "=r"(r[15])                                                                              \
                 : "r"(base))
#define CSA_ST16(base, r)                                                                                     \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" \
                 ::"r"(base), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), \
                   "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])     \
                 : "memory")

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[16];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        CSA_LD16(taddr + 16 * q, r);
#pragma unroll
        for (int k = 0; k < 16; ++k) v[16 * q + k] = __uint_as_float(r[k]);
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    uint32_t r[16];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int k = 0; k < 16; ++k) r[k] = __float_as_uint(v[16 * q + k]);
        CSA_ST16(taddr + 16 * q, r);
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    CSA_LD16(taddr, r);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[k]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    uint32_t r[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) r[k] = __float_as_uint(v[k]);
    CSA_ST16(taddr, r);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Butterfly transpose-reduction of N values per lane (N a power of two <= 32):
// afterwards v[0] of lane L holds the reduction over all 32 lanes of value L % N.
template <int N, bool MAX>
__device__ __forceinline__ void transpose_reduce(float (&v)[N]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = N / 2; half >= 1; half >>= 1) {
        const bool hi = (lane & half) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = hi ? v[k] : v[k + half];
            const float keep = hi ? v[k + half] : v[k];
            const float got = __shfl_xor_sync(0xffffffffu, send, half);
            v[k] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
#pragma unroll
    for (int off = N; off < 32; off <<= 1) {
        const float got = __shfl_xor_sync(0xffffffffu, v[0], off);
        v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
    }
}

// Butterfly transpose-reduction: 32 values per lane -> lane L ends with the
// reduction over all 32 lanes of value L (in v[0]).
template <bool MAX>
__device__ __forceinline__ void transpose_reduce32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = 16; half >= 1; half >>= 1) {
        const bool hi = (lane & half) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = hi ? v[k] : v[k + half];
            const float keep = hi ? v[k + half] : v[k];
            const float got = __shfl_xor_sync(0xffffffffu, send, half);
            v[k] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// ---- two-CTA clusters: distributed shared memory and cluster-scope barriers
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Bulk copy (no multicast) of `bytes` from this CTA's shared memory to another
// CTA's shared memory (dst and mbar are shared::cluster addresses of that CTA),
// completing on that CTA's barrier by transaction bytes.
__device__ __forceinline__ void bulk_s2peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     dst),
                 "r"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

// Arrive on a barrier of another CTA of the cluster, releasing this thread's
// earlier writes (to any CTA's shared memory) at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Bounded wait that also gives up once *abort is set (by another warp of the
// CTA that gave up). CLUSTER: acquire at cluster scope, for barriers that
// another CTA's threads arrive on after writing into this CTA's memory.
template <bool CLUSTER>
__device__ __forceinline__ bool mbar_wait_ab(uint32_t mbar, uint32_t parity, const volatile int *abort) {
    const long long t0 = clock64();
    while (true) {
        uint32_t done;
        if constexpr (CLUSTER) {
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}\n"
                : "=r"(done)
                : "r"(mbar), "r"(parity)
                : "memory");
        } else {
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}\n"
                : "=r"(done)
                : "r"(mbar), "r"(parity)
                : "memory");
        }
        if (done) return true;
        if (*abort) return false;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

// Barrier over all threads of both CTAs of the cluster (every thread calls it).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Named barrier 1 over the first N threads of the CTA (plain and with an OR vote).
template <int N>
__device__ __forceinline__ void bar_sync_n() {
    asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ bool bar_or_n(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(N)
        : "memory");
    return r != 0;
}

}  // namespace

}  // namespace csa
