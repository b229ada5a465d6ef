// noalloc.cu -- csa_index_topk_noalloc: indexer scoring + top-k with its scratch
// space in a fixed device array owned by the library, for callers that cannot
// allocate device memory themselves.
//
// Who needs it: code that runs where cudaMalloc is unavailable or unwelcome --
// a plugin or embedded runtime whose host framework owns every device
// allocation, a fixed-memory-budget deployment that must not grow its
// footprint per call, or a caller that cannot afford the device-wide
// synchronization an allocation may cause. Such a caller still owns and
// passes every input and output; only the scratch comes from here.
//
// The scratch is one file-scope __device__ array of kScratchBytes. Host code
// must not pass the array's symbol itself to a kernel (on the host that name
// is only a stand-in, not a device address), so the first call on each device
// looks up the device address once with cudaGetSymbolAddress and caches it.
// The computation is exactly csa_index_topk's, run on that scratch.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/csa.h"

namespace csa {
// csa_api.cu: the argument checks every indexer call makes, in the same order.
csa_status check_index_args(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                            int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                            const int32_t *sel_idx);
// indexer.cu: the least workspace csa_index_topk accepts (one chunk of queries).
size_t index_topk_min_workspace_bytes(const csa_cache &c, int Nq, int H_I);
}  // namespace csa

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB on every device that loads the library
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_index_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch[kMaxDevices] = {};

// Device address of g_index_scratch on the current device; looked up on the
// first call per device (with that device current) and cached.
csa_status scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_index_scratch) != cudaSuccess || !p) return CSA_ERR_CUDA;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return CSA_OK;
}

}  // namespace

extern "C" csa_status csa_index_topk_noalloc(const csa_cache *cache, const void *q_idx, const float *w,
                                             int32_t n_queries, int32_t idx_heads, const int32_t *q_offsets,
                                             const int32_t *q_pos, int32_t topk, int32_t *sel_idx,
                                             csa_stream_t stream) {
    // the same argument errors as csa_index_topk, reported first; then the size check
    const csa_status arg = csa::check_index_args(cache, q_idx, w, n_queries, idx_heads, q_offsets, q_pos, topk,
                                                 sel_idx);
    if (arg != CSA_OK) return arg;
    // not even one chunk of queries fits the fixed scratch (larger calls run in chunks)
    if (csa::index_topk_min_workspace_bytes(*cache, n_queries, idx_heads) > kScratchBytes) return CSA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const csa_status st = scratch_address(&scratch);
    if (st != CSA_OK) return st;
    return csa_index_topk(cache, q_idx, w, n_queries, idx_heads, q_offsets, q_pos, topk, sel_idx, scratch,
                          kScratchBytes, stream);
}
