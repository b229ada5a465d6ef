// csa_api.cu -- the C ABI declared in include/csa.h: host-side argument checks,
// workspace sizing and kernel dispatch. Nothing here allocates memory; every
// call only enqueues work on the caller's stream.
#include <cstdint>
#include <cstdio>

#include "common.cuh"

namespace csa {
cudaError_t launch_compress(const csa_cache &c, const void *kv_tok, const void *idx_tok, const float *gate_w,
                            const int32_t *tok_offsets, int32_t n_tokens, cudaStream_t s);
size_t index_topk_workspace_bytes(const csa_cache &c, int Nq);
size_t index_topk_min_workspace_bytes(const csa_cache &c, int Nq, int H_I);
cudaError_t launch_index_topk(const csa_cache &c, const void *q_idx, const float *w, int Nq, int H_I,
                              const int32_t *q_offsets, const int32_t *q_pos, int topk, int32_t *sel_idx,
                              void *workspace, size_t workspace_bytes, int num_sms, cudaStream_t s);
size_t index_pool_workspace_bytes(int Nq, int cap, int G, int P);
cudaError_t launch_index_topk_pool(const csa_cache &c, const void *q_idx, const float *w, int Nq, int H_I,
                                   const int32_t *q_offsets, const int32_t *q_pos, int topk, int32_t *sel_idx,
                                   int pool_shift, int P, int32_t *pool_blk, void *workspace, int num_sms,
                                   cudaStream_t s);
size_t index_reindex_workspace_bytes(int Nq, int G, int P);
cudaError_t launch_index_topk_reindex(const csa_cache &c, const void *q_idx, const float *w, int Nq, int H_I,
                                      const int32_t *q_offsets, const int32_t *q_pos, int topk, int32_t *sel_idx,
                                      int pool_shift, int P, const int32_t *pool_blk, void *workspace, int num_sms,
                                      cudaStream_t s, int layers);
size_t attend_workspace_bytes(int Nq, int D, int num_ctas);
cudaError_t launch_mxf4_probe(int iters, int32_t *status, int num_sms, cudaStream_t s);
cudaError_t launch_attend(const csa_cache &c, const void *q, int Nq, int H, const int32_t *q_offsets,
                          const int32_t *q_pos, const int32_t *sel_idx, int topk, const void *win_kv,
                          const int64_t *win_start, const int32_t *win_len, int max_win, float softmax_scale,
                          float *out, float *lse, void *workspace, int num_ctas, cudaStream_t s);
}  // namespace csa

namespace {

constexpr int kMaxCapacity = 1 << 19;  // the top-k select keeps two bitmaps of this many bits in shared memory
constexpr int kMaxTopk = 4096;
constexpr int kMaxReindexLayers = 16;  // Reindex layers in one csa_index_topk_reindex_layers call

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Number of SMs of the current device (the attention and scan grids are sized from it).
int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

csa_status check_cache(const csa_cache *c) {
    if (!c || !c->fp4 || !c->scale || !c->n_blocks) return CSA_ERR_NULL;
    if (c->batch < 1 || c->capacity < 1 || c->block < 1 || c->block > 128) return CSA_ERR_SHAPE;
    if (c->dim < 64 || c->dim % 32 != 0) return CSA_ERR_SHAPE;
    if (c->capacity > kMaxCapacity) return CSA_ERR_UNSUPPORTED;
    if (c->scale_fmt != CSA_SCALE_E8M0_32 && c->scale_fmt != CSA_SCALE_E4M3_16) return CSA_ERR_SHAPE;
    if (!aligned(c->fp4, 16) || !aligned(c->scale, 16) || !aligned(c->n_blocks, 4)) return CSA_ERR_ALIGN;
    if (c->status && !aligned(c->status, 4)) return CSA_ERR_ALIGN;
    if (c->idx_key) {
        if (c->idx_dtype != CSA_IDX_BF16 && c->idx_dtype != CSA_IDX_E4M3 && c->idx_dtype != CSA_IDX_MXFP4)
            return CSA_ERR_SHAPE;
        if (c->idx_dim != 64 && c->idx_dim != 128 && c->idx_dim != 256) return CSA_ERR_UNSUPPORTED;
        if (!aligned(c->idx_key, 16)) return CSA_ERR_ALIGN;
        if (c->idx_dtype == CSA_IDX_MXFP4) {
            if (!c->idx_key_scale) return CSA_ERR_NULL;
            if (!aligned(c->idx_key_scale, 4)) return CSA_ERR_ALIGN;
        }
    }
    return CSA_OK;
}

csa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }

}  // namespace

// Argument checks of every indexer call (csa_index_topk, its pool and Reindex
// forms, and csa_index_topk_noalloc in noalloc.cu), in the order the status
// codes are reported; the workspace is checked by each caller afterwards.
namespace csa {
csa_status check_index_args(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                            int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                            const int32_t *sel_idx) {
    csa_status st = check_cache(cache);
    if (st != CSA_OK) return st;
    if (!cache->idx_key || !q_idx || !w || !q_offsets || !q_pos || !sel_idx) return CSA_ERR_NULL;
    if (n_queries < 1 || idx_heads < 1 || topk < 1) return CSA_ERR_SHAPE;
    if (idx_heads > 8 || topk > kMaxTopk) return CSA_ERR_UNSUPPORTED;
    if (cache->idx_dtype == CSA_IDX_MXFP4 && idx_heads > 4) return CSA_ERR_UNSUPPORTED;
    if (!aligned(q_idx, 16) || !aligned(w, 4) || !aligned(q_offsets, 4) || !aligned(q_pos, 4) ||
        !aligned(sel_idx, 4))
        return CSA_ERR_ALIGN;
    return CSA_OK;
}
}  // namespace csa

extern "C" {

const char *csa_status_string(int32_t status) {
    switch (status) {
        case CSA_OK: return "ok";
        case CSA_ERR_NULL: return "required pointer is NULL";
        case CSA_ERR_SHAPE: return "size out of range or inconsistent";
        case CSA_ERR_ALIGN: return "pointer not aligned";
        case CSA_ERR_UNSUPPORTED: return "configuration not implemented";
        case CSA_ERR_WORKSPACE: return "workspace missing or too small";
        case CSA_ERR_CUDA: return "CUDA runtime error";
        default: return "unknown status";
    }
}

int32_t csa_version(void) { return 103; }

csa_status csa_compress_quantize(const csa_cache *cache, const void *kv_tok, const void *idx_tok, const float *gate_w,
                                 const int32_t *tok_offsets, int32_t n_tokens, csa_stream_t stream) {
    csa_status st = check_cache(cache);
    if (st != CSA_OK) return st;
    if (!kv_tok || !gate_w || !tok_offsets) return CSA_ERR_NULL;
    if ((cache->idx_key != nullptr) != (idx_tok != nullptr)) return CSA_ERR_NULL;
    if (n_tokens < 0) return CSA_ERR_SHAPE;
    if (cache->dim != 64 && cache->dim != 128 && cache->dim != 256 && cache->dim != 512) return CSA_ERR_UNSUPPORTED;
    if (!aligned(kv_tok, 16) || !aligned(gate_w, 16) || !aligned(tok_offsets, 4)) return CSA_ERR_ALIGN;
    if (idx_tok && !aligned(idx_tok, 16)) return CSA_ERR_ALIGN;
    return from_cuda(csa::launch_compress(*cache, kv_tok, idx_tok, gate_w, tok_offsets, n_tokens,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

size_t csa_index_topk_workspace(const csa_cache *cache, int32_t n_queries, int32_t topk) {
    if (!cache || n_queries < 1 || topk < 1 || cache->capacity < 1 || cache->capacity > kMaxCapacity) return 0;
    return csa::index_topk_workspace_bytes(*cache, n_queries);
}

csa_status csa_index_topk(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                          int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                          int32_t *sel_idx, void *workspace, size_t workspace_bytes, csa_stream_t stream) {
    const csa_status st = csa::check_index_args(cache, q_idx, w, n_queries, idx_heads, q_offsets, q_pos, topk,
                                                 sel_idx);
    if (st != CSA_OK) return st;
    // one chunk of queries must fit; a larger workspace runs more queries per chunk
    const size_t need = csa::index_topk_min_workspace_bytes(*cache, n_queries, idx_heads);
    if (!workspace || workspace_bytes < need) return CSA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return CSA_ERR_ALIGN;
    const int sms = num_sms();
    if (sms <= 0) return CSA_ERR_CUDA;
    return from_cuda(csa::launch_index_topk(*cache, q_idx, w, n_queries, idx_heads, q_offsets, q_pos, topk, sel_idx,
                                            workspace, workspace_bytes, sms, reinterpret_cast<cudaStream_t>(stream)));
}

// log2 of a pool block size (1, 2, 4, ... 32 entries), or -1
static int pool_shift_of(int32_t g) {
    for (int k = 0; k <= 5; ++k)
        if (g == (1 << k)) return k;
    return -1;
}


static bool pool_sizes_ok(int32_t pool_group, int32_t pool_blocks) {
    return pool_shift_of(pool_group) >= 0 && pool_blocks >= 1 && pool_blocks <= kMaxTopk &&
           (long long)pool_group * pool_blocks <= kMaxCapacity;
}

size_t csa_index_pool_workspace(const csa_cache *cache, int32_t n_queries, int32_t topk, int32_t pool_group,
                                int32_t pool_blocks) {
    if (!cache || n_queries < 1 || topk < 1 || cache->capacity < 1 || cache->capacity > kMaxCapacity ||
        !pool_sizes_ok(pool_group, pool_blocks))
        return 0;
    return csa::index_pool_workspace_bytes(n_queries, cache->capacity, pool_group, pool_blocks);
}

csa_status csa_index_topk_pool(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                               int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                               int32_t *sel_idx, int32_t pool_group, int32_t pool_blocks, int32_t *pool_blk,
                               void *workspace, size_t workspace_bytes, csa_stream_t stream) {
    csa_status st = csa::check_index_args(cache, q_idx, w, n_queries, idx_heads, q_offsets, q_pos, topk, sel_idx);
    if (st != CSA_OK) return st;
    if (!pool_blk) return CSA_ERR_NULL;
    if (pool_shift_of(pool_group) < 0 || pool_blocks < 1) return CSA_ERR_SHAPE;
    if (!pool_sizes_ok(pool_group, pool_blocks)) return CSA_ERR_UNSUPPORTED;
    if (!aligned(pool_blk, 4)) return CSA_ERR_ALIGN;
    const size_t need = csa_index_pool_workspace(cache, n_queries, topk, pool_group, pool_blocks);
    if (!workspace || workspace_bytes < need) return CSA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return CSA_ERR_ALIGN;
    const int sms = num_sms();
    if (sms <= 0) return CSA_ERR_CUDA;
    return from_cuda(csa::launch_index_topk_pool(*cache, q_idx, w, n_queries, idx_heads, q_offsets, q_pos, topk,
                                                 sel_idx, pool_shift_of(pool_group), pool_blocks, pool_blk, workspace,
                                                 sms, reinterpret_cast<cudaStream_t>(stream)));
}

size_t csa_index_reindex_layers_workspace(const csa_cache *cache, int32_t n_queries, int32_t n_layers,
                                          int32_t pool_group, int32_t pool_blocks) {
    if (!cache || n_queries < 1 || n_layers < 1 || n_layers > kMaxReindexLayers ||
        !pool_sizes_ok(pool_group, pool_blocks) || (long long)n_queries * n_layers > (1 << 30))
        return 0;
    return csa::index_reindex_workspace_bytes(n_queries * n_layers, pool_group, pool_blocks);
}

size_t csa_index_reindex_workspace(const csa_cache *cache, int32_t n_queries, int32_t pool_group,
                                   int32_t pool_blocks) {
    return csa_index_reindex_layers_workspace(cache, n_queries, 1, pool_group, pool_blocks);
}

csa_status csa_index_topk_reindex_layers(const csa_cache *cache, const void *q_idx, const float *w,
                                         int32_t n_queries, int32_t n_layers, int32_t idx_heads,
                                         const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                                         int32_t *sel_idx, int32_t pool_group, int32_t pool_blocks,
                                         const int32_t *pool_blk, void *workspace, size_t workspace_bytes,
                                         csa_stream_t stream) {
    csa_status st = csa::check_index_args(cache, q_idx, w, n_queries, idx_heads, q_offsets, q_pos, topk, sel_idx);
    if (st != CSA_OK) return st;
    if (!pool_blk) return CSA_ERR_NULL;
    if (n_layers < 1 || pool_shift_of(pool_group) < 0 || pool_blocks < 1) return CSA_ERR_SHAPE;
    if (n_layers > kMaxReindexLayers || !pool_sizes_ok(pool_group, pool_blocks)) return CSA_ERR_UNSUPPORTED;
    if (!aligned(pool_blk, 4)) return CSA_ERR_ALIGN;
    const size_t need = csa_index_reindex_layers_workspace(cache, n_queries, n_layers, pool_group, pool_blocks);
    if (!workspace || workspace_bytes < need) return CSA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return CSA_ERR_ALIGN;
    const int sms = num_sms();
    if (sms <= 0) return CSA_ERR_CUDA;
    return from_cuda(csa::launch_index_topk_reindex(*cache, q_idx, w, n_queries, idx_heads, q_offsets, q_pos, topk,
                                                    sel_idx, pool_shift_of(pool_group), pool_blocks, pool_blk,
                                                    workspace, sms, reinterpret_cast<cudaStream_t>(stream),
                                                    n_layers));
}

csa_status csa_index_topk_reindex(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                                  int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                                  int32_t *sel_idx, int32_t pool_group, int32_t pool_blocks,
                                  const int32_t *pool_blk, void *workspace, size_t workspace_bytes,
                                  csa_stream_t stream) {
    return csa_index_topk_reindex_layers(cache, q_idx, w, n_queries, 1, idx_heads, q_offsets, q_pos, topk, sel_idx,
                                         pool_group, pool_blocks, pool_blk, workspace, workspace_bytes, stream);
}

size_t csa_attend_workspace(const csa_cache *cache, int32_t n_queries, int32_t heads) {
    if (!cache || n_queries < 1 || heads < 1 || (cache->dim != 128 && cache->dim != 512)) return 0;
    const int sms = num_sms();
    if (sms <= 0) return 0;
    return csa::attend_workspace_bytes(n_queries, cache->dim, sms);
}

static csa_status check_attend(const csa_cache *cache, const void *q, int32_t n_queries, int32_t heads,
                               const int32_t *q_offsets, const void *win_kv, const int64_t *win_start,
                               const int32_t *win_len, int32_t max_win, float *out, float *lse, void *workspace,
                               size_t workspace_bytes) {
    csa_status st = check_cache(cache);
    if (st != CSA_OK) return st;
    if (!q || !q_offsets || !out) return CSA_ERR_NULL;
    const bool any_win = win_kv || win_start || win_len;
    if (any_win && !(win_kv && win_start && win_len)) return CSA_ERR_NULL;
    if (n_queries < 1 || heads < 1 || max_win < 0) return CSA_ERR_SHAPE;
    if (heads > 64 || (cache->dim != 128 && cache->dim != 512)) return CSA_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(q_offsets, 4) || !aligned(out, 16)) return CSA_ERR_ALIGN;
    if (lse && !aligned(lse, 4)) return CSA_ERR_ALIGN;
    if (any_win && (!aligned(win_kv, 16) || !aligned(win_start, 8) || !aligned(win_len, 4))) return CSA_ERR_ALIGN;
    const size_t need = csa_attend_workspace(cache, n_queries, heads);
    if (need == 0) return CSA_ERR_CUDA;
    if (!workspace || workspace_bytes < need) return CSA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return CSA_ERR_ALIGN;
    return CSA_OK;
}

csa_status csa_decode_attend(const csa_cache *cache, const void *q, int32_t n_queries, int32_t heads,
                             const int32_t *q_offsets, const int32_t *sel_idx, int32_t topk, const void *win_kv,
                             const int64_t *win_start, const int32_t *win_len, int32_t max_win, float softmax_scale,
                             float *out, float *lse, void *workspace, size_t workspace_bytes, csa_stream_t stream) {
    csa_status st = check_attend(cache, q, n_queries, heads, q_offsets, win_kv, win_start, win_len, max_win, out, lse,
                                 workspace, workspace_bytes);
    if (st != CSA_OK) return st;
    if (!sel_idx) return CSA_ERR_NULL;
    if (topk < 1) return CSA_ERR_SHAPE;
    if (!aligned(sel_idx, 4)) return CSA_ERR_ALIGN;
    return from_cuda(csa::launch_attend(*cache, q, n_queries, heads, q_offsets, nullptr, sel_idx, topk, win_kv,
                                        win_start, win_len, max_win, softmax_scale, out, lse, workspace, num_sms(),
                                        reinterpret_cast<cudaStream_t>(stream)));
}

csa_status hca_decode_attend(const csa_cache *cache, const void *q, int32_t n_queries, int32_t heads,
                             const int32_t *q_offsets, const int32_t *q_pos, const void *win_kv,
                             const int64_t *win_start, const int32_t *win_len, int32_t max_win, float softmax_scale,
                             float *out, float *lse, void *workspace, size_t workspace_bytes, csa_stream_t stream) {
    csa_status st = check_attend(cache, q, n_queries, heads, q_offsets, win_kv, win_start, win_len, max_win, out, lse,
                                 workspace, workspace_bytes);
    if (st != CSA_OK) return st;
    if (!q_pos) return CSA_ERR_NULL;
    if (!aligned(q_pos, 4)) return CSA_ERR_ALIGN;
    return from_cuda(csa::launch_attend(*cache, q, n_queries, heads, q_offsets, q_pos, nullptr, 0, win_kv, win_start,
                                        win_len, max_win, softmax_scale, out, lse, workspace, num_sms(),
                                        reinterpret_cast<cudaStream_t>(stream)));
}

csa_status csa_read_device_status(const csa_cache *cache, csa_stream_t stream, int32_t *out_flags) {
    if (!cache || !cache->status || !out_flags) return CSA_ERR_NULL;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return CSA_ERR_CUDA;
    int32_t v = 0, zero = 0;
    if (cudaMemcpy(&v, cache->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return CSA_ERR_CUDA;
    if (cudaMemcpy(cache->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return CSA_ERR_CUDA;
    *out_flags = v;
    return CSA_OK;
}

csa_status csa_probe_mxf4_mma(int32_t iters, int32_t *status, csa_stream_t stream, int64_t *flops) {
    if (!status || !flops) return CSA_ERR_NULL;
    if (iters < 1) return CSA_ERR_SHAPE;
    if (!aligned(status, 4)) return CSA_ERR_ALIGN;
    const int sms = num_sms();
    if (sms <= 0) return CSA_ERR_CUDA;
    *flops = (int64_t)sms * iters * 2 * 128 * 256 * 128;
    return from_cuda(csa::launch_mxf4_probe(iters, status, sms, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
