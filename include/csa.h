/*
 * csa.h -- C ABI of libcsa: compressed sparse attention (CSA), heavily
 * compressed attention (HCA) and the uncompressed sliding window over a KV cache
 * stored as MXFP4, for NVIDIA B200 (sm_100a).
 *
 * What the calls compute (page title and section):
 *   "Frontier Architecture Decoding Notes (4): DeepSeek V4", section 1:
 *     CSA compresses the KV of every 4 tokens into one entry and attends to the
 *     top-k entries chosen per query; HCA compresses up to 128x and attends to
 *     every entry; the most recent 128 tokens are attended uncompressed.
 *   DeepSeek-V4.1-Flash podcast transcript, cue 12: indexer keys come from the
 *     main KV; an indexer query scores them and the top-k are attended.
 *   Same transcript, cue 16: the main KV is stored as MXFP4 (E2M1 elements
 *     with a shared block scale) and dequantized right before attention.
 * Readings where the pages are silent (the library's documented assumptions):
 *   pooling is a softmax-gated weighted sum of the m tokens with one scalar
 *   gate logit per token, g_t = <kv_t, w_g>; indexer score
 *   s_j = sum_h w_h * ReLU(<q_idx_h, k_j>); top-k ties go to the lower block
 *   index; one joint softmax covers the selected entries and the window;
 *   MXFP4 = E2M1 elements with one E8M0 scale per 32 elements (OCP MX v1.0);
 *   a cache may instead hold one E4M3 scale per 16 elements (cue 16's own
 *   wording), selected by csa_cache.scale_fmt.
 *
 * Conventions for every call:
 *   - Pointers inside csa_cache and every tensor argument are DEVICE pointers,
 *     owned by the caller. The library allocates no memory. Scratch space is
 *     the caller's `workspace`, and the calls keep no state between them --
 *     except csa_index_topk_noalloc, which uses a fixed scratch array that the
 *     library holds on every device that loads it, and caches that array's
 *     device address per device after its first call there.
 *   - Every call checks its arguments on the host first. On an argument error
 *     it returns the error code and launches nothing.
 *   - Otherwise it enqueues its kernels on `stream` and returns CSA_OK without
 *     synchronizing; a launch failure returns CSA_ERR_CUDA.
 *   - Conditions only the device can see (a token count that is not a
 *     multiple of m, a cache overflow, an out-of-range selected index or
 *     window) set bits in cache->status (CSA_DEV_* below) when that pointer is
 *     not NULL; the offending item is skipped, never trapped. Read the word
 *     with csa_read_device_status() after the work has completed.
 *   - bf16 means IEEE binary32 truncated to its upper 16 bits; e4m3 is OCP FP8
 *     E4M3 ("fn": no infinities, max 448).
 *   - All tensors are dense and row-major; every pointer must be 16-byte aligned.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *csa_stream_t; /* same type as cudaStream_t; NULL = legacy default stream */

typedef enum {
    CSA_OK = 0,
    CSA_ERR_NULL = 1,        /* a required pointer is NULL                      */
    CSA_ERR_SHAPE = 2,       /* a size is out of range or inconsistent          */
    CSA_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                */
    CSA_ERR_UNSUPPORTED = 4, /* valid request the library does not implement    */
    CSA_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than required         */
    CSA_ERR_CUDA = 6         /* a CUDA runtime call or kernel launch failed     */
} csa_status;

/* Storage of the pooled indexer keys:
 *   CSA_IDX_BF16   bf16;
 *   CSA_IDX_E4M3   OCP FP8 E4M3, round to nearest even, saturating, unscaled;
 *   CSA_IDX_MXFP4  MXFP4 like the main KV: E2M1 codes (two per byte, element
 *                  2i in the low nibble) in idx_key, one E8M0 scale byte per 32
 *                  channels in idx_key_scale. With these keys the indexer query
 *                  is quantized the same way (per 32 channels of each head)
 *                  before the scores, so every product is exact. */
typedef enum { CSA_IDX_BF16 = 0, CSA_IDX_E4M3 = 1, CSA_IDX_MXFP4 = 2 } csa_idx_dtype;

/* Scale format of the FP4 main KV (E2M1 elements in both):
 *   CSA_SCALE_E8M0_32  one E8M0 byte per 32 elements, value 2^(byte - 127)
 *                      (OCP MX v1.0 MXFP4);
 *   CSA_SCALE_E4M3_16  one E4M3 byte per 16 elements, no second-level scale
 *                      (the format the DeepSeek-V4.1-Flash podcast transcript
 *                      names in cue 16). */
typedef enum { CSA_SCALE_E8M0_32 = 0, CSA_SCALE_E4M3_16 = 1 } csa_scale_fmt;

/* Bits OR-ed into *cache->status by the kernels. */
#define CSA_DEV_TOKEN_COUNT 0x1  /* a request's new-token count is not a multiple of m: request skipped */
#define CSA_DEV_CAPACITY    0x2  /* appending would exceed capacity: request skipped                  */
#define CSA_DEV_BAD_INDEX   0x4  /* a selected block index >= the visible count: entry skipped          */
#define CSA_DEV_BAD_WINDOW  0x8  /* win_len outside [0, max_win]: clamped                              */
#define CSA_DEV_TIMEOUT     0x10 /* a bounded wait inside a kernel ran out: that tile's result is invalid */

/*
 * One compressed cache (one layer). Per request b and block j:
 *   fp4     [batch][capacity][dim/2]   two E2M1 codes per byte, element 2i in the
 *                                      low nibble, element 2i+1 in the high nibble
 *   scale   [batch][capacity][dim/32]  E8M0 bytes, value 2^(byte-127)  (CSA_SCALE_E8M0_32)
 *           [batch][capacity][dim/16]  E4M3 bytes                      (CSA_SCALE_E4M3_16)
 *   idx_key [batch][capacity][idx_dim] bf16 or e4m3 pooled indexer keys; NULL for
 *                                      a cache that is only attended densely (HCA)
 *           [batch][capacity][idx_dim/2]  MXFP4 codes of the keys (CSA_IDX_MXFP4)
 *   idx_key_scale [batch][capacity][idx_dim/32]  their E8M0 scale bytes
 *                                      (CSA_IDX_MXFP4 only, else NULL; 4-byte aligned)
 *   n_blocks [batch]                   filled blocks per request; advanced by
 *                                      csa_compress_quantize
 *   status                             one int32 of CSA_DEV_* bits, or NULL
 * An element's value is E2M1(code) * 2^(scale - 127) for E8M0 scales and
 * E2M1(code) * E4M3(scale) for E4M3 scales (the scale byte of its group).
 * scale_fmt (ABI 101) and idx_key_scale (ABI 103) were appended, so the
 * offsets of the other fields are those of ABI version 100.
 */
typedef struct {
    int32_t batch;     /* requests, >= 1                                  */
    int32_t dim;       /* D (K = V latent width): 64, 128, 256 or 512 for compression, 128 or 512 for attention */
    int32_t block;     /* m, tokens pooled per entry, 1..128              */
    int32_t capacity;  /* blocks per request, 1 .. 2^19                   */
    uint8_t *fp4;
    uint8_t *scale;
    void *idx_key;
    int32_t idx_dim;   /* d_I: 64, 128 or 256 (0 when idx_key is NULL)     */
    int32_t idx_dtype; /* csa_idx_dtype                                   */
    int32_t *n_blocks;
    int32_t *status;
    int32_t scale_fmt; /* csa_scale_fmt                                  */
    uint8_t *idx_key_scale; /* CSA_IDX_MXFP4 key scales, else NULL         */
} csa_cache;

/* Human-readable name of a csa_status value. Never NULL. */
const char *csa_status_string(int32_t status);

/* Library ABI version (major * 100 + minor). 101 added csa_cache.scale_fmt, 102 the pool and
 * Reindex calls, 103 the MXFP4 indexer keys (csa_cache.idx_key_scale). */
int32_t csa_version(void);

/*
 * Rows a1 + a2: gated block pooling and MXFP4 quantization.
 * For each request b the new tokens are rows tok_offsets[b] .. tok_offsets[b+1]-1
 * of kv_tok / idx_tok. Every m consecutive tokens become one block, appended at
 * block n_blocks[b], n_blocks[b]+1, ...; n_blocks[b] is then advanced.
 *   gate logit   g_t = sum_d kv_t[d] * gate_w[d]            (float32)
 *   weights      a = softmax over the block's m logits
 *   main entry   e[d] = sum_t a_t kv_t[d], stored as FP4 in the cache's scale format:
 *                E8M0/32: per 32 elements X = floor(log2(max|e|)) - 2 clamped to
 *                [-127,127] (X = -127 for an all-zero group), code = E2M1
 *                round-to-nearest-even of e * 2^-X saturated to +-6;
 *                E4M3/16: per 16 elements s = E4M3 round-to-nearest-even of
 *                max|e| / 6 saturated to 448, code = E2M1 round-to-nearest-even
 *                of e / s saturated to +-6 (zero magnitude when s = 0);
 *                in both the sign is kept (a negative value that rounds to
 *                zero is code 0x8)
 *   indexer key  k[c] = sum_t a_t idx_t[c], stored as bf16 (RNE), e4m3 (RNE,
 *                saturated to +-448) or MXFP4 (the E8M0/32 rule above, codes in
 *                idx_key, scales in idx_key_scale) per cache->idx_dtype
 * Arguments:
 *   kv_tok      bf16 [n_tokens][dim]
 *   idx_tok     bf16 [n_tokens][idx_dim]; required iff cache->idx_key != NULL
 *   gate_w      float32 [dim]
 *   tok_offsets int32 [batch+1] device, non-decreasing, tok_offsets[batch] <= n_tokens
 *   n_tokens    rows of kv_tok (host value; bounds the launch)
 * Device checks: a count that is not a multiple of m sets CSA_DEV_TOKEN_COUNT,
 * an append beyond capacity sets CSA_DEV_CAPACITY; that request is left untouched.
 */
csa_status csa_compress_quantize(const csa_cache *cache, const void *kv_tok, const void *idx_tok,
                                 const float *gate_w, const int32_t *tok_offsets, int32_t n_tokens,
                                 csa_stream_t stream);

/*
 * Bytes of workspace to give csa_index_topk for these sizes (0 on bad sizes):
 * the workspace of all n_queries queries when that stays under 768 MiB, else
 * of the most queries that do, and the call then runs its queries in chunks
 * that fit. When the key format has a GEMM kernel (bf16 keys of 64, 128
 * or 256 channels, MXFP4 keys of 128) and the call brings 16 or more queries
 * per request, a chunk holds at least 4736 queries (one wave of query tiles
 * on the 148 SMs), above 768 MiB if it must.
 */
size_t csa_index_topk_workspace(const csa_cache *cache, int32_t n_queries, int32_t topk);

/*
 * Rows a3 + a4: indexer scoring and top-k block selection.
 * Query i belongs to the request b with q_offsets[b] <= i < q_offsets[b+1] and
 * sits at absolute token position q_pos[i]. It sees the blocks
 * j < n_vis = min(floor((q_pos[i]+1)/m), n_blocks[b]) (causal at block granularity).
 *   s_j = sum_{h < idx_heads} w[i][h] * max(0, sum_c q_idx[i][h][c] * key_j[c])
 * sel_idx[i] receives the min(topk, n_vis) blocks with the largest s_j (float32
 * comparison, -0 counted as +0, ties to the lower j) in ascending block order,
 * padded with -1.
 * Arguments:
 *   q_idx     bf16 [n_queries][idx_heads][idx_dim]
 *   w         float32 [n_queries][idx_heads]
 *   q_offsets int32 [batch+1] device; q_pos int32 [n_queries] device
 *   sel_idx   int32 [n_queries][topk] device, written
 *   idx_heads 1..8; topk 1..4096
 *   workspace 256-byte aligned, workspace_bytes of it usable. Any size from
 *             what one chunk of min(n_queries, 128) queries needs works
 *             (smaller: CSA_ERR_WORKSPACE); csa_index_topk_workspace() bytes
 *             always do. The call runs its queries in consecutive chunks of
 *             the most queries whose workspace fits (multiples of 128), all
 *             on the same stream; every query is scored and selected on its
 *             own, so the results do not depend on the chunks.
 * Calls that bring on average 16 or more queries per request (prefill) with
 * bf16 keys of 64, 128 or 256 channels and 1, 2, 4 or 8 indexer heads, or
 * with MXFP4 keys of 128 channels and 1 to 4 heads, compute the scores as one
 * tensor-core GEMM per request (TMA tensor maps over the key plane and q_idx,
 * which must then be 16-byte aligned, as every pointer here; MXFP4 keys on the
 * block-scaled MXFP4 MMA after the query is quantized); when the cache holds
 * at most 40960 blocks the top-k then runs one thread block per query over its
 * score row in shared memory. The results are the same as on the streaming
 * path; only the speed differs. (With MXFP4 keys this holds while the scale
 * products of a score's 32-channel blocks -- key scale times query scale --
 * lie less than 2^38 apart: the block-scaled MMA drops the products of a
 * block that far below the largest one.)
 */
csa_status csa_index_topk(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                          int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                          int32_t *sel_idx, void *workspace, size_t workspace_bytes, csa_stream_t stream);

/*
 * csa_index_topk without a caller workspace. The method has no counterpart to
 * this call: it exists for callers that cannot allocate device memory -- a
 * plugin or embedded runtime whose host framework owns every allocation, a
 * deployment with a fixed memory budget, or code that cannot afford the
 * device-wide synchronization an allocation may bring. The caller still
 * passes all inputs and outputs exactly as for csa_index_topk (same meaning,
 * same results); only the scratch space is the library's.
 *   - The scratch is one fixed 32 MiB array in device memory, held on every
 *     GPU that loads the library until the process exits. A call runs as
 *     csa_index_topk does with a 32 MiB workspace: in chunks of queries when
 *     all of them do not fit. Sizes where not even one chunk of 128 queries
 *     fits are rejected with CSA_ERR_WORKSPACE before anything is launched;
 *     the argument checks of csa_index_topk come first (same codes, same
 *     order).
 *   - The first call on each device looks up that array's device address
 *     (once, with the device current). Make that first call before any
 *     stream capture on the device.
 *   - Every call uses the same array; each call clears what must start at
 *     zero, so leftovers from the previous call do not matter. Calls that
 *     overlap on the GPU (other streams, or another host thread) race on the
 *     array: serialize them.
 *   - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 */
csa_status csa_index_topk_noalloc(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                                  int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                                  int32_t *sel_idx, csa_stream_t stream);

/*
 * Hierarchical indexer and CSA2 Reindex mode.
 * Source: DeepSeek-V4.1-Flash podcast transcript, cue 12 (three per-layer modes:
 * Full computes its own indexer scores and top-k; Reindex reuses the main KV and
 * indexer keys of an earlier Full layer but runs its own indexer query; Reuse
 * takes an earlier layer's top-k indices, i.e. calls csa_decode_attend with
 * them) and cue 14 (the first Full layer also keeps the highest-scoring blocks
 * of about eight positions, scored by their best position, as a candidate pool
 * of about sixteen thousand positions; Reindex layers search only that pool).
 *
 * csa_index_topk_pool: everything csa_index_topk does, plus the pool. The
 * visible blocks j < n_vis (as for csa_index_topk) are grouped into pool blocks
 * of pool_group consecutive blocks; pool block p scores max s_j over its
 * visible j; the min(pool_blocks, ceil(n_vis / pool_group)) pool blocks with
 * the largest score (ties to the lower p) are written ascending to
 * pool_blk[i][0 ..], padded with -1.
 *   pool_group  1, 2, 4, 8, 16 or 32 (8 in the transcript)
 *   pool_blocks 1 .. 4096 (about 2000 in the transcript); pool_group *
 *               pool_blocks <= 2^19
 *   pool_blk    int32 [n_queries][pool_blocks] device, written
 *   workspace   >= csa_index_pool_workspace(...) bytes, 256-byte aligned
 * Other arguments as for csa_index_topk.
 */
size_t csa_index_pool_workspace(const csa_cache *cache, int32_t n_queries, int32_t topk, int32_t pool_group,
                                int32_t pool_blocks);
csa_status csa_index_topk_pool(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                               int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                               int32_t *sel_idx, int32_t pool_group, int32_t pool_blocks, int32_t *pool_blk,
                               void *workspace, size_t workspace_bytes, csa_stream_t stream);

/*
 * csa_index_topk_reindex: a Reindex-mode layer's own indexer query (q_idx, w)
 * scored only against the blocks of its pool (as written by csa_index_topk_pool
 * for the same queries and cache): the candidates are the visible blocks
 * j < n_vis of pool blocks pool_blk[i][0 ..] (ascending, -1 padding at the end);
 * sel_idx[i] receives the min(topk, #candidates) with the largest s_j (ties to
 * the lower j), ascending, padded with -1. A pool block at or beyond n_vis, or
 * out of ascending order, ends the list there and sets CSA_DEV_BAD_INDEX.
 *   workspace >= csa_index_reindex_workspace(...) bytes, 256-byte aligned
 * The work per query is bounded by pool_group * pool_blocks, not by the context.
 */
size_t csa_index_reindex_workspace(const csa_cache *cache, int32_t n_queries, int32_t pool_group,
                                   int32_t pool_blocks);
csa_status csa_index_topk_reindex(const csa_cache *cache, const void *q_idx, const float *w, int32_t n_queries,
                                  int32_t idx_heads, const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                                  int32_t *sel_idx, int32_t pool_group, int32_t pool_blocks,
                                  const int32_t *pool_blk, void *workspace, size_t workspace_bytes,
                                  csa_stream_t stream);

/*
 * csa_index_topk_reindex_layers: n_layers Reindex-mode layers over the same pool
 * in one call (cue 12: every Reindex layer runs its own indexer query against
 * the shared keys of the earlier Full layer). For caller query i and layer l the
 * result is exactly csa_index_topk_reindex's for that layer's query and weights;
 * the layers of a query share its pool, its counts and its key reads (adjacent
 * in one pass, so the pool's keys come from HBM about once), and the call
 * launches the kernels of one Reindex call, not n_layers of them.
 *   q_idx    bf16 [n_queries][n_layers][idx_heads][idx_dim]
 *   w        float32 [n_queries][n_layers][idx_heads]
 *   sel_idx  int32 [n_queries][n_layers][topk] device, written
 *   n_layers 1 .. 16 (1 is csa_index_topk_reindex)
 *   workspace >= csa_index_reindex_layers_workspace(...) bytes, 256-byte aligned
 * q_offsets, q_pos and pool_blk are per caller query, as for csa_index_topk_reindex.
 */
size_t csa_index_reindex_layers_workspace(const csa_cache *cache, int32_t n_queries, int32_t n_layers,
                                          int32_t pool_group, int32_t pool_blocks);
csa_status csa_index_topk_reindex_layers(const csa_cache *cache, const void *q_idx, const float *w,
                                         int32_t n_queries, int32_t n_layers, int32_t idx_heads,
                                         const int32_t *q_offsets, const int32_t *q_pos, int32_t topk,
                                         int32_t *sel_idx, int32_t pool_group, int32_t pool_blocks,
                                         const int32_t *pool_blk, void *workspace, size_t workspace_bytes,
                                         csa_stream_t stream);

/* Bytes of workspace csa_decode_attend / hca_decode_attend need (0 on bad sizes). */
size_t csa_attend_workspace(const csa_cache *cache, int32_t n_queries, int32_t heads);

/*
 * Rows a5 + a6 + a8: CSA joint attention.
 * For query i and head h the entries are the dequantized blocks sel_idx[i][0..topk)
 * of request b (negative indices are padding and ignored) followed by the window
 * rows win_kv[win_start[i] + t], 0 <= t < win_len[i]. With
 * logit = softmax_scale * <q[i][h], x>:
 *   out[i][h] = sum_x softmax(logit)_x * x,   lse[i][h] = ln sum_x exp(logit_x).
 * An empty entry set gives out = 0 and lse = -inf.
 * Arguments:
 *   q          bf16 [n_queries][heads][dim]   heads 1..64, dim 128 or 512
 *   sel_idx    int32 [n_queries][topk] device; entries must be < n_blocks[b]
 *              (larger ones set CSA_DEV_BAD_INDEX and are skipped)
 *   win_kv     bf16 [rows][dim]; win_start int64 [n_queries]; win_len int32 [n_queries]
 *              (all three may be NULL together: no window); max_win bounds win_len
 *   out        float32 [n_queries][heads][dim]; lse float32 [n_queries][heads] or NULL
 *   workspace  >= csa_attend_workspace(cache, n_queries, heads) bytes, 256-byte aligned;
 *              it holds an fp16 copy of every query (n_queries * 64 * dim * 2 bytes)
 *              and two partial outputs per SM
 */
csa_status csa_decode_attend(const csa_cache *cache, const void *q, int32_t n_queries, int32_t heads,
                             const int32_t *q_offsets, const int32_t *sel_idx, int32_t topk,
                             const void *win_kv, const int64_t *win_start, const int32_t *win_len,
                             int32_t max_win, float softmax_scale, float *out, float *lse,
                             void *workspace, size_t workspace_bytes, csa_stream_t stream);

/*
 * Row a7 (+ a8): HCA dense attention. As csa_decode_attend, but the compressed
 * entries of query i are every visible block j < min(floor((q_pos[i]+1)/m),
 * n_blocks[b]) of the cache, in order; no indexer, no selection.
 */
csa_status hca_decode_attend(const csa_cache *cache, const void *q, int32_t n_queries, int32_t heads,
                             const int32_t *q_offsets, const int32_t *q_pos,
                             const void *win_kv, const int64_t *win_start, const int32_t *win_len,
                             int32_t max_win, float softmax_scale, float *out, float *lse,
                             void *workspace, size_t workspace_bytes, csa_stream_t stream);

/*
 * Waits for `stream`, then copies *cache->status to *out_flags and clears the
 * device word. The only call that synchronizes. Returns CSA_ERR_NULL when
 * cache->status is NULL.
 */
csa_status csa_read_device_status(const csa_cache *cache, csa_stream_t stream, int32_t *out_flags);

/*
 * Measurement helper with no counterpart on the pages: the issue rate of the
 * block-scaled MXFP4 tensor-core MMA that the prefill indexer GEMM uses
 * (tcgen05.mma kind::mxf4, M = 128, N = 256, K = 64, E8M0 scales per 32), so
 * that the GEMM can be reported against a measured MXFP4 peak. One CTA per SM
 * issues `iters` pairs of MMAs from resident shared-memory tiles into tensor
 * memory; no global data moves. *flops receives the dense FLOPs of the launch
 * (SMs x iters x 2 x 128 x 256 x 128); time the call with events on `stream`.
 * `status`: a device int32 word (4-byte aligned) that receives CSA_DEV_TIMEOUT
 * if the MMAs' completion is not seen (read it with cudaMemcpy or the caller's
 * own means). Errors: CSA_ERR_NULL (status or flops NULL), CSA_ERR_SHAPE
 * (iters < 1), CSA_ERR_ALIGN, CSA_ERR_CUDA (launch failure).
 */
csa_status csa_probe_mxf4_mma(int32_t iters, int32_t *status, csa_stream_t stream, int64_t *flops);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H */
