"""csa_index_topk in chunks of queries, through the C ABI.

A call runs its queries in consecutive chunks on one workspace when the
workspace it is given cannot hold all of them at once (any size from one
chunk of 128 queries up). Every query is scored and selected on its own, so a
chunked call must return exactly what one pass returns, and both must match
the oracle. Cases: the tensor-core GEMM with row selection (bf16 and MXFP4
keys: the quantized query is rebuilt per chunk), the streamed path with a
GEMM-capable key format but a head count the GEMM does not serve (bf16, 3
heads), the streamed path with e4m3 keys in chunks above and below the
in-kernel schedule's 512 queries, and a workspace below one chunk."""
import numpy as np
import pytest

import oracle
from fp4_kv_cache_csa_b200 import datagen
from gpu_util import dev, host, make_cache
import parity
from test_gpu_index import gen_keys
from test_gpu_mxfp4_index import mx_cache, mx_keys

pytestmark = pytest.mark.gpu

LENGTHS = [3000, 2100, 500]  # filled blocks per request
COUNTS = [700, 513, 187]     # queries per request (1400): ragged, requests share query tiles and chunks
CAP = 3001


def layout(counts=COUNTS, lengths=LENGTHS):
    qo = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    # each request's queries at increasing positions up to its last token (m = 4)
    qp = np.concatenate([np.linspace(0, 4 * L - 1, c).astype(np.int32) for c, L in zip(counts, lengths)])
    return qo, qp


def check(cache, keys, scales, idx_dtype, H_I, k, ws_bytes, seed):
    """One pass and a chunked call on a workspace of ws_bytes: equal to each other and to the oracle."""
    import torch

    import fp4_kv_cache_csa_b200 as csa

    B, cap, _ = keys.shape
    dI = 2 * keys.shape[2] if idx_dtype == 2 else (keys.shape[2] // 2 if idx_dtype == 0 else keys.shape[2])
    qo, qp = layout()
    Nq = int(qo[-1])
    q_idx = datagen.normal_bf16((Nq, H_I, dI), seed, 8)
    w = datagen.normal_f32((Nq, H_I), seed, 9, std=1.0 / np.sqrt(H_I))
    args = (dev(q_idx), dev(w), dev(qo), dev(qp), k)
    one = host(csa.csa_index_topk(cache, *args))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    chunked = host(csa.csa_index_topk(cache, *args, workspace=ws))
    assert csa.csa_read_device_status(cache) == 0
    assert np.array_equal(chunked, one)
    sel_ref, scores, n_vis = oracle.index_topk(keys, LENGTHS, qo, qp, q_idx, w, m=4, k=k, idx_dtype=idx_dtype,
                                               **({"idx_key_scale": scales} if idx_dtype == 2 else {}))
    near = parity.check_topk(chunked, sel_ref, scores, n_vis, k)
    assert len(near) <= max(1, Nq // 4)
    return Nq


def plain_cache(keys, idx_dtype):
    B, cap, _ = keys.shape
    return make_cache(np.zeros((B, cap, 64), np.uint8), np.zeros((B, cap, 4), np.uint8), LENGTHS, 4,
                      keys if idx_dtype == 1 else keys.view(np.uint16), idx_dtype)


@pytest.mark.parametrize("idx_dtype", [0, 2])
def test_gemm_row_selection_in_chunks(idx_dtype):
    # score rows of 400 queries fit (4 CAP bytes each, plus the quantized query): chunks of 384
    # queries, the last one ragged; all 1400 queries' rows would need 3.5x that
    if idx_dtype == 2:
        keys, scales = mx_keys(3, CAP, 128, 90)
        cache = mx_cache(keys, scales, LENGTHS)
    else:
        keys, scales = gen_keys(3, CAP, 128, 0, 90), None
        cache = plain_cache(keys, 0)
    ws_bytes = 4 * CAP * 400 + (256 << 10)
    assert ws_bytes < 4 * CAP * 1400
    check(cache, keys, scales, idx_dtype, 4, 256, ws_bytes, seed=91)


@pytest.mark.parametrize("idx_dtype,H_I,queries", [(0, 3, 128), (1, 4, 640), (1, 4, 256)])
def test_streamed_path_in_chunks(idx_dtype, H_I, queries):
    # the full workspace layout (score rows, segment candidates, selection state: about
    # 12 CAP + 290K bytes per query) for `queries` queries: chunks of 128 or 256 queries
    # (the scan computes their schedule itself) or 640 (the schedule kernel does)
    keys = gen_keys(3, CAP, 128, idx_dtype, 92 + H_I)
    cache = plain_cache(keys, idx_dtype)
    per_query = 12 * CAP + 4 * 4096 + 8 * 32768 + 4 * ((CAP + 31) // 32) + 64
    ws_bytes = per_query * queries + (1 << 20)
    assert ws_bytes < per_query * 1400
    check(cache, keys, None, idx_dtype, H_I, 300, ws_bytes, seed=93)


def test_workspace_below_one_chunk_is_refused():
    import torch

    import fp4_kv_cache_csa_b200 as csa

    keys = gen_keys(3, CAP, 128, 0, 94)
    cache = plain_cache(keys, 0)
    qo, qp = layout()
    Nq = int(qo[-1])
    q_idx = dev(datagen.normal_bf16((Nq, 4, 128), 95, 8))
    w = dev(datagen.normal_f32((Nq, 4), 95, 9, std=0.5))
    ws = torch.empty(4 * CAP * 100, dtype=torch.uint8, device="cuda")  # 100 queries' score rows < 128
    with pytest.raises(csa.CsaError, match="workspace"):
        csa.csa_index_topk(cache, q_idx, w, dev(qo), dev(qp), 256, workspace=ws)
