"""csa_index_topk_noalloc: the indexer + top-k call for callers that cannot
allocate device memory (a host framework that owns every allocation, a fixed
memory budget, or code that cannot afford an allocation's synchronization).
Its scratch is a fixed 32 MiB array inside the library instead of a caller
workspace, so its results must equal csa_index_topk's exactly; and since every
call reuses that array, two calls in a row (with different inputs) must each
still match. A call larger than the scratch runs its queries in chunks
that fit. This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

import fp4_kv_cache_csa_b200 as csa
from fp4_kv_cache_csa_b200 import build as csa_build
from fp4_kv_cache_csa_b200 import datagen

ERR_WORKSPACE = 5


def _inputs(seed, lengths, dI, idx_dtype, k, per_req=1):
    """A cache of random keys; per_req queries per request: one decode query at the end of the
    context (per_req = 1), or per_req queries at spread positions (a prefill-shaped call, which the
    library scores with a tensor-core GEMM and selects per row)."""
    import torch

    from gpu_util import dev, make_cache

    B = len(lengths)
    cap = max(lengths) + 3
    x = datagen.normal_f32((B, cap, dI), seed, 1, std=0.5)
    keys = datagen.to_bf16_bits(x) if idx_dtype == 0 else datagen.to_e4m3_bytes(x)
    cache = make_cache(np.zeros((B, cap, 64), np.uint8), np.zeros((B, cap, 4), np.uint8), lengths, 4, keys,
                       idx_dtype)
    Nq = B * per_req
    q_idx = dev(datagen.normal_bf16((Nq, 4, dI), seed, 2))
    w = dev(datagen.normal_f32((Nq, 4), seed, 3, std=0.5))
    qo = dev((np.arange(B + 1) * per_req).astype(np.int32))
    if per_req == 1:
        pos = np.asarray(lengths) * 4 - 1
    else:
        rng = datagen.generator(seed, 4)
        pos = np.concatenate([np.sort(rng.integers(0, 4 * n, per_req)) for n in lengths])
        pos[::per_req] = 4 * np.asarray(lengths) - 1  # each request's last query sees every block
    qp = dev(pos.astype(np.int32))
    return cache, q_idx, w, qo, qp, torch


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_call_twice_in_a_row():
    cases = [(71, [5000, 16384, 700, 12001], 128, 1, 512, 1),   # e4m3 keys, ragged decode
             (72, [9000, 300, 16000], 64, 0, 1024, 1),          # bf16 keys, another shape
             (73, [8192, 6000], 128, 0, 512, 32),               # prefill-shaped, right after decode
             (74, [3000, 7000, 200], 64, 1, 256, 1)]            # decode again, after the prefill call
    for seed, lengths, dI, dt, k, per_req in cases:  # consecutive calls on the shared scratch
        cache, q_idx, w, qo, qp, torch = _inputs(seed, lengths, dI, dt, k, per_req)
        assert csa.csa_index_topk_workspace(cache, q_idx.shape[0], k) <= (32 << 20)
        want = csa.csa_index_topk(cache, q_idx, w, qo, qp, k)
        got = torch.full_like(want, -7)
        csa.csa_index_topk_noalloc(cache, q_idx, w, qo, qp, k, got)
        torch.cuda.synchronize()
        assert torch.equal(got, want), seed
        assert csa.csa_read_device_status(cache) == 0


@pytest.mark.gpu
def test_noalloc_runs_a_larger_prefill_in_chunks():
    # 1400 prefill queries over 8195-block score rows need 46 MB of rows: the fixed scratch
    # holds 896 queries' rows, so the call runs in two chunks and must still equal one pass
    cache, q_idx, w, qo, qp, torch = _inputs(75, [8192, 6000], 128, 0, 512, per_req=700)
    assert q_idx.shape[0] * 4 * 8195 > (32 << 20)
    want = csa.csa_index_topk(cache, q_idx, w, qo, qp, 512)
    got = torch.full_like(want, -7)
    csa.csa_index_topk_noalloc(cache, q_idx, w, qo, qp, 512, got)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    assert csa.csa_read_device_status(cache) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # checked on the host before any device work: one chunk of 32 queries x 262144 blocks
    # (decode: the streamed layout) needs > 32 MiB
    csa_build.build()
    lib = csa.load_library()
    c = csa._CCache(32, 512, 4, 262144, 0x10000, 0x20000, 0x30000, 128, 1, 0x40000, None)
    assert lib.csa_index_topk_workspace(ctypes.byref(c), 32, 1024) > (32 << 20)
    st = lib.csa_index_topk_noalloc(ctypes.byref(c), 0x90000, 0xA0000, 32, 4, 0xB0000, 0xC0000, 1024, 0xD0000, None)
    assert st == ERR_WORKSPACE
    # argument errors come first, with csa_index_topk's codes: top-k beyond the supported
    # maximum, a NULL output, a misaligned query
    for args, want in (((0x90000, 0xA0000, 32, 4, 0xB0000, 0xC0000, 5000, 0xD0000), 4),
                       ((0x90000, 0xA0000, 32, 4, 0xB0000, 0xC0000, 1024, None), 1),
                       ((0x90001, 0xA0000, 32, 4, 0xB0000, 0xC0000, 1024, 0xD0000), 3)):
        assert lib.csa_index_topk_noalloc(ctypes.byref(c), *args, None) == want
        assert lib.csa_index_topk(ctypes.byref(c), *args, 0x100000, 1 << 40, None) == want
