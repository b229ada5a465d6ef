"""GPU parity of csa_index_topk (rows a3 + a4) against the oracle, through the C ABI.

Keys are seeded inputs: bf16 N(0, 0.5^2) (the spread of 4-token pooled N(0,1)
keys) or the same values cast to E4M3."""
import numpy as np
import pytest

import oracle
from fp4_kv_cache_csa_b200 import datagen
from gpu_util import dev, host, make_cache
import parity

pytestmark = pytest.mark.gpu


def gen_keys(B, cap, dI, idx_dtype, seed):
    x = datagen.normal_f32((B, cap, dI), seed, 7, std=0.5)
    if idx_dtype == 0:
        return datagen.to_bf16_bits(x).view(np.uint8).reshape(B, cap, 2 * dI)
    return datagen.to_e4m3_bytes(x).reshape(B, cap, dI)


def run(keys, n_blocks, q_offsets, q_pos, H_I, dI, k, idx_dtype, seed, m=4):
    import fp4_kv_cache_csa_b200 as csa

    B, cap, _ = keys.shape
    Nq = int(q_offsets[-1])
    q_idx = datagen.normal_bf16((Nq, H_I, dI), seed, 8)
    w = datagen.normal_f32((Nq, H_I), seed, 9, std=1.0 / np.sqrt(H_I))
    sel_ref, scores, n_vis = oracle.index_topk(keys, n_blocks, q_offsets, q_pos, q_idx, w, m=m, k=k,
                                               idx_dtype=idx_dtype)
    D = 128
    fp4 = np.zeros((B, cap, D // 2), np.uint8)
    sc = np.zeros((B, cap, D // 32), np.uint8)
    cache = make_cache(fp4, sc, n_blocks, m, keys if idx_dtype == 1 else keys.view(np.uint16), idx_dtype)
    sel = csa.csa_index_topk(cache, dev(q_idx), dev(w), dev(np.asarray(q_offsets, np.int32)),
                             dev(np.asarray(q_pos, np.int32)), k)
    assert csa.csa_read_device_status(cache) == 0
    sel = host(sel)
    near = parity.check_topk(sel, sel_ref, scores, n_vis, k)
    assert len(near) <= max(1, Nq // 4)
    return sel, sel_ref, n_vis


def decode_layout(lengths):
    B = len(lengths)
    q_offsets = np.arange(B + 1, dtype=np.int32)
    q_pos = (np.asarray(lengths) * 4 - 1).astype(np.int32)  # query at the last token; m = 4
    return q_offsets, q_pos


def test_tiny_bf16_dim64():
    keys = gen_keys(1, 1024, 64, 0, 20)
    qo, qp = decode_layout([1024])
    run(keys, [1024], qo, qp, 4, 64, 64, 0, seed=21)


@pytest.mark.parametrize("idx_dtype,dI", [(0, 128), (1, 128), (1, 64), (0, 256)])
def test_ragged_batch(idx_dtype, dI):
    lengths = [5000, 16384, 700, 12001]
    keys = gen_keys(4, 16384, dI, idx_dtype, 22)
    qo, qp = decode_layout(lengths)
    run(keys, lengths, qo, qp, 4, dI, 512, idx_dtype, seed=23)


def test_fewer_visible_than_k_and_empty():
    lengths = [300, 0, 1024, 1]
    keys = gen_keys(4, 2048, 128, 1, 24)
    qo, qp = decode_layout(lengths)
    sel, _, n_vis = run(keys, lengths, qo, qp, 4, 128, 512, 1, seed=25)
    assert list(sel[0, :300]) == list(range(300)) and np.all(sel[0, 300:] == -1)
    assert np.all(sel[1] == -1)
    assert sel[3, 0] == 0 and np.all(sel[3, 1:] == -1)


def test_exact_ties_go_to_the_lower_index():
    # 3000 identical keys among random ones: equal scores, the lower block index wins
    keys = gen_keys(1, 8192, 128, 1, 26)
    rng = np.random.default_rng(27)
    dup = rng.choice(8192, 3000, replace=False)
    keys[0, dup] = keys[0, dup[0]]
    qo, qp = decode_layout([8192])
    for k in (100, 1000, 2999, 3500):
        run(keys, [8192], qo, qp, 4, 128, k, 1, seed=28)


def test_candidate_overflow_path():
    # 60000 identical keys: the threshold bin holds more candidates than the list keeps
    keys = gen_keys(1, 65536, 64, 0, 29)
    keys[0, :60000] = keys[0, 12345]
    qo, qp = decode_layout([65536])
    for k in (777, 4096):
        run(keys, [65536], qo, qp, 4, 64, k, 0, seed=30)


@pytest.mark.parametrize("idx_dtype", [0, 1])
def test_two_ctas_per_query_merge(idx_dtype):
    # 24 decode queries (one per request) take the merge on two CTAs (a cluster) per
    # query, each ranking half of the candidates: ragged contexts, one query with fewer
    # visible blocks than k, and one whose keys are all equal (every score ties, so the
    # k lowest indices win across the two halves)
    lengths = [2000 + 613 * b for b in range(24)]
    lengths[3] = 100
    cap = max(lengths)
    keys = gen_keys(24, cap, 128, idx_dtype, 40)
    keys[7, :] = keys[7, 0]
    qo, qp = decode_layout(lengths)
    sel, _, n_vis = run(keys, lengths, qo, qp, 4, 128, 512, idx_dtype, seed=41)
    assert list(sel[3, :100]) == list(range(100)) and np.all(sel[3, 100:] == -1)
    assert np.array_equal(sel[7], np.arange(512))


def test_prefill_queries_are_causal():
    # 2 requests, several queries each at increasing positions (causal at block granularity)
    lengths = [4000, 2500]
    keys = gen_keys(2, 4096, 128, 0, 31)
    q_offsets = np.array([0, 5, 9], np.int32)
    q_pos = np.array([3, 100, 4000, 9000, 15999, 1, 5000, 8003, 9999], np.int32)
    sel, _, n_vis = run(keys, lengths, q_offsets, q_pos, 4, 128, 256, 0, seed=32)
    assert list(n_vis) == [1, 25, 1000, 2250, 4000, 0, 1250, 2001, 2500]


@pytest.mark.parametrize("H_I", [1, 3, 8])
def test_head_counts(H_I):
    keys = gen_keys(2, 4096, 128, 1, 33)
    qo, qp = decode_layout([4096, 3000])
    run(keys, [4096, 3000], qo, qp, H_I, 128, 200, 1, seed=34)


def test_maximum_sizes():
    # the largest capacity (2^19 blocks, a 2M-token context), the largest top-k (4096),
    # the most indexer heads (8) and the widest keys (256 bf16 channels)
    cap = 1 << 19
    keys = gen_keys(1, cap, 256, 0, 28)
    qo, qp = decode_layout([cap])
    sel, _, n_vis = run(keys, [cap], qo, qp, 8, 256, 4096, 0, seed=29)
    assert n_vis[0] == cap and np.all(sel[0] >= 0) and np.all(np.diff(sel[0]) > 0)


@pytest.mark.parametrize("H_I,dI,cap", [(4, 128, 3000), (1, 64, 3000), (2, 256, 3001), (8, 128, 3001), (4, 64, 3002),
                                        (4, 256, 3000)])
def test_many_queries_per_request_gemm_path(H_I, dI, cap):
    # calls with many queries per request (prefill) score on the tensor cores; ragged
    # request sizes put two or three requests into one query tile, and capacities that
    # are not multiples of 4 give score rows that are not 16-byte aligned
    counts = [300, 213, 1]
    lengths = [3000, 2100, 500]  # filled blocks per request
    keys = gen_keys(3, cap, dI, 0, 60 + H_I)
    qo = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    # each request's queries at increasing positions up to its last token (m = 4)
    qp = np.concatenate([np.linspace(0, 4 * L - 1, c).astype(np.int32) for c, L in zip(counts, lengths)])
    sel, _, n_vis = run(keys, lengths, qo, qp, H_I, dI, 256, 0, seed=61)
    assert n_vis.min() < 256 < n_vis.max()


@pytest.mark.parametrize("case", ["duplicates", "zeros"])
def test_gemm_path_exact_ties(case):
    # prefill-sized calls (many queries per request) take the GEMM path and the
    # one-CTA-per-query selection; equal scores at the threshold go to the lower index:
    # 3000 identical keys per request, or 5000 all-zero keys (every score exactly 0)
    cap = 8192
    keys = gen_keys(2, cap, 128, 0, 70)
    rng = np.random.default_rng(71)
    for b in range(2):
        if case == "duplicates":
            dup = rng.choice(cap, 3000, replace=False)
            keys[b, dup] = keys[b, dup[0]]
        else:
            keys[b, :5000] = 0
    counts, lengths = [64, 64], [8192, 6000]
    qo = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    qp = np.concatenate([np.linspace(2 * L, 4 * L - 1, c).astype(np.int32) for c, L in zip(counts, lengths)])
    for k in (100, 2999, 3500):
        run(keys, lengths, qo, qp, 4, 128, k, 0, seed=72)
