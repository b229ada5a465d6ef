"""GPU parity of the MXFP4 indexer-key mode (CSA_IDX_MXFP4) against the oracle, through the C ABI.

The pooled indexer keys are stored like the main KV -- E2M1 codes with one E8M0
scale per 32 channels (DeepSeek-V4.1-Flash podcast transcript, cue 16: MXFP4
main KV; cue 12: indexer keys come from the main KV) -- and the indexer query
is quantized by the same rule before the scores, so every product is exact.
Cases: the key store (m = 1 strict, pooled with the near-tie rule), decode
scoring at d_I = 64 / 128 / 256 with ragged contexts, many queries per request
(the block-scaled tensor-core GEMM: several requests per query tile, ragged key
counts, 60 binades of scales, exact ties), exact ties on the streamed path, the
pool + Reindex calls, and the head limit."""
import numpy as np
import pytest

import oracle
from fp4_kv_cache_csa_b200 import datagen
from gpu_util import dev, host, make_cache
import parity
from test_gpu_index import decode_layout
from test_gpu_pool import block_max_rows, check_reindex

pytestmark = pytest.mark.gpu


def mx_keys(B, cap, dI, seed, scale_lo=122, scale_hi=128):
    """Random MXFP4 keys: code bytes uniform, E8M0 scale bytes in [scale_lo, scale_hi)."""
    g = datagen.generator(seed, 60)
    codes = g.integers(0, 256, size=(B, cap, dI // 2)).astype(np.uint8)
    scales = g.integers(scale_lo, scale_hi, size=(B, cap, dI // 32)).astype(np.uint8)
    return codes, scales


def mx_cache(codes, scales, n_blocks, m=4, D=128):
    B, cap, _ = codes.shape
    return make_cache(np.zeros((B, cap, D // 2), np.uint8), np.zeros((B, cap, D // 32), np.uint8), n_blocks, m,
                      codes, 2, idx_key_scale=scales)


def run_index(codes, scales, n_blocks, q_offsets, q_pos, H_I, k, seed, m=4):
    import fp4_kv_cache_csa_b200 as csa

    B, cap, half = codes.shape
    dI = 2 * half
    Nq = int(q_offsets[-1])
    q_idx = datagen.normal_bf16((Nq, H_I, dI), seed, 61)
    w = datagen.normal_f32((Nq, H_I), seed, 62, std=1.0 / np.sqrt(H_I))
    sel_ref, scores, n_vis = oracle.index_topk(codes, n_blocks, q_offsets, q_pos, q_idx, w, m=m, k=k,
                                               idx_dtype=oracle.IDX_MXFP4, idx_key_scale=scales)
    cache = mx_cache(codes, scales, n_blocks, m)
    sel = host(csa.csa_index_topk(cache, dev(q_idx), dev(w), dev(np.asarray(q_offsets, np.int32)),
                                  dev(np.asarray(q_pos, np.int32)), k))
    assert csa.csa_read_device_status(cache) == 0
    near = parity.check_topk(sel, sel_ref, scores, n_vis, k)
    assert len(near) <= max(1, Nq // 4)
    return sel, sel_ref, n_vis


@pytest.mark.parametrize("D,dI", [(128, 64), (512, 128), (256, 256)])
def test_key_store_m1_is_bit_exact(D, dI):
    import torch

    import fp4_kv_cache_csa_b200 as csa

    # m = 1: the gate weight is exactly 1; the stored codes and scales must equal the oracle's
    counts = [37, 5, 64]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    T = int(offs[-1])
    kv = datagen.normal_bf16((T, D), 63, 1)
    idx = datagen.normal_bf16((T, dI), 63, 2, std=2.0)
    wg = datagen.normal_f32((D,), 63, 3, std=0.02)
    base = [0, 3, 1]
    ref = oracle.compress(kv, idx, wg, offs, np.asarray(base, np.int32), m=1, cap=128, idx_dtype=oracle.IDX_MXFP4)
    cache = csa.Cache.allocate(3, 128, D, 1, dI, csa.CSA_IDX_MXFP4)
    cache.n_blocks.copy_(torch.tensor(base, dtype=torch.int32))
    csa.csa_compress_quantize(cache, dev(kv), dev(idx), dev(wg), dev(offs))
    assert csa.csa_read_device_status(cache) == 0
    assert np.array_equal(host(cache.idx_key), ref["idx_key"])
    assert np.array_equal(host(cache.idx_key_scale), ref["idx_key_scale"])


@pytest.mark.parametrize("dI,m", [(128, 4), (64, 16), (256, 4)])
def test_key_store_pooled(dI, m):
    import torch

    import fp4_kv_cache_csa_b200 as csa

    D = 512
    counts = [m * 300, m * 7, 0, m * 129]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    T = int(offs[-1])
    kv = datagen.normal_bf16((T, D), 64, 1, channel_lognormal=0.5)
    idx = datagen.normal_bf16((T, dI), 64, 2, channel_lognormal=0.5)
    wg = datagen.normal_f32((D,), 64, 3, std=0.02)
    base = np.array([5, 0, 2, 17], np.int32)
    cap = 512
    ref = oracle.compress(kv, idx, wg, offs, base, m=m, cap=cap, idx_dtype=oracle.IDX_MXFP4, return_pooled=True)
    cache = csa.Cache.allocate(4, cap, D, m, dI, csa.CSA_IDX_MXFP4)
    cache.n_blocks.copy_(torch.tensor(base))
    csa.csa_compress_quantize(cache, dev(kv), dev(idx), dev(wg), dev(offs))
    assert csa.csa_read_device_status(cache) == 0
    tol = parity.pooling_tolerance(idx, offs, base, m, cap, kv_bits=kv, w_g=wg)
    parity.check_mxfp4(host(cache.idx_key).reshape(4 * cap, -1), host(cache.idx_key_scale).reshape(4 * cap, -1),
                       ref["idx_key"].reshape(4 * cap, -1), ref["idx_key_scale"].reshape(4 * cap, -1),
                       ref["pooled_idx"].reshape(4 * cap, dI), tol=tol.reshape(4 * cap, dI))


@pytest.mark.parametrize("dI", [64, 128, 256])
def test_decode_ragged(dI):
    lengths = [5000, 16384, 700, 12001]
    codes, scales = mx_keys(4, 16384, dI, 65)
    qo, qp = decode_layout(lengths)
    run_index(codes, scales, lengths, qo, qp, 4, 512, seed=66)


def test_wide_scale_spread_and_few_heads():
    # scale bytes over 60 binades and fewer heads than the four the scores pair with groups
    lengths = [3000, 2500]
    codes, scales = mx_keys(2, 4096, 128, 67, scale_lo=100, scale_hi=160)
    qo, qp = decode_layout(lengths)
    for H_I in (1, 3):
        run_index(codes, scales, lengths, qo, qp, H_I, 300, seed=68 + H_I)


def test_fewer_visible_than_k_and_empty():
    lengths = [300, 0, 1024, 1]
    codes, scales = mx_keys(4, 2048, 128, 70)
    qo, qp = decode_layout(lengths)
    sel, _, n_vis = run_index(codes, scales, lengths, qo, qp, 4, 512, seed=71)
    assert list(sel[0, :300]) == list(range(300)) and np.all(sel[0, 300:] == -1)
    assert np.all(sel[1] == -1)
    assert sel[3, 0] == 0 and np.all(sel[3, 1:] == -1)


def test_exact_ties_go_to_the_lower_index():
    # every key zero: all scores 0, the k lowest indices win
    lengths = [3000, 1500]
    codes = np.zeros((2, 3000, 64), np.uint8)
    scales = np.full((2, 3000, 4), 127, np.uint8)
    qo, qp = decode_layout(lengths)
    sel, _, _ = run_index(codes, scales, lengths, qo, qp, 4, 256, seed=72)
    assert np.array_equal(sel[0], np.arange(256)) and np.array_equal(sel[1], np.arange(256))


def test_many_queries_per_request_causal():
    # prefill-shaped: 40 queries per request at spread positions (the block-scaled GEMM path)
    lengths = [3000, 2200]
    codes, scales = mx_keys(2, 3001, 128, 73)
    g = datagen.generator(73, 1)
    per = 40
    qo = (np.arange(3) * per).astype(np.int32)
    qp = np.concatenate([np.sort(g.integers(0, 4 * n, per)) for n in lengths]).astype(np.int32)
    run_index(codes, scales, lengths, qo, qp, 4, 256, seed=74)


@pytest.mark.parametrize("H_I,cap", [(4, 3000), (2, 3001), (1, 3002)])
def test_prefill_gemm_path(H_I, cap):
    # many queries per request score on the block-scaled tensor-core GEMM (kind::mxf4):
    # ragged request sizes put two or three requests into one 128-column query tile,
    # key counts end inside a 128-key stage, one request has a single query
    counts = [300, 213, 1]
    lengths = [3000, 2100, 500]
    codes, scales = mx_keys(3, cap, 128, 80 + H_I)
    qo = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    qp = np.concatenate([np.linspace(0, 4 * L - 1, c).astype(np.int32) for c, L in zip(counts, lengths)])
    sel, _, n_vis = run_index(codes, scales, lengths, qo, qp, H_I, 256, seed=81)
    assert n_vis.min() < 256 < n_vis.max()


def test_prefill_gemm_path_scale_spread():
    # key scales over 20 binades on the block-scaled MMA (the streamed path's test above
    # spans 60): the tensor core anchors a block-scaled sum at the largest block scale
    # taking part, even where that block's products cancel to zero, so keys whose
    # 32-channel scales lie dozens of binades apart can lose a small block's part that
    # fp32 keeps; pooled keys' scales span a few binades
    counts, lengths = [64, 64], [4000, 3500]
    codes, scales = mx_keys(2, 4096, 128, 82, scale_lo=117, scale_hi=137)
    qo = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    qp = np.concatenate([np.linspace(2 * L, 4 * L - 1, c).astype(np.int32) for c, L in zip(counts, lengths)])
    run_index(codes, scales, lengths, qo, qp, 4, 500, seed=83)


@pytest.mark.parametrize("case", ["duplicates", "zeros"])
def test_prefill_gemm_path_exact_ties(case):
    # equal scores at the threshold go to the lower index on the GEMM path as well
    cap = 8192
    codes, scales = mx_keys(2, cap, 128, 84)
    rng = np.random.default_rng(85)
    for b in range(2):
        if case == "duplicates":
            dup = rng.choice(cap, 3000, replace=False)
            codes[b, dup] = codes[b, dup[0]]
            scales[b, dup] = scales[b, dup[0]]
        else:
            codes[b, :5000] = 0
    counts, lengths = [64, 64], [8192, 6000]
    qo = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    qp = np.concatenate([np.linspace(2 * L, 4 * L - 1, c).astype(np.int32) for c, L in zip(counts, lengths)])
    for k in (100, 2999, 3500):
        run_index(codes, scales, lengths, qo, qp, 4, k, seed=86)


def test_pool_and_reindex():
    import fp4_kv_cache_csa_b200 as csa

    lengths = [16384, 9000, 700, 12001]
    B, cap, dI, H_I, k, G, P = 4, 16384, 128, 4, 512, 8, 300
    codes, scales = mx_keys(B, cap, dI, 75)
    qo, qp = decode_layout(lengths)
    q_full = datagen.normal_bf16((B, H_I, dI), 76, 30)
    w_full = datagen.normal_f32((B, H_I), 76, 31, std=0.5)
    q_re = datagen.normal_bf16((B, H_I, dI), 76, 32)
    w_re = datagen.normal_f32((B, H_I), 76, 33, std=0.5)
    kw = dict(m=4, idx_dtype=oracle.IDX_MXFP4, idx_key_scale=scales)
    s_full, n_vis = oracle.index_scores(codes, lengths, qo, qp, q_full, w_full, **kw)
    s_re, _ = oracle.index_scores(codes, lengths, qo, qp, q_re, w_re, **kw)
    cache = mx_cache(codes, scales, lengths)
    sel, pool = csa.csa_index_topk_pool(cache, dev(q_full), dev(w_full), dev(qo), dev(qp), k, pool_group=G,
                                        pool_blocks=P)
    assert csa.csa_read_device_status(cache) == 0
    sel, pool = host(sel), host(pool)
    parity.check_topk(sel, oracle.topk(s_full, n_vis, k), s_full, n_vis, k)
    bmax, nb = block_max_rows(s_full, n_vis, G)
    parity.check_topk(pool, oracle.index_pool(s_full, n_vis, G=G, P=P), bmax, nb, P)
    sel_re = host(csa.csa_index_topk_reindex(cache, dev(q_re), dev(w_re), dev(qo), dev(qp), k, dev(pool),
                                             pool_group=G))
    assert csa.csa_read_device_status(cache) == 0
    check_reindex(sel_re, oracle.reindex_topk(s_re, n_vis, pool, G=G, k=k), s_re, n_vis, pool, G, k)


def test_more_than_four_heads_is_refused():
    import fp4_kv_cache_csa_b200 as csa

    codes, scales = mx_keys(1, 256, 128, 77)
    cache = mx_cache(codes, scales, [200])
    qo, qp = decode_layout([200])
    q = dev(datagen.normal_bf16((1, 8, 128), 77, 1))
    w = dev(datagen.normal_f32((1, 8), 77, 2))
    with pytest.raises(csa.CsaError, match="status 4"):
        csa.csa_index_topk(cache, q, w, dev(qo), dev(qp), 16)


def test_mxf4_mma_probe_completes():
    # the measurement helper behind the MXFP4 peak: block-scaled MMAs on every SM finish
    # within the wait limit and report the FLOPs they issued
    import torch

    import fp4_kv_cache_csa_b200 as csa

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flops = csa.csa_probe_mxf4_mma(64, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert flops == torch.cuda.get_device_properties(0).multi_processor_count * 64 * 2 * 128 * 256 * 128
