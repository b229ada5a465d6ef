"""GPU parity of the hierarchical indexer pool (csa_index_topk_pool) and the CSA2
Reindex selection (csa_index_topk_reindex) against the oracle, through the C ABI.

Keys are seeded E4M3 (or bf16) N(0, 0.5^2) values as in the indexer tests; the
Full-mode and Reindex-mode layers have independent seeded indexer queries."""
import numpy as np
import pytest

import oracle
from fp4_kv_cache_csa_b200 import datagen
from gpu_util import dev, host, make_cache
import parity
from test_gpu_index import decode_layout, gen_keys

pytestmark = pytest.mark.gpu


def block_max_rows(scores, n_vis, G):
    """Per query the G-block maxima of its visible scores (rows padded with -inf)."""
    Nq, cap = scores.shape
    nb = (np.asarray(n_vis) + G - 1) // G
    out = np.full((Nq, max(1, (cap + G - 1) // G)), -np.inf, np.float32)
    for i in range(Nq):
        for b in range(nb[i]):
            out[i, b] = scores[i, G * b:min(G * b + G, n_vis[i])].max()
    return out, nb.astype(np.int32)


def check_reindex(sel, ref, scores, n_vis, pool, G, k):
    """Exact match unless the k-th and (k+1)-th best pool candidates are a near-tie
    (then the GPU set must be a valid top-k of the candidates within 1e-5)."""
    for i in range(sel.shape[0]):
        if np.array_equal(sel[i], ref[i]):
            continue
        cand = np.array(sorted(j for b in pool[i] if b >= 0 for j in range(G * b, min(G * b + G, n_vis[i]))))
        K = min(k, len(cand))
        s = scores[i, cand].astype(np.float64)
        order = np.lexsort((cand, -s))
        kth, nxt = s[order[K - 1]], s[order[K]] if K < len(cand) else -np.inf
        tol = parity.REL * max(abs(kth), 1e-30)
        assert abs(kth - nxt) < tol, f"query {i}: Reindex top-k differs without a near-tie"
        g = sel[i]
        assert np.all(g[K:] == -1) and np.all(np.diff(g[:K]) > 0) and set(g[:K]) <= set(cand)


def run(lengths, cap, dI, idx_dtype, k, G, P, seed, H_I=4, m=4):
    import fp4_kv_cache_csa_b200 as csa

    B = len(lengths)
    keys = gen_keys(B, cap, dI, idx_dtype, seed)
    qo, qp = decode_layout(lengths)
    Nq = B
    q_full = datagen.normal_bf16((Nq, H_I, dI), seed, 30)
    w_full = datagen.normal_f32((Nq, H_I), seed, 31, std=1.0 / np.sqrt(H_I))
    q_re = datagen.normal_bf16((Nq, H_I, dI), seed, 32)
    w_re = datagen.normal_f32((Nq, H_I), seed, 33, std=1.0 / np.sqrt(H_I))
    s_full, n_vis = oracle.index_scores(keys, lengths, qo, qp, q_full, w_full, m=m, idx_dtype=idx_dtype)
    s_re, _ = oracle.index_scores(keys, lengths, qo, qp, q_re, w_re, m=m, idx_dtype=idx_dtype)
    sel_ref = oracle.topk(s_full, n_vis, k)
    pool_ref = oracle.index_pool(s_full, n_vis, G=G, P=P)

    D = 128
    cache = make_cache(np.zeros((B, cap, D // 2), np.uint8), np.zeros((B, cap, D // 32), np.uint8), lengths, m,
                       keys if idx_dtype == 1 else keys.view(np.uint16), idx_dtype)
    sel, pool = csa.csa_index_topk_pool(cache, dev(q_full), dev(w_full), dev(qo), dev(qp), k, pool_group=G,
                                        pool_blocks=P)
    assert csa.csa_read_device_status(cache) == 0
    sel, pool = host(sel), host(pool)
    parity.check_topk(sel, sel_ref, s_full, n_vis, k)
    bmax, nb = block_max_rows(s_full, n_vis, G)
    parity.check_topk(pool, pool_ref, bmax, nb, P)  # same near-tie rule on the block scores

    # Reindex on the GPU's own pool
    sel_re = host(csa.csa_index_topk_reindex(cache, dev(q_re), dev(w_re), dev(qo), dev(qp), k, dev(pool),
                                             pool_group=G))
    assert csa.csa_read_device_status(cache) == 0
    ref_re = oracle.reindex_topk(s_re, n_vis, pool, G=G, k=k)
    check_reindex(sel_re, ref_re, s_re, n_vis, pool, G, k)
    return dict(sel=sel, pool=pool, sel_re=sel_re, s_re=s_re, n_vis=n_vis)


@pytest.mark.parametrize("idx_dtype,dI", [(1, 128), (0, 64)])
def test_pool_and_reindex_ragged(idx_dtype, dI):
    r = run([16384, 9000, 700, 12001], 16384, dI, idx_dtype, k=512, G=8, P=300, seed=40)
    # a context of 700 blocks has 88 pool blocks: all kept, so Reindex is its plain top-k
    assert np.all(r["pool"][2, :88] == np.arange(88)) and np.all(r["pool"][2, 88:] == -1)
    plain = oracle.topk(r["s_re"][2:3], r["n_vis"][2:3], 512)
    assert np.array_equal(r["sel_re"][2:3], plain)


def test_single_block_groups_and_small_pool():
    # G = 1: the pool is the Full layer's top-P; a pool smaller than k pads the Reindex row
    r = run([5000, 3000], 8192, 128, 1, k=256, G=1, P=100, seed=41)
    assert np.all(r["sel_re"][:, 100:] == -1)


def test_large_groups_and_pool_covering_everything():
    r = run([4096, 1000], 4096, 128, 1, k=128, G=32, P=200, seed=42)
    for i in range(2):
        plain = oracle.topk(r["s_re"][i:i + 1], r["n_vis"][i:i + 1], 128)
        assert np.array_equal(r["sel_re"][i:i + 1], plain)


def test_bad_pool_entries_are_flagged_and_end_the_list():
    import fp4_kv_cache_csa_b200 as csa

    lengths = [2000]
    keys = gen_keys(1, 2048, 128, 1, 43)
    qo, qp = decode_layout(lengths)
    q = datagen.normal_bf16((1, 4, 128), 43, 30)
    w = datagen.normal_f32((1, 4), 43, 31, std=0.5)
    s, n_vis = oracle.index_scores(keys, lengths, qo, qp, q, w, m=4, idx_dtype=1)
    cache = make_cache(np.zeros((1, 2048, 64), np.uint8), np.zeros((1, 2048, 4), np.uint8), lengths, 4, keys, 1)
    pool = np.array([[3, 10, 9, 40, -1]], np.int32)  # 9 after 10 breaks the ascending order
    sel = host(csa.csa_index_topk_reindex(cache, dev(q), dev(w), dev(qo), dev(qp), 8, dev(pool), pool_group=8))
    assert csa.csa_read_device_status(cache) & csa.CSA_DEV_BAD_INDEX
    ref = oracle.reindex_topk(s, n_vis, np.array([[3, 10, -1, -1, -1]], np.int32), G=8, k=8)
    check_reindex(sel, ref, s, n_vis, np.array([[3, 10, -1, -1, -1]]), 8, 8)


@pytest.mark.parametrize("idx_dtype,dI,L", [(1, 128, 3), (0, 64, 2), (2, 128, 4)])
def test_reindex_layers_in_one_call(idx_dtype, dI, L):
    # L Reindex layers over one Full layer's pool in one call: each layer's selection is
    # the oracle's Reindex selection for that layer's own query and weights
    import fp4_kv_cache_csa_b200 as csa

    lengths = [16384, 9000, 700, 12001]
    B, cap, H_I, k, G, P = 4, 16384, 4, 512, 8, 300
    qo, qp = decode_layout(lengths)
    if idx_dtype == 2:
        from test_gpu_mxfp4_index import mx_keys
        keys, ksc = mx_keys(B, cap, dI, 90)
        kw = dict(m=4, idx_dtype=2, idx_key_scale=ksc)
        cache = make_cache(np.zeros((B, cap, 64), np.uint8), np.zeros((B, cap, 4), np.uint8), lengths, 4, keys, 2,
                           idx_key_scale=ksc)
    else:
        keys = gen_keys(B, cap, dI, idx_dtype, 90)
        kw = dict(m=4, idx_dtype=idx_dtype)
        cache = make_cache(np.zeros((B, cap, 64), np.uint8), np.zeros((B, cap, 4), np.uint8), lengths, 4,
                           keys if idx_dtype == 1 else keys.view(np.uint16), idx_dtype)
    q_full = datagen.normal_bf16((B, H_I, dI), 91, 30)
    w_full = datagen.normal_f32((B, H_I), 91, 31, std=0.5)
    _, pool = csa.csa_index_topk_pool(cache, dev(q_full), dev(w_full), dev(qo), dev(qp), k, pool_group=G,
                                      pool_blocks=P)
    pool = host(pool)
    q_re = datagen.normal_bf16((B, L, H_I, dI), 91, 32)
    w_re = datagen.normal_f32((B, L, H_I), 91, 33, std=0.5)
    sel = host(csa.csa_index_topk_reindex_layers(cache, dev(q_re), dev(w_re), dev(qo), dev(qp), k, dev(pool),
                                                 pool_group=G))
    assert csa.csa_read_device_status(cache) == 0
    assert sel.shape == (B, L, k)
    for l in range(L):
        s_re, n_vis = oracle.index_scores(keys, lengths, qo, qp, np.ascontiguousarray(q_re[:, l]),
                                          np.ascontiguousarray(w_re[:, l]), **kw)
        ref = oracle.reindex_topk(s_re, n_vis, pool, G=G, k=k)
        check_reindex(sel[:, l], ref, s_re, n_vis, pool, G, k)
