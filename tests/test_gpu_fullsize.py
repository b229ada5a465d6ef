"""Parity at the full workload sizes, in the launch configuration the benchmark times.

The GPU runs the whole batch; the oracle recomputes sampled queries one by one.
  * csa_b32_1m: 32 requests, 131072..262144 blocks each (512K..1M tokens, m = 4),
    e4m3 indexer keys, k = 1024, D = 512, 64 heads, 128-token window.
  * hca_b64_1m: 64 requests x 8192 blocks (1M tokens, m = 128), dense.
  * csa2 at csa_b32_1m: the Full layer's pool (2000 blocks of 8 entries) and a
    Reindex layer over it, on the same kind of cache.
  * csa_b8_64k: 8 requests x 65536 tokens from raw tokens through every kernel
    (per-channel LogNormal(0, 0.5) activations), checked stage by stage, in both
    scale formats (E8M0 per 32, E4M3 per 16).
  * prefill_b4_8k: 8192 new tokens appended to 65536 cached ones in each of 4
    requests; every new block checked, then 32768 causal queries indexed and
    attended with sampled queries recomputed; and the same indexer call over
    MXFP4 indexer keys (the block-scaled tensor-core GEMM), sampled.
Cache contents for the first two are seeded bytes (the kernels' inputs), not
outputs of the compression kernel."""
import numpy as np
import pytest

import oracle
from fp4_kv_cache_csa_b200 import datagen
from gpu_util import dev, host, make_cache
import parity

pytestmark = pytest.mark.gpu


def test_csa_b32_1m_sampled():
    import torch

    import fp4_kv_cache_csa_b200 as csa

    wl = datagen.WORKLOADS["csa_b32_1m"]
    B, D, H, dI, k, W = wl.batch, wl.dim, wl.heads, wl.idx_dim, wl.topk, wl.window
    n = (datagen.context_lengths(wl, 500) // wl.block).astype(np.int64)
    cap = int(n.max())
    sample = [0, 17, int(np.argmax(n))]
    fp4_d = torch.empty(B, cap, D // 2, dtype=torch.uint8, device="cuda")
    sc_d = torch.empty(B, cap, D // 32, dtype=torch.uint8, device="cuda")
    key_d = torch.empty(B, cap, dI, dtype=torch.uint8, device="cuda")
    host_rows = {}
    for b in range(B):
        f, s = datagen.random_cache_bytes(cap, D, 501, b)
        kx = datagen.to_e4m3_bytes(datagen.normal_f32((cap, dI), 502, b, std=0.5))
        fp4_d[b].copy_(torch.from_numpy(f))
        sc_d[b].copy_(torch.from_numpy(s))
        key_d[b].copy_(torch.from_numpy(kx))
        if b in sample:
            host_rows[b] = (f, s, kx)
    cache = csa.Cache(fp4=fp4_d, scale=sc_d, n_blocks=dev(n.astype(np.int32)), block=wl.block, idx_key=key_d,
                      idx_dtype=csa.CSA_IDX_E4M3, status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    q = datagen.normal_bf16((B, H, D), 503, 1)
    q_idx = datagen.normal_bf16((B, wl.idx_heads, dI), 503, 2)
    w = datagen.normal_f32((B, wl.idx_heads), 503, 3, std=0.5)
    win = datagen.normal_bf16((B * W, D), 503, 4)
    qo = np.arange(B + 1, dtype=np.int32)
    qp = (n * wl.block - 1).astype(np.int32)
    ws_, wl_ = (np.arange(B) * W).astype(np.int64), np.full(B, W, np.int32)
    sel = host(csa.csa_index_topk(cache, dev(q_idx), dev(w), dev(qo), dev(qp), k))
    out = host(csa.csa_decode_attend(cache, dev(q), dev(qo), dev(sel), dev(win), dev(ws_), dev(wl_)))
    assert csa.csa_read_device_status(cache) == 0
    for b in sample:
        f, s, kx = host_rows[b]
        one = np.array([0, 1], np.int32)
        sel_ref, scores, n_vis = oracle.index_topk(kx[None], n[b:b + 1].astype(np.int32), one, qp[b:b + 1],
                                                   q_idx[b:b + 1], w[b:b + 1], m=wl.block, k=k, idx_dtype=1)
        near = parity.check_topk(sel[b:b + 1], sel_ref, scores, n_vis, k)
        use = sel[b:b + 1] if near else sel_ref  # near-tie: attention on the GPU's own selection
        ref, _ = oracle.csa_attend(f[None], s[None], one, q[b:b + 1], use, win[b * W:(b + 1) * W],
                                   np.array([0], np.int64), np.array([W], np.int32), D ** -0.5)
        err, _ = parity.attention_row_error(out[b:b + 1], ref)
        assert err <= parity.ATT_TOL, (b, err)


def test_csa2_pool_reindex_b32_1m_sampled():
    # the Full layer's pool (2000 blocks of 8 entries) and a Reindex layer over it,
    # in the benchmark's configuration; sampled queries recomputed by the oracle
    import torch

    import fp4_kv_cache_csa_b200 as csa
    from test_gpu_pool import block_max_rows, check_reindex

    wl = datagen.WORKLOADS["csa_b32_1m"]
    B, dI, k, G, P = wl.batch, wl.idx_dim, wl.topk, 8, 2000
    n = (datagen.context_lengths(wl, 530) // wl.block).astype(np.int64)
    cap = int(n.max())
    sample = [3, int(np.argmin(n))]
    key_d = torch.empty(B, cap, dI, dtype=torch.uint8, device="cuda")
    host_keys = {}
    for b in range(B):
        kx = datagen.to_e4m3_bytes(datagen.normal_f32((cap, dI), 531, b, std=0.5))
        key_d[b].copy_(torch.from_numpy(kx))
        if b in sample:
            host_keys[b] = kx
    D = 128
    cache = csa.Cache(fp4=torch.zeros(B, cap, D // 2, dtype=torch.uint8, device="cuda"),
                      scale=torch.zeros(B, cap, D // 32, dtype=torch.uint8, device="cuda"),
                      n_blocks=dev(n.astype(np.int32)), block=wl.block, idx_key=key_d, idx_dtype=csa.CSA_IDX_E4M3,
                      status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    q_full = datagen.normal_bf16((B, wl.idx_heads, dI), 532, 1)
    w_full = datagen.normal_f32((B, wl.idx_heads), 532, 2, std=0.5)
    q_re = datagen.normal_bf16((B, wl.idx_heads, dI), 532, 3)
    w_re = datagen.normal_f32((B, wl.idx_heads), 532, 4, std=0.5)
    qo = np.arange(B + 1, dtype=np.int32)
    qp = (n * wl.block - 1).astype(np.int32)
    sel, pool = csa.csa_index_topk_pool(cache, dev(q_full), dev(w_full), dev(qo), dev(qp), k, pool_group=G,
                                        pool_blocks=P)
    sel_re = csa.csa_index_topk_reindex(cache, dev(q_re), dev(w_re), dev(qo), dev(qp), k, pool, pool_group=G)
    assert csa.csa_read_device_status(cache) == 0
    sel, pool, sel_re = host(sel), host(pool), host(sel_re)
    one = np.array([0, 1], np.int32)
    for b in sample:
        kx = host_keys[b][None]
        nb = n[b:b + 1].astype(np.int32)
        s_full, n_vis = oracle.index_scores(kx, nb, one, qp[b:b + 1], q_full[b:b + 1], w_full[b:b + 1], m=wl.block,
                                            idx_dtype=1)
        parity.check_topk(sel[b:b + 1], oracle.topk(s_full, n_vis, k), s_full, n_vis, k)
        bmax, nbk = block_max_rows(s_full, n_vis, G)
        parity.check_topk(pool[b:b + 1], oracle.index_pool(s_full, n_vis, G=G, P=P), bmax, nbk, P)
        s_re, _ = oracle.index_scores(kx, nb, one, qp[b:b + 1], q_re[b:b + 1], w_re[b:b + 1], m=wl.block,
                                      idx_dtype=1)
        ref_re = oracle.reindex_topk(s_re, n_vis, pool[b:b + 1], G=G, k=k)
        check_reindex(sel_re[b:b + 1], ref_re, s_re, n_vis, pool[b:b + 1], G, k)


def test_hca_b64_1m_sampled():
    import torch

    import fp4_kv_cache_csa_b200 as csa

    wl = datagen.WORKLOADS["hca_b64_1m"]
    B, D, H, W = wl.batch, wl.dim, wl.heads, wl.window
    cap = wl.ctx_max // wl.block
    f, s = datagen.random_cache_bytes(B * cap, D, 510, 0, scale_lo=119, scale_hi=122)
    f, s = f.reshape(B, cap, D // 2), s.reshape(B, cap, D // 32)
    cache = make_cache(f, s, np.full(B, cap, np.int32), wl.block)
    q = datagen.normal_bf16((B, H, D), 511, 1)
    win = datagen.normal_bf16((B * W, D), 511, 2)
    qo = np.arange(B + 1, dtype=np.int32)
    qp = np.full(B, wl.ctx_max - 1, np.int32)
    ws_, wl_ = (np.arange(B) * W).astype(np.int64), np.full(B, W, np.int32)
    out = host(csa.hca_decode_attend(cache, dev(q), dev(qo), dev(qp), dev(win), dev(ws_), dev(wl_)))
    assert csa.csa_read_device_status(cache) == 0
    one = np.array([0, 1], np.int32)
    for b in (0, 31, 63):
        ref, _ = oracle.hca_attend(f[b:b + 1], s[b:b + 1], np.array([cap], np.int32), one, qp[b:b + 1], q[b:b + 1],
                                   win[b * W:(b + 1) * W], np.array([0], np.int64), np.array([W], np.int32),
                                   D ** -0.5, m=wl.block)
        err, _ = parity.attention_row_error(out[b:b + 1], ref)
        assert err <= parity.ATT_TOL, (b, err)


@pytest.mark.parametrize("scale_fmt", [oracle.SCALE_E8M0_32, oracle.SCALE_E4M3_16])
def test_csa_b8_64k_from_tokens(scale_fmt):
    import torch

    import fp4_kv_cache_csa_b200 as csa

    wl = datagen.WORKLOADS["csa_b8_64k"]
    B, D, H, dI, m, k, W, T = wl.batch, wl.dim, wl.heads, wl.idx_dim, wl.block, wl.topk, wl.window, wl.ctx_max
    cap = T // m
    kv = datagen.normal_bf16((B * T, D), 520, 1, channel_lognormal=wl.channel_lognormal)
    it = datagen.normal_bf16((B * T, dI), 520, 2, channel_lognormal=wl.channel_lognormal)
    wg = datagen.normal_f32((D,), 520, 3, std=0.02)
    offs = (np.arange(B + 1) * T).astype(np.int32)
    ref = oracle.compress(kv, it, wg, offs, np.zeros(B, np.int32), m=m, cap=cap, scale_fmt=scale_fmt,
                          return_pooled=True)
    # stage 1: pooling + quantization of all 8 x 16384 blocks
    cache = csa.Cache.allocate(B, cap, D, m, dI, csa.CSA_IDX_BF16, scale_fmt=scale_fmt)
    csa.csa_compress_quantize(cache, dev(kv), dev(it), dev(wg), dev(offs))
    assert csa.csa_read_device_status(cache) == 0
    tol = parity.pooling_tolerance(kv, offs, np.zeros(B, np.int64), m, cap, kv_bits=kv, w_g=wg)
    parity.check_mxfp4(host(cache.fp4).reshape(B * cap, -1), host(cache.scale).reshape(B * cap, -1),
                       ref["fp4"].reshape(B * cap, -1), ref["scale"].reshape(B * cap, -1),
                       ref["pooled"].reshape(B * cap, D), tol=tol.reshape(B * cap, D), scale_fmt=scale_fmt)
    parity.check_keys(host(cache.idx_key).view(np.uint16), ref["idx_key"].view(np.uint16).reshape(B, cap, dI),
                      ref["pooled_idx"], "bf16", tol=parity.pooling_tolerance(it, offs, np.zeros(B, np.int64), m, cap, kv_bits=kv, w_g=wg))
    # stage 2: indexer + top-k on the oracle's cache
    ocache = make_cache(ref["fp4"], ref["scale"], ref["n_blocks"], m, ref["idx_key"].view(np.uint16), 0,
                        scale_fmt=scale_fmt)
    q = datagen.normal_bf16((B, H, D), 521, 1, channel_lognormal=wl.channel_lognormal)
    q_idx = datagen.normal_bf16((B, wl.idx_heads, dI), 521, 2, channel_lognormal=wl.channel_lognormal)
    w = datagen.normal_f32((B, wl.idx_heads), 521, 3, std=0.5)
    qo = np.arange(B + 1, dtype=np.int32)
    qp = np.full(B, T - 1, np.int32)
    sel_ref, scores, n_vis = oracle.index_topk(ref["idx_key"], ref["n_blocks"], qo, qp, q_idx, w, m=m, k=k)
    sel = host(csa.csa_index_topk(ocache, dev(q_idx), dev(w), dev(qo), dev(qp), k))
    near = parity.check_topk(sel, sel_ref, scores, n_vis, k)
    # stage 3: joint attention over the selection (the GPU's where the oracle has a near-tie) + window
    use = sel_ref.copy()
    use[near] = sel[near]
    win = np.concatenate([kv[b * T + T - W:b * T + T] for b in range(B)])
    ws_, wl_ = (np.arange(B) * W).astype(np.int64), np.full(B, W, np.int32)
    out = host(csa.csa_decode_attend(ocache, dev(q), dev(qo), dev(use), dev(win), dev(ws_), dev(wl_)))
    want, _ = oracle.csa_attend(ref["fp4"], ref["scale"], qo, q, use, win, ws_, wl_, D ** -0.5, scale_fmt=scale_fmt)
    err, _ = parity.attention_row_error(out, want)
    assert err <= parity.ATT_TOL, err
    assert csa.csa_read_device_status(ocache) == 0


def test_prefill_b4_8k_sampled():
    # prefill: 4 requests with 16384 cached blocks each (seeded bytes) receive 8192 new
    # tokens (2048 blocks); every new token is a query at its own position (causal at
    # block granularity), with the 128 raw tokens ending at it as its window
    import torch

    import fp4_kv_cache_csa_b200 as csa

    wl = datagen.WORKLOADS["prefill_b4_8k"]
    B, D, H, dI, m, k, W = wl.batch, wl.dim, wl.heads, wl.idx_dim, wl.block, wl.topk, wl.window
    T0, T1 = wl.ctx_min, wl.ctx_max
    n0, cap, NEW = T0 // m, T1 // m, T1 - T0
    f0, s0 = datagen.random_cache_bytes(B * n0, D, 540, 0)
    k0 = datagen.normal_bf16((B * n0, dI), 540, 1, std=0.5)
    kv = datagen.normal_bf16((B * NEW, D), 541, 1)
    it = datagen.normal_bf16((B * NEW, dI), 541, 2)
    wg = datagen.normal_f32((D,), 541, 3, std=0.02)
    offs = (np.arange(B + 1) * NEW).astype(np.int32)
    base = np.full(B, n0, np.int32)
    ref = oracle.compress(kv, it, wg, offs, base, m=m, cap=cap, return_pooled=True)
    # stage 1: the GPU appends the new blocks behind the cached ones
    fp4 = np.zeros((B, cap, D // 2), np.uint8)
    sc = np.zeros((B, cap, D // 32), np.uint8)
    keys = np.zeros((B, cap, dI), np.uint16)
    fp4[:, :n0], sc[:, :n0], keys[:, :n0] = (f0.reshape(B, n0, -1), s0.reshape(B, n0, -1),
                                             k0.reshape(B, n0, dI))
    cache = make_cache(fp4, sc, base, m, keys, 0)
    csa.csa_compress_quantize(cache, dev(kv), dev(it), dev(wg), dev(offs))
    assert csa.csa_read_device_status(cache) == 0
    assert np.array_equal(host(cache.n_blocks), ref["n_blocks"])
    new = slice(n0, cap)
    tol = parity.pooling_tolerance(kv, offs, base, m, cap, kv_bits=kv, w_g=wg)[:, new]
    parity.check_mxfp4(host(cache.fp4)[:, new].reshape(-1, D // 2), host(cache.scale)[:, new].reshape(-1, D // 32),
                       ref["fp4"][:, new].reshape(-1, D // 2), ref["scale"][:, new].reshape(-1, D // 32),
                       ref["pooled"][:, new].reshape(-1, D), tol=tol.reshape(-1, D))
    assert np.array_equal(host(cache.fp4)[:, :n0], fp4[:, :n0])  # cached blocks untouched
    parity.check_keys(host(cache.idx_key).view(np.uint16)[:, new], ref["idx_key"].view(np.uint16)[:, new],
                      ref["pooled_idx"][:, new], "bf16",
                      tol=parity.pooling_tolerance(it, offs, base, m, cap, kv_bits=kv, w_g=wg)[:, new])
    # stages 2 and 3 run on the oracle's new blocks behind the cached ones
    fp4[:, new], sc[:, new] = ref["fp4"][:, new], ref["scale"][:, new]
    keys[:, new] = ref["idx_key"].view(np.uint16)[:, new]
    ocache = make_cache(fp4, sc, ref["n_blocks"], m, keys, 0)
    Nq = B * NEW
    qo = (np.arange(B + 1) * NEW).astype(np.int32)
    qp = np.tile(np.arange(T0, T1, dtype=np.int32), B)
    q_idx = datagen.normal_bf16((Nq, wl.idx_heads, dI), 542, 1)
    w = datagen.normal_f32((Nq, wl.idx_heads), 542, 2, std=0.5)
    sel_d = csa.csa_index_topk(ocache, dev(q_idx), dev(w), dev(qo), dev(qp), k)
    # windows: the 127 raw tokens before the new ones (seeded) and the new tokens themselves
    tail = datagen.normal_bf16((B * (W - 1), D), 543, 1)
    rows = NEW + W - 1
    win = np.concatenate([np.concatenate([tail[b * (W - 1):(b + 1) * (W - 1)], kv[b * NEW:(b + 1) * NEW]])
                          for b in range(B)])
    ws_ = (np.arange(Nq) // NEW * rows + np.arange(Nq) % NEW).astype(np.int64)
    wl_ = np.full(Nq, W, np.int32)
    g = torch.Generator(device="cuda").manual_seed(544)
    q_d = torch.randn(Nq, H, D, generator=g, device="cuda").to(torch.bfloat16)
    out_d = csa.csa_decode_attend(ocache, q_d, dev(qo), sel_d, dev(win), dev(ws_), dev(wl_))
    assert csa.csa_read_device_status(ocache) == 0
    sel = host(sel_d)
    one = np.array([0, 1], np.int32)
    for b in range(B):
        for t in (0, 1, NEW // 2 - 1, NEW - 1):
            i = b * NEW + t
            sel_ref, scores, n_vis = oracle.index_topk(keys[b:b + 1].view(np.uint8), ref["n_blocks"][b:b + 1], one,
                                                       qp[i:i + 1], q_idx[i:i + 1], w[i:i + 1], m=m, k=k)
            assert n_vis[0] == (T0 + t + 1) // m
            parity.check_topk(sel[i:i + 1], sel_ref, scores, n_vis, k)  # the GPU's set is a valid top-k
            qi = host(q_d[i:i + 1])
            want, _ = oracle.csa_attend(fp4[b:b + 1], sc[b:b + 1], one, qi, sel[i:i + 1], win[b * rows:(b + 1) * rows],
                                        np.array([t], np.int64), np.array([W], np.int32), D ** -0.5)
            err, _ = parity.attention_row_error(host(out_d[i:i + 1]), want)
            assert err <= parity.ATT_TOL, (b, t, err)


def test_prefill_b4_8k_mxfp4_index_sampled():
    # the prefill_b4_8k indexer call with MXFP4 indexer keys (E2M1 codes, one E8M0 scale
    # per 32 channels): 32768 causal queries over 16384..18432 blocks per request score on
    # the block-scaled tensor-core GEMM; sampled queries are recomputed by the oracle
    import fp4_kv_cache_csa_b200 as csa

    wl = datagen.WORKLOADS["prefill_b4_8k"]
    B, D, dI, m, k = wl.batch, wl.dim, wl.idx_dim, wl.block, wl.topk
    T0, T1 = wl.ctx_min, wl.ctx_max
    cap, NEW = T1 // m, T1 - T0
    g = datagen.generator(545, 1)
    codes = g.integers(0, 256, size=(B, cap, dI // 2)).astype(np.uint8)
    scales = g.integers(122, 127, size=(B, cap, dI // 32)).astype(np.uint8)
    n_blocks = np.full(B, cap, np.int32)
    cache = make_cache(np.zeros((B, cap, D // 2), np.uint8), np.zeros((B, cap, D // 32), np.uint8), n_blocks, m,
                       codes, 2, idx_key_scale=scales)
    Nq = B * NEW
    qo = (np.arange(B + 1) * NEW).astype(np.int32)
    qp = np.tile(np.arange(T0, T1, dtype=np.int32), B)
    q_idx = datagen.normal_bf16((Nq, wl.idx_heads, dI), 546, 1)
    w = datagen.normal_f32((Nq, wl.idx_heads), 546, 2, std=0.5)
    sel = host(csa.csa_index_topk(cache, dev(q_idx), dev(w), dev(qo), dev(qp), k))
    assert csa.csa_read_device_status(cache) == 0
    one = np.array([0, 1], np.int32)
    for b in range(B):
        for t in (0, 1, NEW // 2 - 1, NEW - 1):
            i = b * NEW + t
            sel_ref, scores, n_vis = oracle.index_topk(codes[b:b + 1], n_blocks[b:b + 1], one, qp[i:i + 1],
                                                       q_idx[i:i + 1], w[i:i + 1], m=m, k=k,
                                                       idx_dtype=oracle.IDX_MXFP4, idx_key_scale=scales[b:b + 1])
            assert n_vis[0] == (T0 + t + 1) // m
            parity.check_topk(sel[i:i + 1], sel_ref, scores, n_vis, k)
