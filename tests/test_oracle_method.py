"""Pins for the oracle's pooling, indexer, top-k and attention.

Every check ties the oracle to something other than its own code: closed forms
(single entry, identical entries, a 1:3 softmax), invariants (m = 1 identity,
constant blocks, zero gate = mean, positive homogeneity, causal visibility),
a hand-computed worked example (tests/golden/indexer_tiny.txt), brute-force
subset enumeration, and special cases that reduce to textbook softmax attention
computed with scipy.
"""
import itertools
import math
import os

import numpy as np
import pytest
from scipy.special import softmax as sp_softmax

import oracle
from fp4_kv_cache_csa_b200 import datagen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(x):
    return datagen.to_bf16_bits(np.asarray(x, np.float32))


def bf16_val(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def lossless_tokens(n, D, seed):
    """Tokens whose every 32-group is exactly E2M1 x 2^X with amax in [4, 8) x 2^X,
    so MXFP4 stores them without loss (and bf16 holds them exactly)."""
    g = np.random.default_rng(seed)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    vals = g.choice(mags, size=(n, D)) * g.choice([-1.0, 1.0], size=(n, D))
    X = g.integers(-4, 2, size=(n, D // 32))
    vals = vals.reshape(n, D // 32, 32)
    vals[:, :, 0] = 4.0 * np.sign(vals[:, :, 0] + 0.5)
    vals = vals * np.ldexp(1.0, X)[:, :, None]
    return vals.reshape(n, D).astype(np.float32)


# ---------------------------------------------------------------- pooling

def _compress(kv_f32, w_g, m, idx_f32=None, idx_dtype=0):
    T, D = kv_f32.shape
    return oracle.compress(bf16(kv_f32), None if idx_f32 is None else bf16(idx_f32), np.asarray(w_g, np.float32),
                           np.array([0, T], np.int32), np.zeros(1, np.int32), m=m, cap=T // m,
                           idx_dtype=idx_dtype, return_pooled=True)


def test_pool_m1_is_identity_and_quantizes_the_token():
    g = np.random.default_rng(10)
    kv = g.standard_normal((64, 128)).astype(np.float32)
    idx = g.standard_normal((64, 64)).astype(np.float32)
    r = _compress(kv, g.standard_normal(128) * 0.02, 1, idx)
    tok = bf16_val(bf16(kv))
    assert np.array_equal(r["pooled"][0].astype(np.float64), tok)
    assert np.array_equal(r["idx_key"][0].view(np.uint16), bf16(idx))
    for j in range(64):
        for grp in range(4):
            codes, sb = oracle.mxfp4_quantize_group(tok[j, 32 * grp:32 * grp + 32].astype(np.float32))
            assert r["scale"][0, j, grp] == sb
            packed = codes[0::2] | (codes[1::2] << 4)
            assert np.array_equal(r["fp4"][0, j, 16 * grp:16 * grp + 16], packed)


def test_pool_constant_block_gives_the_token():
    g = np.random.default_rng(11)
    tok = g.standard_normal((8, 128)).astype(np.float32)
    kv = np.repeat(tok, 4, axis=0)  # each block of 4 holds one token 4 times
    r = _compress(kv, g.standard_normal(128), 4)
    assert np.array_equal(r["pooled"][0], bf16_val(bf16(tok)).astype(np.float32))


def test_pool_zero_gate_is_the_mean():
    g = np.random.default_rng(12)
    for m in (4, 128):
        kv = g.standard_normal((4 * m, 64)).astype(np.float32)
        r = _compress(kv, np.zeros(64), m)
        mean = bf16_val(bf16(kv)).reshape(4, m, 64).mean(axis=1)
        np.testing.assert_allclose(r["pooled"][0], mean.astype(np.float32), rtol=2 ** -23, atol=0)


def test_pool_dominant_gate_selects_the_token():
    # w_g picks channel 0; the token with a large channel-0 value takes all the weight
    kv = np.zeros((4, 32), np.float32)
    kv[:, 1:] = np.arange(4 * 31, dtype=np.float32).reshape(4, 31) / 8.0
    kv[2, 0] = 120.0
    w = np.zeros(32)
    w[0] = 1.0
    r = _compress(kv, w, 4)
    np.testing.assert_allclose(r["pooled"][0, 0], bf16_val(bf16(kv[2])), rtol=1e-40, atol=0)


def test_pool_one_to_three_gate():
    # gate logits 0 and ln 3 -> weights exactly 1/4 and 3/4 (w_g carries ln 3 on channel 0)
    kv = np.zeros((2, 32), np.float32)
    kv[1, 0] = 1.0
    kv[0, 1], kv[1, 1] = 8.0, 16.0
    w = np.zeros(32, np.float32)
    w[0] = np.float32(math.log(3.0))
    r = _compress(kv, w, 2)
    a = 1.0 / (1.0 + math.exp(float(w[0])))
    assert abs(a - 0.25) < 1e-7
    np.testing.assert_allclose(r["pooled"][0, 0, 1], 0.25 * 8 + 0.75 * 16, rtol=1e-6)
    np.testing.assert_allclose(r["pooled"][0, 0, 0], 0.75, rtol=1e-6)


# ---- the pooled indexer key (same gate weights as the main KV) at m > 1
#
# The main-KV closed forms above are repeated on the indexer-key plane, whose
# tokens are chosen independently of the main KV: the gate is a function of
# the main KV alone, so a key pooled with its own channels as gate input, a
# plain mean where the gate is not flat, or a key cast to E4M3 before pooling
# rather than after, each fails one of these.

def _e4m3_byte(x):
    """E4M3 byte of a float (RNE, saturating at +-448) from PyTorch's own cast."""
    import torch
    v = float(np.clip(x, -448.0, 448.0))
    return int(torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def _gated_block(m, logits_over_ln3, dI=32, seed=0):
    """One block of m tokens whose gate logits are c_t * ln 3 (w_g = ln 3 on main-KV channel 0,
    kv[t, 0] = c_t); the main KV's other channels are random, the indexer keys are set by the caller."""
    g = np.random.default_rng(seed)
    kv = g.standard_normal((m, 32)).astype(np.float32)
    kv[:, 0] = np.asarray(logits_over_ln3, np.float32)
    w = np.zeros(32, np.float32)
    w[0] = np.float32(math.log(3.0))
    return kv, w


@pytest.mark.parametrize("m", [2, 4, 128])
@pytest.mark.parametrize("idx_dtype", [0, 1])
def test_pool_key_one_to_three_gate(m, idx_dtype):
    # logits 0, ln 3, then -128 ln 3 for the rest: weights 1/4, 3/4 and ~1e-61 -> key 0.25 a + 0.75 b
    c = np.full(m, -128.0, np.float32)
    c[0], c[1] = 0.0, 1.0
    kv, w = _gated_block(m, c)
    idx = np.zeros((m, 32), np.float32)
    idx[0, :4] = [8.0, -2.0, 0.5, 40.0]
    idx[1, :4] = [16.0, 6.0, 0.5, 0.0]
    idx[2:, :4] = 1000.0  # gated away: any weight they kept would show
    r = _compress(kv, w, m, idx, idx_dtype=idx_dtype)
    want = np.zeros(32)
    want[:4] = [14.0, 4.0, 0.5, 10.0]
    np.testing.assert_allclose(r["pooled_idx"][0, 0], want, rtol=1e-6, atol=1e-30)
    key = r["idx_key"][0, 0]
    if idx_dtype == 0:
        assert np.array_equal(key.view(np.uint16), bf16(want))
    else:
        assert [int(b) for b in key[:4]] == [_e4m3_byte(v) for v in want[:4]]
        assert np.all(key[4:] == 0)


@pytest.mark.parametrize("m", [2, 4, 128])
@pytest.mark.parametrize("idx_dtype", [0, 1])
def test_pool_key_dominant_gate_selects_the_token(m, idx_dtype):
    g = np.random.default_rng(20 + m)
    c = np.full(m, -100.0, np.float32)
    hot = m // 2
    c[hot] = 20.0  # logit 20 ln 3 against -100 ln 3: the other weights are below 1e-57
    kv, w = _gated_block(m, c, seed=m)
    idx = g.standard_normal((m, 64)).astype(np.float32) * 4.0
    r = _compress(kv, w, m, idx, idx_dtype=idx_dtype)
    tok = bf16_val(bf16(idx[hot]))
    np.testing.assert_array_equal(r["pooled_idx"][0, 0].astype(np.float64), tok)
    key = r["idx_key"][0, 0]
    if idx_dtype == 0:
        assert np.array_equal(key.view(np.uint16), bf16(idx[hot]))
    else:
        assert [int(b) for b in key] == [_e4m3_byte(v) for v in tok]


@pytest.mark.parametrize("m", [2, 4, 128])
def test_pool_key_zero_gate_is_the_mean(m):
    g = np.random.default_rng(30 + m)
    kv = g.standard_normal((3 * m, 32)).astype(np.float32)
    idx = g.standard_normal((3 * m, 48)).astype(np.float32)
    r = _compress(kv, np.zeros(32), m, idx)
    mean = bf16_val(bf16(idx)).reshape(3, m, 48).mean(axis=1)
    np.testing.assert_allclose(r["pooled_idx"][0, :3], mean.astype(np.float32), rtol=2 ** -22, atol=1e-30)
    # the stored bf16 key is the RNE rounding of that float32 mean
    assert np.array_equal(r["idx_key"][0, :3].view(np.uint16), bf16(r["pooled_idx"][0, :3]))


def test_pool_key_e4m3_is_cast_after_pooling():
    # keys 0 and 1000 under a flat gate: the mean 500 saturates to 448; casting each token first
    # (0 and 448) would give 224
    kv = np.zeros((2, 32), np.float32)
    idx = np.zeros((2, 32), np.float32)
    idx[1, 0] = 1000.0
    idx[0, 1], idx[1, 1] = 3.0, 5.0  # mean 4 (E4M3 exact)
    r = _compress(kv, np.zeros(32), 2, idx, idx_dtype=1)
    key = r["idx_key"][0, 0]
    assert int(key[0]) == _e4m3_byte(448.0) == 0x7E
    assert int(key[1]) == _e4m3_byte(4.0)


@pytest.mark.parametrize("m", [2, 4, 128])
@pytest.mark.parametrize("idx_dtype", [0, 1])
def test_pool_key_constant_block_gives_the_token(m, idx_dtype):
    g = np.random.default_rng(40 + m)
    tok = g.standard_normal((3, 40)).astype(np.float32)
    idx = np.repeat(tok, m, axis=0)
    kv = g.standard_normal((3 * m, 32)).astype(np.float32)  # any gate: the weights sum to one
    r = _compress(kv, g.standard_normal(32), m, idx, idx_dtype=idx_dtype)
    tv = bf16_val(bf16(tok))
    np.testing.assert_allclose(r["pooled_idx"][0, :3].astype(np.float64), tv, rtol=2 ** -22, atol=0)
    key = r["idx_key"][0, :3]
    if idx_dtype == 0:
        assert np.array_equal(key.view(np.uint16), bf16(tok))
    else:
        assert [int(b) for b in key.reshape(-1)] == [_e4m3_byte(v) for v in tv.reshape(-1)]


def test_pool_token_order_within_block_does_not_matter():
    g = np.random.default_rng(13)
    kv = g.standard_normal((4, 256)).astype(np.float32)
    w = g.standard_normal(256) * 0.05
    a = _compress(kv, w, 4)["pooled"][0, 0]
    b = _compress(kv[[2, 0, 3, 1]], w, 4)["pooled"][0, 0]
    np.testing.assert_allclose(a, b, rtol=2 ** -22, atol=0)


def test_compress_appends_at_n_blocks_and_checks_counts():
    g = np.random.default_rng(14)
    kv = bf16(g.standard_normal((12, 64)))
    offs = np.array([0, 8, 12], np.int32)
    r = oracle.compress(kv, None, np.zeros(64, np.float32), offs, np.array([3, 0], np.int32), m=4, cap=8)
    assert list(r["n_blocks"]) == [5, 1] and r["status"] == 0
    assert np.all(r["scale"][0, :3] == 0) and np.any(r["scale"][0, 3:5] != 0)
    bad = oracle.compress(kv, None, np.zeros(64, np.float32), np.array([0, 6, 12], np.int32),
                          np.zeros(2, np.int32), m=4, cap=8)
    assert bad["status"] == -1 and list(bad["n_blocks"]) == [0, 0]


# ---------------------------------------------------------------- indexer + top-k

def _read_indexer_golden():
    spec = {"sel": {}}
    with open(os.path.join(GOLDEN, "indexer_tiny.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tag, rest = line.split(" ", 1)
            if tag == "sel":
                k, idx = rest.split(":")
                spec["sel"][int(k)] = [int(v) for v in idx.split()]
            elif tag in ("keys", "q"):
                spec[tag] = np.array([[float(v) for v in grp.split()] for grp in rest.split("|")])
            else:
                spec[tag] = np.array([float(v) for v in rest.split()])
    return spec


def test_indexer_worked_example():
    s = _read_indexer_golden()
    keys = bf16(s["keys"]).view(np.uint8).reshape(1, 6, 8)
    q_idx = bf16(s["q"])[None]
    w = s["w"].astype(np.float32)[None]
    scores, n_vis = oracle.index_scores(keys, np.array([6], np.int32), np.array([0, 1], np.int32),
                                        np.array([23], np.int32), q_idx, w, m=4)
    assert n_vis[0] == 6
    assert np.array_equal(scores[0], s["scores"].astype(np.float32))
    for k, want in s["sel"].items():
        assert list(oracle.topk(scores, n_vis, k)[0]) == want


def _read_mxfp4_golden():
    spec = {"sel": {}}
    with open(os.path.join(GOLDEN, "indexer_mxfp4_tiny.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tag, rest = line.split(" ", 1)
            if tag == "sel":
                k, idx = rest.split(":")
                spec["sel"][int(k)] = [int(v) for v in idx.split()]
            elif tag in ("qbits", "codes", "scales"):
                base = 16 if tag != "scales" else 10
                spec[tag] = [[[int(v, base) for v in grp.split()] for grp in item.split("|")]
                             for item in rest.split(";")]
            else:
                spec[tag] = np.array([float(v) for v in rest.split()])
    return spec


def _mxfp4_golden_inputs(s):
    """Query [1, 2, 64] bf16 bits, codes [1, 3, 32], scales [1, 3, 2] from the golden file
    (listed channels c0, c1 of group 0 and c32, c33 of group 1; all others zero)."""
    q = np.zeros((1, 2, 64), np.uint16)
    for h, (g0, g1) in enumerate(s["qbits"]):
        q[0, h, 0:2], q[0, h, 32:34] = g0, g1
    codes = np.zeros((1, 3, 32), np.uint8)
    for j, (g0, g1) in enumerate(s["codes"]):
        codes[0, j, 0] = g0[0] | (g0[1] << 4)
        codes[0, j, 16] = g1[0] | (g1[1] << 4)
    scales = np.array([[sc[0] for sc in s["scales"]]], np.uint8).reshape(1, 3, 2)
    return q, codes, scales


def test_indexer_mxfp4_worked_example():
    # MXFP4 keys and the query quantized the same way: hand-derived scores, exact
    s = _read_mxfp4_golden()
    q, codes, scales = _mxfp4_golden_inputs(s)
    w = s["w"].astype(np.float32)[None]
    args = (np.array([3], np.int32), np.array([0, 1], np.int32), np.array([11], np.int32))
    scores, n_vis = oracle.index_scores(codes, *args, q, w, m=4, idx_dtype=oracle.IDX_MXFP4, idx_key_scale=scales)
    assert n_vis[0] == 3
    assert np.array_equal(scores[0], s["scores"].astype(np.float32))
    for k, want in s["sel"].items():
        assert list(oracle.topk(scores, n_vis, k)[0]) == want


def _e2m1_value(code):
    mag = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0][code & 7]
    return -mag if code & 8 else mag


def test_indexer_mxfp4_equals_bf16_on_representable_values():
    # when the query is already MXFP4-representable (every 32-group holds E2M1 x 2^X with its
    # largest magnitude in [4, 8) x 2^X) its quantization is the identity, and MXFP4 keys hold
    # values that bf16 stores exactly: the MXFP4-mode scores must equal the bf16-mode scores of
    # the same values
    g = np.random.default_rng(50)
    B, cap, dI, H_I, Nq = 2, 40, 128, 4, 3
    codes = g.integers(0, 256, size=(B, cap, dI // 2)).astype(np.uint8)
    scales = g.integers(120, 131, size=(B, cap, dI // 32)).astype(np.uint8)
    lo, hi = codes & 0xF, codes >> 4
    elem = np.stack([lo, hi], axis=-1).reshape(B, cap, dI)
    vals = np.vectorize(_e2m1_value)(elem) * np.ldexp(1.0, np.repeat(scales.astype(int) - 127, 32, axis=-1))
    keys_bf16 = bf16(vals.astype(np.float32)).view(np.uint8).reshape(B, cap, 2 * dI)
    assert np.array_equal(bf16_val(bf16(vals.astype(np.float32))), vals)  # exact in bf16
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    qv = g.choice(mags, size=(Nq, H_I, dI)) * g.choice([-1.0, 1.0], size=(Nq, H_I, dI))
    qv = qv.reshape(Nq, H_I, dI // 32, 32)
    qv[..., 0] = 4.0 * np.sign(qv[..., 0] + 0.5)
    qv = (qv * np.ldexp(1.0, g.integers(-3, 3, size=(Nq, H_I, dI // 32)))[..., None]).reshape(Nq, H_I, dI)
    w = g.standard_normal((Nq, H_I)).astype(np.float32)
    args = (np.array([cap, 31], np.int32), np.array([0, 2, 3], np.int32), np.array([10 ** 5, 10 ** 5, 50], np.int32))
    s_mx, n1 = oracle.index_scores(codes, *args, bf16(qv), w, m=4, idx_dtype=oracle.IDX_MXFP4, idx_key_scale=scales)
    s_bf, n2 = oracle.index_scores(keys_bf16, *args, bf16(qv), w, m=4)
    assert np.array_equal(n1, n2) and list(n1) == [cap, cap, 12]
    assert np.array_equal(s_mx, s_bf)


def test_pool_m1_mxfp4_key_store():
    # m = 1: the stored MXFP4 key decodes to the token's value when the token is representable,
    # and otherwise to its quantization by the main KV's rule (the same codes and scale bytes
    # the main-KV plane gets for the same values)
    g = np.random.default_rng(51)
    T, dI = 16, 64
    kv = g.standard_normal((T, 64)).astype(np.float32)
    idx = g.standard_normal((T, dI)).astype(np.float32) * 3
    r = _compress(kv, np.zeros(64), 1, idx, idx_dtype=oracle.IDX_MXFP4)
    ref = _compress(idx, np.zeros(dI), 1)  # the same values through the main-KV plane
    assert np.array_equal(r["idx_key"][0], ref["fp4"][0])
    assert np.array_equal(r["idx_key_scale"][0], ref["scale"][0])
    lossless = lossless_tokens(T, dI, 52)
    r2 = _compress(kv, np.zeros(64), 1, lossless, idx_dtype=oracle.IDX_MXFP4)
    codes = r2["idx_key"][0]
    elem = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(T, dI)
    dec = np.vectorize(_e2m1_value)(elem) * np.ldexp(1.0, np.repeat(r2["idx_key_scale"][0].astype(int) - 127, 32, axis=-1))
    assert np.array_equal(dec, lossless.astype(np.float64))


def test_indexer_e4m3_keys_and_homogeneity():
    g = np.random.default_rng(20)
    keys = datagen.to_e4m3_bytes(g.standard_normal((1, 50, 32)) * 0.5)
    q = g.standard_normal((1, 3, 32)).astype(np.float32)
    w = np.abs(g.standard_normal((1, 3))).astype(np.float32)
    args = (keys, np.array([50], np.int32), np.array([0, 1], np.int32), np.array([10 ** 6], np.int32))
    s1, _ = oracle.index_scores(*args, bf16(q), w, m=4, idx_dtype=1)
    s2, _ = oracle.index_scores(*args, bf16(2 * q), w, m=4, idx_dtype=1)
    assert np.array_equal(2 * s1, s2)  # ReLU is positively homogeneous; x2 is exact
    assert np.all(s1 >= 0) and np.any(s1 == 0)  # w >= 0 -> no negative score; ReLU zeros occur


def test_indexer_causal_visibility():
    keys = np.zeros((1, 10, 8), np.uint8)
    for pos, n_filled, want in [(0, 10, 0), (3, 10, 1), (6, 10, 1), (7, 10, 2), (39, 10, 10), (1000, 7, 7), (1000, 0, 0)]:
        _, n_vis = oracle.index_scores(keys, np.array([n_filled], np.int32), np.array([0, 1], np.int32),
                                       np.array([pos], np.int32), np.zeros((1, 1, 4), np.uint16),
                                       np.ones((1, 1), np.float32), m=4)
        assert n_vis[0] == want, (pos, n_filled)


def test_topk_brute_force_subsets():
    g = np.random.default_rng(21)
    for trial in range(200):
        n = int(g.integers(1, 11))
        k = int(g.integers(1, 12))
        sc = g.integers(-3, 4, size=n).astype(np.float32)  # small integers: many exact ties
        best = None
        for sub in itertools.combinations(range(n), min(k, n)):
            key = (sum(sc[list(sub)]), tuple(-j for j in sub))
            if best is None or key > best[0]:
                best = (key, sub)
        want = list(best[1]) + [-1] * (k - min(k, n))
        got = oracle.topk(np.concatenate([sc, np.zeros(3, np.float32)])[None], np.array([n], np.int32), k)
        assert list(got[0]) == want, (sc, k)


def test_topk_empty_and_all():
    sc = np.array([[3, 1, 2]], np.float32)
    assert list(oracle.topk(sc, np.array([0], np.int32), 2)[0]) == [-1, -1]
    assert list(oracle.topk(sc, np.array([3], np.int32), 5)[0]) == [0, 1, 2, -1, -1]


# ---------------------------------------------------------------- attention

def _cache_from_rows(rows_f32):
    """Put lossless rows into an MXFP4 cache with m = 1 pooling."""
    n, D = rows_f32.shape
    r = oracle.compress(bf16(rows_f32), None, np.zeros(D, np.float32), np.array([0, n], np.int32),
                        np.zeros(1, np.int32), m=1, cap=n)
    deq = oracle.mxfp4_dequantize(r["fp4"][0], r["scale"][0])
    assert np.array_equal(deq, rows_f32.astype(np.float64))
    return r


def _textbook(q, x, scale):
    """softmax(scale * q x^T) x with scipy; q [H, D], x [n, D]."""
    logits = scale * q @ x.T
    p = sp_softmax(logits, axis=-1)
    lse = np.log(np.exp(logits - logits.max(-1, keepdims=True)).sum(-1)) + logits.max(-1)
    return p @ x, lse


def test_attend_single_entry_is_the_entry():
    rows = lossless_tokens(3, 64, 30)
    r = _cache_from_rows(rows)
    q = bf16(np.random.default_rng(31).standard_normal((1, 4, 64)))
    out, lse = oracle.csa_attend(r["fp4"], r["scale"], np.array([0, 1], np.int32), q,
                                 np.array([[2, -1]], np.int32), None, None, None, 0.125)
    assert np.array_equal(out[0], np.repeat(rows[2:3].astype(np.float64), 4, axis=0))
    np.testing.assert_allclose(lse[0], 0.125 * bf16_val(q[0]) @ rows[2].astype(np.float64), rtol=1e-13)


def test_attend_identical_entries_and_one_to_three_softmax():
    D = 32
    x1 = np.zeros(D, np.float32)
    x2 = np.zeros(D, np.float32)
    x1[1], x2[0], x2[1] = 4.0, 2.0, 1.0
    win = bf16(np.stack([x1, x2]))
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, 0] = 1.0
    scale = math.log(3.0) / 2.0  # logits 0 and ln 3 -> weights 1/4 and 3/4
    out, lse = oracle.csa_attend(np.zeros((1, 1, D // 2), np.uint8), np.zeros((1, 1, 1), np.uint8),
                                 np.array([0, 1], np.int32), bf16(q), np.full((1, 1), -1, np.int32),
                                 win, np.array([0], np.int64), np.array([2], np.int32), scale)
    np.testing.assert_allclose(out[0, 0], 0.25 * x1 + 0.75 * x2, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], math.log(4.0), rtol=1e-14)
    same = bf16(np.repeat(x2[None], 5, axis=0))
    out2, _ = oracle.csa_attend(np.zeros((1, 1, D // 2), np.uint8), np.zeros((1, 1, 1), np.uint8),
                                np.array([0, 1], np.int32), bf16(q), np.full((1, 1), -1, np.int32),
                                same, np.array([0], np.int64), np.array([5], np.int32), 0.7)
    np.testing.assert_allclose(out2[0, 0], x2, rtol=1e-14)


def test_attend_empty_set():
    out, lse = oracle.csa_attend(np.zeros((1, 4, 16), np.uint8), np.zeros((1, 4, 1), np.uint8),
                                 np.array([0, 1], np.int32), np.zeros((1, 2, 32), np.uint16),
                                 np.full((1, 3), -1, np.int32), None, None, None, 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_m1_lossless_dense_is_textbook_attention():
    # m = 1, values MXFP4 stores exactly, k >= n, no window -> textbook softmax attention
    n, D, H = 40, 128, 8
    rows = lossless_tokens(n, D, 32)
    r = _cache_from_rows(rows)
    g = np.random.default_rng(33)
    q = bf16(g.standard_normal((1, H, D)))
    sel = np.arange(n + 5, dtype=np.int32)
    sel[n:] = -1
    out, lse = oracle.csa_attend(r["fp4"], r["scale"], np.array([0, 1], np.int32), q, sel[None],
                                 None, None, None, 1 / math.sqrt(D))
    ref, ref_lse = _textbook(bf16_val(q[0]), rows.astype(np.float64), 1 / math.sqrt(D))
    np.testing.assert_allclose(out[0], ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse[0], ref_lse, rtol=1e-12)


def test_csa_with_k_at_least_n_equals_dense_hca():
    g = np.random.default_rng(34)
    D, H, m, T = 64, 4, 4, 96
    kv = g.standard_normal((T, D)).astype(np.float32)
    r = oracle.compress(bf16(kv), None, (g.standard_normal(D) * 0.02).astype(np.float32), np.array([0, T], np.int32),
                        np.zeros(1, np.int32), m=m, cap=T // m)
    q = bf16(g.standard_normal((1, H, D)))
    win = bf16(kv[-16:])
    ws, wl = np.array([0], np.int64), np.array([16], np.int32)
    sel = np.arange(T // m, dtype=np.int32)[None]
    a, la = oracle.csa_attend(r["fp4"], r["scale"], np.array([0, 1], np.int32), q, sel, win, ws, wl, 0.125)
    b, lb = oracle.hca_attend(r["fp4"], r["scale"], r["n_blocks"], np.array([0, 1], np.int32),
                              np.array([T - 1], np.int32), q, win, ws, wl, 0.125, m=m)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=1e-12)


def test_csa_brute_force_subset_then_textbook():
    # indexer + top-k + attention end to end on tiny inputs against a brute-force
    # choice of the best block subset and textbook attention over it
    g = np.random.default_rng(35)
    n, D, H, dI, HI, k, W = 9, 64, 2, 16, 2, 3, 4
    rows = lossless_tokens(n, D, 36)
    r = _cache_from_rows(rows)
    keys = datagen.to_e4m3_bytes(np.round(g.standard_normal((1, n, dI)) * 4) / 4)
    q_idx = bf16(np.round(g.standard_normal((1, HI, dI)) * 4) / 4)
    w = np.array([[1.0, 0.5]], np.float32)
    sel, scores, n_vis = oracle.index_topk(keys, np.array([n], np.int32), np.array([0, 1], np.int32),
                                           np.array([n - 1], np.int32), q_idx, w, m=1, k=k, idx_dtype=1)
    sc = scores[0, :n].astype(np.float64)
    best = max(itertools.combinations(range(n), k), key=lambda s: (sum(sc[list(s)]), tuple(-j for j in s)))
    assert list(sel[0]) == list(best)
    win_rows = g.standard_normal((W, D)).astype(np.float32)
    q = bf16(g.standard_normal((1, H, D)))
    out, _ = oracle.csa_attend(r["fp4"], r["scale"], np.array([0, 1], np.int32), q, sel, bf16(win_rows),
                               np.array([0], np.int64), np.array([W], np.int32), 0.2)
    x = np.concatenate([rows[list(best)].astype(np.float64), bf16_val(bf16(win_rows))])
    ref, _ = _textbook(bf16_val(q[0]), x, 0.2)
    np.testing.assert_allclose(out[0], ref, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- E4M3 scale per 16 elements

def lossless_tokens_e4m3x16(n, D, seed):
    """Tokens whose every 16-group is exactly E2M1 x s with amax = 6 s for an E4M3
    scale s, so the E4M3-per-16 format stores them without loss."""
    g = np.random.default_rng(seed)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    vals = g.choice(mags, size=(n, D // 16, 16)) * g.choice([-1.0, 1.0], size=(n, D // 16, 16))
    vals[:, :, 3] = np.where(vals[:, :, 3] < 0, -6.0, 6.0)
    s_codes = g.integers(0x20, 0x48, size=(n, D // 16))  # E4M3 scales 2^-3 .. 2^2 * 1.875
    s = np.array([[oracle.e4m3_decode(int(c)) for c in row] for row in s_codes])
    return (vals * s[:, :, None]).reshape(n, D).astype(np.float32)


def test_pool_m1_quantizes_the_token_e4m3x16():
    g = np.random.default_rng(40)
    kv = g.standard_normal((32, 128)).astype(np.float32)
    r = oracle.compress(bf16(kv), None, np.zeros(128, np.float32), np.array([0, 32], np.int32),
                        np.zeros(1, np.int32), m=1, cap=32, scale_fmt=oracle.SCALE_E4M3_16, return_pooled=True)
    tok = bf16_val(bf16(kv))
    assert r["scale"].shape == (1, 32, 8)
    for j in range(32):
        for grp in range(8):
            codes, sb = oracle.e4m3x16_quantize_group(tok[j, 16 * grp:16 * grp + 16].astype(np.float32))
            assert r["scale"][0, j, grp] == sb
            assert np.array_equal(r["fp4"][0, j, 8 * grp:8 * grp + 8], codes[0::2] | (codes[1::2] << 4))


def test_e4m3x16_lossless_dense_is_textbook_attention():
    n, D, H = 24, 128, 4
    rows = lossless_tokens_e4m3x16(n, D, 41)
    r = oracle.compress(bf16(rows), None, np.zeros(D, np.float32), np.array([0, n], np.int32),
                        np.zeros(1, np.int32), m=1, cap=n, scale_fmt=oracle.SCALE_E4M3_16)
    assert np.array_equal(oracle.fp4_dequantize(r["fp4"][0], r["scale"][0], oracle.SCALE_E4M3_16),
                          rows.astype(np.float64))
    g = np.random.default_rng(42)
    q = bf16(g.standard_normal((1, H, D)))
    sel = np.arange(n, dtype=np.int32)[None]
    out, lse = oracle.csa_attend(r["fp4"], r["scale"], np.array([0, 1], np.int32), q, sel, None, None, None,
                                 1 / math.sqrt(D), scale_fmt=oracle.SCALE_E4M3_16)
    ref, ref_lse = _textbook(bf16_val(q[0]), rows.astype(np.float64), 1 / math.sqrt(D))
    np.testing.assert_allclose(out[0], ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse[0], ref_lse, rtol=1e-12)
    hout, hlse = oracle.hca_attend(r["fp4"], r["scale"], r["n_blocks"], np.array([0, 1], np.int32),
                                   np.array([n - 1], np.int32), q, None, None, None, 1 / math.sqrt(D), m=1,
                                   scale_fmt=oracle.SCALE_E4M3_16)
    np.testing.assert_allclose(hout, out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(hlse, lse, rtol=1e-12)


def test_e4m3x16_is_finer_than_e8m0x32_on_gaussian_blocks():
    # the per-16 E4M3 scale tracks each group's magnitude more closely than a
    # power-of-two per-32 scale: its mean squared error is lower on N(0,1) rows
    g = np.random.default_rng(43)
    kv = g.standard_normal((256, 128)).astype(np.float32)
    tok = bf16_val(bf16(kv))
    err = {}
    for fmt in (oracle.SCALE_E8M0_32, oracle.SCALE_E4M3_16):
        r = oracle.compress(bf16(kv), None, np.zeros(128, np.float32), np.array([0, 256], np.int32),
                            np.zeros(1, np.int32), m=1, cap=256, scale_fmt=fmt)
        err[fmt] = np.mean((oracle.fp4_dequantize(r["fp4"][0], r["scale"][0], fmt) - tok) ** 2)
    assert err[oracle.SCALE_E4M3_16] < err[oracle.SCALE_E8M0_32]


# ---------------------------------------------------------------- hierarchical pool and Reindex

def _read_pool_golden():
    rows = []
    with open(os.path.join(GOLDEN, "pool_reindex_tiny.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.split() for p in line.split("|")]
            rows.append((int(parts[0][0]), np.array(parts[1], np.float32), np.array(parts[2], np.float32),
                         [int(x) for x in parts[3]], [int(x) for x in parts[4]], [int(x) for x in parts[5]]))
    return rows


def test_pool_and_reindex_golden():
    for n, full, re, pool_want, k3, k5 in _read_pool_golden():
        pool = oracle.index_pool(full[None], [n], G=4, P=2)
        assert list(pool[0]) == pool_want
        assert list(oracle.reindex_topk(re[None], [n], pool, G=4, k=3)[0]) == k3
        assert list(oracle.reindex_topk(re[None], [n], pool, G=4, k=5)[0]) == k5


def test_pool_brute_force_subsets():
    # the kept set maximises the sum of block maxima, ties broken towards lower block ids
    g = np.random.default_rng(50)
    for trial in range(60):
        n = int(g.integers(1, 30))
        G = int(g.choice([1, 2, 3, 4, 8]))
        P = int(g.integers(1, 6))
        sc = (g.integers(-3, 4, size=32)).astype(np.float32)  # many ties
        pool = oracle.index_pool(sc[None], [n], G=G, P=P)[0]
        nb = (n + G - 1) // G
        bmax = [max(sc[G * b:min(G * b + G, n)]) for b in range(nb)]
        take = min(P, nb)
        best = max(itertools.combinations(range(nb), take),
                   key=lambda s: (sum(bmax[b] for b in s), tuple(-b for b in s)))
        assert list(pool[:take]) == list(best)
        assert all(x == -1 for x in pool[take:])


def test_reindex_brute_force_subsets():
    g = np.random.default_rng(51)
    for trial in range(60):
        n, G, P = int(g.integers(1, 24)), int(g.choice([2, 4])), int(g.integers(1, 5))
        k = int(g.integers(1, 6))
        full = g.integers(-3, 4, size=24).astype(np.float32)
        re = g.integers(-3, 4, size=24).astype(np.float32)
        pool = oracle.index_pool(full[None], [n], G=G, P=P)
        sel = oracle.reindex_topk(re[None], [n], pool, G=G, k=k)[0]
        cand = sorted(j for b in pool[0] if b >= 0 for j in range(G * b, min(G * b + G, n)))
        take = min(k, len(cand))
        best = max(itertools.combinations(cand, take), key=lambda s: (sum(re[j] for j in s), tuple(-j for j in s)))
        assert list(sel[:take]) == list(best)
        assert all(x == -1 for x in sel[take:])


def test_reindex_with_the_whole_context_pooled_is_the_full_topk():
    # when the pool covers every visible entry, Reindex is the plain top-k of its scores
    g = np.random.default_rng(52)
    sc = g.standard_normal((3, 200)).astype(np.float32)
    n_vis = np.array([200, 137, 9], np.int32)
    pool = oracle.index_pool(g.standard_normal((3, 200)).astype(np.float32), n_vis, G=8, P=25)
    for k in (1, 16, 64):
        assert np.array_equal(oracle.reindex_topk(sc, n_vis, pool, G=8, k=k), oracle.topk(sc, n_vis, k))


def test_pool_with_single_entry_blocks_is_the_topk():
    g = np.random.default_rng(53)
    sc = np.round(g.standard_normal((4, 100)) * 3).astype(np.float32)
    n_vis = np.array([100, 50, 7, 0], np.int32)
    assert np.array_equal(oracle.index_pool(sc, n_vis, G=1, P=10), oracle.topk(sc, n_vis, 10))
