"""Comparison rules between the CUDA path and the oracle (shared by the GPU tests).

Bytes and indices are compared exactly. The only allowed differences are the
near-ties where both sides legitimately round differently because the GPU
accumulates in float32 in another order than the oracle's double precision:

* MXFP4 element code: the oracle's scaled value v * 2^-X lies within
  1e-5 relative (floor 4e-6) of an E2M1 rounding midpoint, or within the GPU's
  float32 pooling error bound tol (pooling_tolerance below: a forward error
  bound of the kernel's float32 arithmetic, in value units, proportional to
  the largest |token| pooled into that element -- the pooled value is a
  weighted sum whose rounding error scales with its terms, not with the
  result); the GPU code must then be one of the two neighbouring codes.
* The sign of a zero code (0x0 / 0x8) follows the sign of a value that rounds to
  zero magnitude; it may differ where the oracle's value is within that same
  bound of 0.
* MXFP4 scale byte: the oracle's float32 group amax lies within 1e-5 relative of
  a power of two (E8M0 per 32), or amax / 6 lies within 1e-5 relative of the
  midpoint of the two E4M3 scales (E4M3 per 16); the GPU group must then be a
  correct quantization of the oracle's pooled values with the GPU's scale
  (same near-midpoint rule).
* E4M3-per-16 codes: as for MXFP4, with the scaled value v / s.
* BF16 / E4M3 indexer keys: the oracle's float32 value lies within 1e-5 relative
  of a rounding midpoint of the format; the GPU byte must be a neighbour.
* top-k: where the oracle's k-th and (k+1)-th scores differ by less than 1e-5
  relative, the GPU's set only has to be a valid top-k of the oracle's scores
  within that tolerance (attention is then checked on the GPU's own set).
Such exceptions must stay rare (the tests bound their count).

Attention outputs: per (query, head) row, max_d |gpu - ref| / max_d |ref| <= 2e-3.
"""
import math

import numpy as np

import oracle

REL = 1e-5
E2M1_MID = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
ATT_TOL = 2e-3
U32 = 2.0 ** -24        # float32 unit roundoff
EXPF_REL = 2.0 ** -22   # expf: at most 2 ulp (CUDA's stated bound)


def _gamma(n):
    return n * U32 / (1.0 - n * U32)


def pooling_coefficient(S_max, m, D):
    """Relative forward error bound (times max_t |x_t|) of the kernel's float32 gated pooling.

    The kernel (one warp per block; lane l holds E = D/32 channels) computes
      g_t = sum_d kv_t[d] w_g[d]   an FMA chain of E terms per lane, then a 5-level butterfly,
      p_t = expf(g_t - mu), den = sum_t p_t, acc = sum_t p_t x_t (online: rescaled by
      expf(mu_old - mu) whenever the running max rises), e = acc / den;
    with m >= 32 up to 16 warps each pool a slice of the tokens and their states are merged
    with expf(mu_w - M) factors. Against the exact e = sum_t alpha_t x_t:
      * logit error |dg_t| <= gamma(E + 5) * S_t, S_t = sum_d |kv_t[d] w_g[d]|; an error common
        to all t cancels in the ratio, so p_t carries a relative error
        eps_t <= gamma(E + 5) S_max + EXPF_REL + U32 |g_t - mu| (the argument's rounding);
      * perturbing every p_t by (1 + eps_t) moves e by at most 2 max|x| sum_t alpha_t |eps_t|,
        and alpha_t U32 |g_t - mu| <= U32 / e since alpha_t <= exp(g_t - mu);
      * the sums acc and den of m terms: gamma(m) each; the rescales multiply acc and den by
        the same rounded factor (its error cancels), adding one rounding per rescale, at most
        m: gamma(m) each; the warp merge: one expf per warp (2 EXPF_REL spread) and a 16-term
        sum (gamma(17) for acc and den); the division, and the oracle's own float32 rounding
        of its double result: U32 each.
    """
    E = max(D // 32, 1)
    return (2.0 * (_gamma(E + 5) * S_max + EXPF_REL + m * U32 / math.e) + 4.0 * _gamma(m)
            + 2.0 * EXPF_REL + 2.0 * _gamma(17) + 2.0 * U32)


def pooling_tolerance(tok_bits, offsets, n_blocks_before, m, cap, *, kv_bits, w_g):
    """[B, cap, C] bound on the GPU's pooled-value error for the tokens tok_bits (the main KV or
    the indexer keys, pooled with the gate computed from kv_bits and w_g):
    pooling_coefficient(block's max S_t) * max |token| over each block's tokens, per channel."""
    x = np.abs((np.asarray(tok_bits, np.uint32) << 16).view(np.float32)).astype(np.float64)
    kv = (np.asarray(kv_bits, np.uint32) << 16).view(np.float32).astype(np.float64)
    D = kv.shape[1]
    S = np.abs(kv) @ np.abs(np.asarray(w_g, np.float64))
    B = len(offsets) - 1
    out = np.zeros((B, cap, x.shape[1]), np.float64)
    for b in range(B):
        t0, t1 = int(offsets[b]), int(offsets[b + 1])
        nb = (t1 - t0) // m
        if nb:
            blk = x[t0:t0 + nb * m].reshape(nb, m, -1).max(axis=1)
            smax = S[t0:t0 + nb * m].reshape(nb, m).max(axis=1)
            coef = np.array([pooling_coefficient(s, m, D) for s in smax])
            out[b, n_blocks_before[b]:n_blocks_before[b] + nb] = coef[:, None] * blk
    return out


# near-tie exceptions used by the byte comparisons of the running test session,
# reported in the terminal summary (tests/conftest.py)
EXCEPTIONS = []


def record(kind, count, total):
    import os
    EXCEPTIONS.append((os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], kind, int(count), int(total)))


def unpack_codes(fp4):
    fp4 = np.asarray(fp4, np.uint8)
    return np.stack([fp4 & 0xF, fp4 >> 4], axis=-1).reshape(*fp4.shape[:-1], fp4.shape[-1] * 2)


def near_e2m1_midpoint(s, tol_scaled=0.0):
    """Within tolerance of an E2M1 rounding midpoint, or of 0 (where the sign bit of a value that
    rounds to zero magnitude is decided: codes 0x0 and 0x8)."""
    a = np.abs(s)
    d = np.min(np.abs(a[..., None] - E2M1_MID), axis=-1)
    nearest_mid = E2M1_MID[np.argmin(np.abs(a[..., None] - E2M1_MID), axis=-1)]
    near_mid = d <= np.maximum(np.maximum(REL * nearest_mid, 4e-6), tol_scaled)
    near_zero = a <= np.maximum(4e-6, tol_scaled)
    return near_mid | near_zero


def e2m1_neighbours(c1, c2):
    c1 = c1.astype(np.int32)
    c2 = c2.astype(np.int32)
    same_sign = (c1 & 8) == (c2 & 8)
    both_zero = ((c1 & 7) == 0) & ((c2 & 7) == 0)
    return (same_sign & (np.abs((c1 & 7) - (c2 & 7)) <= 1)) | both_zero | \
        (((c1 & 7) <= 1) & ((c2 & 7) <= 1))


def _scale_values(scale_bytes, scale_fmt):
    """Decoded scale of every group: 2^(byte-127) (E8M0) or the E4M3 value."""
    b = np.asarray(scale_bytes).astype(np.int64)
    if scale_fmt == oracle.SCALE_E8M0_32:
        return np.ldexp(1.0, b - 127)
    table = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float64)
    return table[b]


def _scale_near_tie(amax, gpu_byte, orc_byte, scale_fmt, gtol):
    """Whether a differing scale byte is a near-tie of the scale rule on the oracle's group amax."""
    if scale_fmt == oracle.SCALE_E8M0_32:
        lo_p, hi_p = 2.0 ** math.floor(math.log2(amax)), 2.0 ** math.ceil(math.log2(amax))
        return min(abs(amax - lo_p), abs(amax - hi_p)) <= max(REL * amax, gtol)
    # E4M3 of amax / 6: two neighbouring scale codes, the ratio near their midpoint
    if abs(int(gpu_byte) - int(orc_byte)) != 1 or max(int(gpu_byte), int(orc_byte)) > 0x7E:
        return False
    mid = 0.5 * (oracle.e4m3_decode(int(gpu_byte)) + oracle.e4m3_decode(int(orc_byte)))
    return abs(amax / 6.0 - mid) <= max(REL * mid, gtol / 6.0)


def check_mxfp4(gpu_fp4, gpu_scale, orc_fp4, orc_scale, pooled, strict=False, max_frac=1e-3, tol=None,
                scale_fmt=oracle.SCALE_E8M0_32):
    """Compare FP4 planes [n, D/2], [n, D/G] (G = 32 for E8M0 scales, 16 for E4M3) against the
    oracle's bytes and float32 pooled values [n, D]. tol: optional [n, D] absolute error bound of
    the GPU's pooled values."""
    gpu_fp4, gpu_scale = np.asarray(gpu_fp4), np.asarray(gpu_scale)
    if strict:
        assert np.array_equal(gpu_scale, orc_scale), "scale bytes differ (strict)"
        assert np.array_equal(gpu_fp4, orc_fp4), "codes differ (strict)"
        return 0
    G = oracle.group_size(scale_fmt)
    n, D = pooled.shape
    gc, oc = unpack_codes(gpu_fp4), unpack_codes(orc_fp4)
    exceptions = 0
    bad_scale = np.argwhere(gpu_scale != orc_scale)
    pooled64 = pooled.astype(np.float64)
    for r, g in bad_scale:
        grp = pooled[r, G * g:G * g + G]
        amax = float(np.max(np.abs(grp)))
        assert amax > 0
        gtol = 0.0 if tol is None else float(np.max(tol[r, G * g:G * g + G]))
        assert _scale_near_tie(amax, gpu_scale[r, g], orc_scale[r, g], scale_fmt, gtol), \
            f"scale byte differs at row {r} group {g} (amax {amax})"
        sv = float(_scale_values(gpu_scale[r, g], scale_fmt))
        assert sv > 0
        s = pooled64[r, G * g:G * g + G] / sv
        ts = 0.0 if tol is None else tol[r, G * g:G * g + G].astype(np.float64) / sv
        want = np.array([oracle.e2m1_encode(float(v)) for v in np.clip(s, -1e9, 1e9)])
        got = gc[r, G * g:G * g + G]
        ok = (got == want) | (near_e2m1_midpoint(s, ts) & e2m1_neighbours(got, want))
        assert ok.all(), f"group ({r},{g}) with the GPU scale is not a valid quantization"
        oc[r, G * g:G * g + G] = got
        exceptions += 1
    diff = np.argwhere(gc != oc)
    if len(diff):
        sv = _scale_values(orc_scale, scale_fmt).repeat(G, axis=-1)
        rr, dd = diff[:, 0], diff[:, 1]
        svd = sv[rr, dd]
        # a zero scale stores every element as a zero magnitude: only the sign can differ
        s = np.where(svd > 0, pooled64[rr, dd] / np.where(svd > 0, svd, 1.0), 0.0)
        ts = 0.0 if tol is None else tol[rr, dd].astype(np.float64) / np.where(svd > 0, svd, 1.0)
        ok = near_e2m1_midpoint(s, ts) & e2m1_neighbours(gc[rr, dd], oc[rr, dd])
        assert ok.all(), f"{(~ok).sum()} codes differ away from a rounding midpoint, e.g. {diff[~ok][:5]}"
        exceptions += len(diff)
    assert exceptions <= max(4, max_frac * gc.size), f"too many near-tie exceptions: {exceptions}"
    record("fp4 codes/scales", exceptions, gc.size)
    return exceptions


def check_keys(gpu_keys, orc_keys, pooled_keys, dtype, max_frac=1e-3, tol=None):
    """Indexer keys: bf16 (uint16 view) or e4m3 (uint8) against the oracle's, near-ties allowed
    (within 1e-5 relative of a rounding midpoint, or within tol: the GPU's pooling error bound)."""
    gpu_keys, orc_keys = np.asarray(gpu_keys), np.asarray(orc_keys)
    diff = np.argwhere(gpu_keys != orc_keys)
    record(f"{dtype} keys", len(diff), gpu_keys.size)
    if not len(diff):
        return 0
    vals = pooled_keys[tuple(diff.T)].astype(np.float64)
    tols = np.zeros(len(vals)) if tol is None else tol[tuple(diff.T)].astype(np.float64)
    for v, g, o, tv in zip(vals, gpu_keys[tuple(diff.T)], orc_keys[tuple(diff.T)], tols):
        if dtype == "bf16":
            dec = lambda b: oracle.bf16_decode(int(b))
        else:
            dec = lambda b: oracle.e4m3_decode(int(b))
        a, b = dec(g), dec(o)
        mid = 0.5 * (a + b)
        assert abs(v - mid) <= max(REL * max(abs(mid), 1e-30), tv), \
            f"key byte differs away from a midpoint: v={v} gpu={a} orc={b}"
    assert len(diff) <= max(4, max_frac * gpu_keys.size)
    return len(diff)


def check_topk(gpu_sel, orc_sel, scores, n_vis, k):
    """Exact match per query unless the oracle's k-th/(k+1)-th scores are a near-tie; then the GPU set
    must be a valid top-k of the oracle scores within the tolerance. Returns the near-tie query ids."""
    gpu_sel, orc_sel = np.asarray(gpu_sel), np.asarray(orc_sel)
    near = []
    for i in range(gpu_sel.shape[0]):
        if np.array_equal(gpu_sel[i], orc_sel[i]):
            continue
        n = int(n_vis[i])
        K = min(k, n)
        s = scores[i, :n].astype(np.float64)
        order = np.lexsort((np.arange(n), -s))
        kth, nxt = s[order[K - 1]], s[order[K]] if K < n else -np.inf
        tol = REL * max(abs(kth), 1e-30)
        assert abs(kth - nxt) < tol, f"query {i}: top-k differs without a near-tie ({kth} vs {nxt})"
        g = gpu_sel[i]
        assert np.all(g[K:] == -1) and np.all(np.diff(g[:K]) > 0) and g[0] >= 0 and g[K - 1] < n
        chosen = np.zeros(n, bool)
        chosen[g[:K]] = True
        assert s[chosen].min() >= kth - tol and (not (~chosen).any() or s[~chosen].max() <= kth + tol)
        near.append(i)
    return near


def attention_row_error(gpu_out, ref_out):
    """max over rows of max_d |gpu - ref| / max_d |ref| (rows with ref == 0 compare absolutely)."""
    g = np.asarray(gpu_out, np.float64)
    r = np.asarray(ref_out, np.float64)
    num = np.max(np.abs(g - r), axis=-1)
    den = np.max(np.abs(r), axis=-1)
    err = np.where(den > 0, num / np.where(den > 0, den, 1), num)
    return float(err.max()), err
