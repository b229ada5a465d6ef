"""Pins for the oracle's number formats (MXFP4 = E2M1 + E8M0/32, E4M3, BF16).

Each check compares the oracle with something other than itself: the bit-level
definition of the format written out here, hand-derived rounding cases in
tests/golden, PyTorch's own casts, or an error bound.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            rows.append((float(a), int(b, 0)))
    return rows


def e2m1_by_bits(code):
    """E2M1 from its bit fields: s | ee | m, exponent bias 1, subnormal when ee == 0."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = (m / 2.0) if e == 0 else (2.0 ** (e - 1)) * (1 + m / 2.0)
    return -mag if s else mag


def test_e2m1_decode_all_codes():
    for c in range(16):
        assert oracle.e2m1_decode(c) == e2m1_by_bits(c)
    assert sorted({abs(e2m1_by_bits(c)) for c in range(16)}) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_encode_roundtrip_every_code():
    for c in range(16):
        v = e2m1_by_bits(c)
        if c == 0x8:  # -0.0: sign is kept
            assert oracle.e2m1_encode(-0.0) == 0x8
            continue
        assert oracle.e2m1_encode(v) == c


def test_e2m1_rne_golden():
    for x, code in _read_golden("e2m1_rounding.txt"):
        assert oracle.e2m1_encode(x) == code, x


def test_e2m1_nearest_property():
    # brute force: the chosen code is a nearest magnitude, and on a tie its mantissa bit is 0
    g = np.random.default_rng(1)
    for x in np.concatenate([g.uniform(-8, 8, 2000), np.arange(-7, 7.01, 0.125)]):
        c = oracle.e2m1_encode(float(x))
        d = abs(abs(x) - abs(e2m1_by_bits(c)))
        best = min(abs(abs(x) - abs(e2m1_by_bits(k))) for k in range(8))
        assert d == best
        ties = [k for k in range(8) if abs(abs(x) - abs(e2m1_by_bits(k))) == best]
        if len(ties) > 1:
            assert (c & 1) == 0


def test_mxfp4_scale_golden():
    for amax, byte in _read_golden("mxfp4_scale.txt"):
        v = np.zeros(32, np.float32)
        v[7] = np.float32(amax)
        _, sb = oracle.mxfp4_quantize_group(v)
        assert sb == byte, amax


def test_mxfp4_roundtrip_exhaustive():
    # every code x every scale byte whose values fit float32: quantizing an
    # exactly representable block gives back the same codes and scale
    for sb in range(0, 253):
        X = sb - 127
        codes = np.arange(32) % 16
        v = np.array([math.ldexp(e2m1_by_bits(int(c)), X) for c in codes], np.float64)
        v[0] = math.ldexp(4.0, X)  # pins amax to [4, 8) * 2^X -> byte sb
        v32 = v.astype(np.float32)
        assert np.all(v32.astype(np.float64) == v)
        got, gsb = oracle.mxfp4_quantize_group(v32)
        assert gsb == sb
        want = codes.copy()
        want[0] = 0x6
        # -0 inputs (code 8) come back as 0x8 too: the sign is kept
        assert np.array_equal(got, want.astype(np.uint8)), sb


def test_mxfp4_error_bound():
    # |dequant - v| <= half the E2M1 spacing at |v|, times 2^X; values above 6*2^X saturate
    g = np.random.default_rng(2)
    for trial in range(300):
        v = (g.standard_normal(32) * 10.0 ** g.uniform(-6, 6)).astype(np.float32)
        codes, sb = oracle.mxfp4_quantize_group(v)
        X = sb - 127
        deq = np.array([math.ldexp(e2m1_by_bits(int(c)), X) for c in codes])
        for x, y in zip(v.astype(np.float64), deq):
            s = abs(x) / 2.0 ** X
            assert s < 8.0
            if s > 6.0:
                assert abs(y) == 6.0 * 2.0 ** X and np.sign(y) == np.sign(x)
                continue
            half_step = 0.25 if s <= 2.0 else 0.5 if s <= 4.0 else 1.0
            assert abs(y - x) <= half_step * 2.0 ** X * (1 + 1e-12)


def e4m3_by_bits(code):
    s, e, m = (code >> 7) & 1, (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return math.nan
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


def test_e4m3_decode_all_codes():
    for c in range(256):
        a, b = oracle.e4m3_decode(c), e4m3_by_bits(c)
        assert (math.isnan(a) and math.isnan(b)) or a == b
    assert e4m3_by_bits(0x7E) == 448.0


def test_e4m3_encode_matches_torch_in_range():
    g = np.random.default_rng(3)
    x = np.concatenate([g.standard_normal(20000) * 30, g.uniform(-448, 448, 5000),
                        g.standard_normal(2000) * 1e-2, np.array([0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10])])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_saturates():
    assert oracle.e4m3_encode(449.0) == 0x7E
    assert oracle.e4m3_encode(1e9) == 0x7E
    assert oracle.e4m3_encode(-1e9) == 0xFE
    # midpoint between 416 (1.101b * 2^8) and 448 (1.110b * 2^8) goes to the even mantissa
    assert oracle.e4m3_encode(432.0) == 0x7E
    assert oracle.e4m3_encode(400.0) == 0x7C  # midpoint of 384 (m=4) and 416 (m=5)


def test_bf16_encode_matches_torch():
    g = np.random.default_rng(4)
    x = np.concatenate([g.standard_normal(20000).astype(np.float32) * 10.0 ** g.uniform(-30, 30, 20000),
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], np.float64)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_encode(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, ref)
    for bits in g.integers(0, 0x7F80, 2000):
        assert oracle.bf16_decode(int(bits)) == float(np.array([int(bits) << 16], np.uint32).view(np.float32)[0])


# ---------------------------------------------------------------- E4M3 scale per 16 elements

def _read_groups(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            v, sb, codes = line.split("|")
            rows.append((np.array([float(x) for x in v.split()], np.float32), int(sb, 0),
                         np.array([int(c, 0) for c in codes.split()], np.uint8)))
    return rows


def test_e4m3x16_scale_golden():
    for amax, byte in _read_golden("e4m3x16_scale.txt"):
        for pos in (0, 9, 15):
            v = np.zeros(16, np.float32)
            v[pos] = np.float32(amax)
            _, sb = oracle.e4m3x16_quantize_group(v)
            assert sb == byte, amax
            v[pos] = -np.float32(amax)  # the sign of the largest element does not matter
            assert oracle.e4m3x16_quantize_group(v)[1] == byte, amax


def test_e4m3x16_group_golden():
    for v, sb, codes in _read_groups("e4m3x16_groups.txt"):
        got, gsb = oracle.e4m3x16_quantize_group(v)
        assert gsb == sb, v
        assert np.array_equal(got, codes), v


def test_e4m3x16_roundtrip_every_scale_and_code():
    # a group of exactly representable values E2M1(c) * s whose largest magnitude is
    # 6 s comes back with scale s and the same codes, for every positive finite s
    for sb in range(1, 0x7F):
        s = e4m3_by_bits(sb)
        codes = np.arange(16, dtype=np.uint8)
        v = np.array([e2m1_by_bits(int(c)) * s for c in codes], np.float64)
        assert np.all(v.astype(np.float32).astype(np.float64) == v)
        got, gsb = oracle.e4m3x16_quantize_group(v.astype(np.float32))
        assert gsb == sb
        assert np.array_equal(got, codes), sb  # includes -0 -> 0x8 and +-6 -> 0x7 / 0xF


def test_e4m3x16_brute_force_nearest():
    # scale: the nearest E4M3 value to amax / 6 among all 127 finite magnitudes
    # (ties to the even code, saturation at 448); codes: the nearest E2M1 value
    # to v / s, again by brute force over the 8 magnitudes
    mags = np.array([e4m3_by_bits(c) for c in range(0x7F)])
    e2 = np.array([e2m1_by_bits(c) for c in range(8)])
    g = np.random.default_rng(5)
    for trial in range(400):
        v = (g.standard_normal(16) * 10.0 ** g.uniform(-4, 3.6)).astype(np.float32)
        codes, sb = oracle.e4m3x16_quantize_group(v)
        r = float(np.max(np.abs(v.astype(np.float64)))) / 6.0
        d = np.abs(mags - r)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        if r > 448.0:
            want = 0x7E
        assert sb == want
        s = mags[sb]
        for x, c in zip(v.astype(np.float64), codes):
            if s == 0.0:
                assert (c & 7) == 0
                continue
            qd = np.abs(e2 - abs(x) / s)
            cand = np.flatnonzero(qd == qd.min())
            mag = cand[0] if len(cand) == 1 else [k for k in cand if k % 2 == 0][0]
            assert (c & 7) == mag
            assert (c >> 3) == (1 if np.signbit(x) else 0)


def test_e4m3x16_error_bound():
    # every element within half an E2M1 step of v at scale s, or saturated at 6 s;
    # the scale within half an E4M3 step of amax / 6 (relative 2^-4 for normal s)
    g = np.random.default_rng(6)
    for trial in range(300):
        v = (g.standard_normal(16) * 10.0 ** g.uniform(-1, 2.5)).astype(np.float32)
        codes, sb = oracle.e4m3x16_quantize_group(v)
        s = e4m3_by_bits(sb)
        amax = float(np.max(np.abs(v.astype(np.float64))))
        assert abs(s - amax / 6.0) <= (amax / 6.0) * 2.0 ** -4 * (1 + 1e-12)
        deq = np.array([e2m1_by_bits(int(c)) * s for c in codes])
        for x, y in zip(v.astype(np.float64), deq):
            q = abs(x) / s
            if q > 6.0:
                assert abs(y) == 6.0 * s and np.sign(y) == np.sign(x)
                continue
            half_step = 0.25 if q <= 2.0 else 0.5 if q <= 4.0 else 1.0
            assert abs(y - x) <= half_step * s * (1 + 1e-12)


def test_e4m3x16_dequantize_matches_definition():
    g = np.random.default_rng(7)
    fp4 = g.integers(0, 256, size=(3, 32), dtype=np.uint8)
    sc = g.integers(0, 0x7F, size=(3, 4), dtype=np.uint8)
    deq = oracle.fp4_dequantize(fp4, sc, oracle.SCALE_E4M3_16)
    for r in range(3):
        for d in range(64):
            code = (fp4[r, d // 2] >> (4 * (d % 2))) & 0xF
            assert deq[r, d] == e2m1_by_bits(int(code)) * e4m3_by_bits(int(sc[r, d // 16]))
