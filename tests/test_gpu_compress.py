"""GPU parity of csa_compress_quantize (rows a1 + a2) against the oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
from fp4_kv_cache_csa_b200 import datagen
from gpu_util import dev, host
import parity

pytestmark = pytest.mark.gpu


def run(D, dI, m, idx_dtype, counts, base, cap, seed, gate_std=0.02, lognormal=0.0, scale_fmt=0):
    import torch

    import fp4_kv_cache_csa_b200 as csa

    counts = np.asarray(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    T = int(offs[-1])
    kv = datagen.normal_bf16((max(T, 1), D), seed, 1, channel_lognormal=lognormal)
    idx = datagen.normal_bf16((max(T, 1), dI), seed, 2, channel_lognormal=lognormal) if dI else None
    wg = datagen.normal_f32((D,), seed, 3, std=gate_std)
    B = len(counts)
    ref = oracle.compress(kv, idx, wg, offs, np.asarray(base, np.int32), m=m, cap=cap, idx_dtype=idx_dtype,
                          scale_fmt=scale_fmt, return_pooled=True)
    cache = csa.Cache.allocate(B, cap, D, m, dI, idx_dtype, scale_fmt=scale_fmt)
    cache.n_blocks.copy_(torch.tensor(base, dtype=torch.int32))
    csa.csa_compress_quantize(cache, dev(kv), dev(idx) if dI else None, dev(wg), dev(offs))
    status = csa.csa_read_device_status(cache)
    got = dict(fp4=host(cache.fp4), scale=host(cache.scale), n_blocks=host(cache.n_blocks),
               idx_key=None if not dI else host(cache.idx_key))
    ref["tol"] = parity.pooling_tolerance(kv, offs, base, m, cap, kv_bits=kv, w_g=wg)
    ref["tol_idx"] = parity.pooling_tolerance(idx, offs, base, m, cap, kv_bits=kv, w_g=wg) if dI else None
    return ref, got, status


def compare(ref, got, D, dI, idx_dtype, strict=False, scale_fmt=0):
    assert np.array_equal(got["n_blocks"], ref["n_blocks"])
    B, cap = ref["fp4"].shape[:2]
    ex = parity.check_mxfp4(got["fp4"].reshape(B * cap, -1), got["scale"].reshape(B * cap, -1),
                            ref["fp4"].reshape(B * cap, -1), ref["scale"].reshape(B * cap, -1),
                            ref["pooled"].reshape(B * cap, D), strict=strict, tol=ref["tol"].reshape(B * cap, D),
                            scale_fmt=scale_fmt)
    if dI:
        gk = got["idx_key"]
        if idx_dtype == 0:
            gk = gk.view(np.uint16).reshape(B, cap, dI)
            rk = ref["idx_key"].view(np.uint16).reshape(B, cap, dI)
            if strict:
                assert np.array_equal(gk, rk)
            else:
                ex += parity.check_keys(gk, rk, ref["pooled_idx"], "bf16", tol=ref["tol_idx"])
        else:
            rk = ref["idx_key"].reshape(B, cap, dI)
            if strict:
                assert np.array_equal(gk, rk)
            else:
                ex += parity.check_keys(gk, rk, ref["pooled_idx"], "e4m3", tol=ref["tol_idx"])
    return ex


@pytest.mark.parametrize("D,dI,idx_dtype", [(128, 64, 0), (512, 128, 1), (512, 128, 0), (256, 256, 1), (64, 64, 0)])
def test_m1_is_bit_exact(D, dI, idx_dtype):
    # m = 1: the gate weight is exactly 1, pooling is the identity and the bytes must match exactly
    ref, got, st = run(D, dI, 1, idx_dtype, [37, 5, 64], [0, 3, 1], 128, seed=11)
    assert st == 0
    compare(ref, got, D, dI, idx_dtype, strict=True)


@pytest.mark.parametrize("D,dI,idx_dtype,m", [(128, 64, 0, 4), (512, 128, 1, 4), (512, 128, 0, 4),
                                              (512, 0, 0, 128), (128, 128, 1, 16)])
def test_pooling_parity(D, dI, idx_dtype, m):
    counts = [m * 300, m * 7, 0, m * 129]  # ragged, one request with nothing new
    ref, got, st = run(D, dI, m, idx_dtype, counts, [5, 0, 2, 17], 512, seed=12 + m)
    assert st == 0
    compare(ref, got, D, dI, idx_dtype)


def test_channel_scaled_inputs_exercise_scales():
    # per-channel LogNormal(0, 0.5) scales spread the E8M0 exponents
    ref, got, st = run(512, 128, 4, 0, [4 * 2048], [0], 2048, seed=13, lognormal=0.5)
    assert st == 0
    assert len(np.unique(ref["scale"])) > 4
    compare(ref, got, 512, 128, 0)


def test_device_checks_skip_bad_requests():
    import torch

    import fp4_kv_cache_csa_b200 as csa

    # request 0: count not a multiple of m; request 1: overflows capacity; request 2: fine
    offs = np.array([0, 6, 6 + 40, 6 + 40 + 8], np.int32)
    kv = datagen.normal_bf16((54, 128), 14, 1)
    cache = csa.Cache.allocate(3, 10, 128, 4)
    cache.n_blocks.copy_(torch.tensor([0, 2, 1], dtype=torch.int32))
    csa.csa_compress_quantize(cache, dev(kv), None, dev(np.zeros(128, np.float32)), dev(offs))
    st = csa.csa_read_device_status(cache)
    assert st & csa.CSA_DEV_TOKEN_COUNT and st & csa.CSA_DEV_CAPACITY
    assert list(host(cache.n_blocks)) == [0, 2, 3]
    assert not host(cache.scale)[0].any() and not host(cache.scale)[1].any()
    assert csa.csa_read_device_status(cache) == 0  # cleared


# ---------------------------------------------------------------- E4M3 scale per 16 elements

E4 = oracle.SCALE_E4M3_16


@pytest.mark.parametrize("D,dI,idx_dtype", [(128, 64, 0), (512, 128, 1), (256, 256, 0), (64, 64, 1)])
def test_e4m3x16_m1_is_bit_exact(D, dI, idx_dtype):
    ref, got, st = run(D, dI, 1, idx_dtype, [37, 5, 64], [0, 3, 1], 128, seed=21, scale_fmt=E4)
    assert st == 0
    assert got["scale"].shape[-1] == D // 16
    compare(ref, got, D, dI, idx_dtype, strict=True, scale_fmt=E4)


def test_e4m3x16_m1_tiny_and_huge_values_are_bit_exact():
    # m = 1 tokens spanning 2^-20 .. 2^14: zero scales (sign-only codes), subnormal
    # E4M3 scales and saturated scales (amax / 6 > 448) all round like the oracle
    import torch

    import fp4_kv_cache_csa_b200 as csa

    D, T = 128, 96
    g = np.random.default_rng(22)
    mag = np.ldexp(1.0, g.integers(-20, 15, size=(T, D // 16)))
    x = (g.standard_normal((T, D // 16, 16)) * mag[:, :, None]).reshape(T, D).astype(np.float32)
    kv = datagen.to_bf16_bits(x)
    offs = np.array([0, T], np.int32)
    ref = oracle.compress(kv, None, np.zeros(D, np.float32), offs, np.zeros(1, np.int32), m=1, cap=T, scale_fmt=E4)
    assert (ref["scale"] == 0).any() and (ref["scale"] == 0x7E).any() and ((ref["scale"] & 0x78) == 0).sum() > 8
    cache = csa.Cache.allocate(1, T, D, 1, scale_fmt=E4)
    csa.csa_compress_quantize(cache, dev(kv), None, dev(np.zeros(D, np.float32)), dev(offs))
    assert csa.csa_read_device_status(cache) == 0
    assert np.array_equal(host(cache.scale), ref["scale"])
    assert np.array_equal(host(cache.fp4), ref["fp4"])


@pytest.mark.parametrize("D,dI,idx_dtype,m", [(512, 128, 1, 4), (128, 64, 0, 4), (512, 0, 0, 128), (64, 64, 1, 16)])
def test_e4m3x16_pooling_parity(D, dI, idx_dtype, m):
    counts = [m * 300, m * 7, 0, m * 129]
    ref, got, st = run(D, dI, m, idx_dtype, counts, [5, 0, 2, 17], 512, seed=23 + m, scale_fmt=E4)
    assert st == 0
    compare(ref, got, D, dI, idx_dtype, scale_fmt=E4)
