"""GPU parity of csa_decode_attend / hca_decode_attend (rows a5-a8) against the oracle.

Cache bytes are seeded inputs (uniform E2M1 code bytes, E8M0 or E4M3 scale bytes
in the range pooled N(0,1) blocks land in); queries and window rows are N(0,1) bf16.
Tolerance: per (query, head) row, max_d |gpu - oracle| / max_d |oracle| <= 2e-3;
lse within 1e-3 + 1e-4 |lse|."""
import numpy as np
import pytest

import oracle
from fp4_kv_cache_csa_b200 import datagen
from gpu_util import dev, host, make_cache
import parity

pytestmark = pytest.mark.gpu


def cache_bytes(B, cap, D, seed, lo=123, hi=126):
    fp4, sc = datagen.random_cache_bytes(B * cap, D, seed, 40, scale_lo=lo, scale_hi=hi)
    return fp4.reshape(B, cap, D // 2), sc.reshape(B, cap, D // 32)


def cache_bytes_e4m3x16(B, cap, D, seed, lo=0x1C, hi=0x2C):
    fp4, sc = datagen.random_cache_bytes_e4m3x16(B * cap, D, seed, 44, scale_lo=lo, scale_hi=hi)
    return fp4.reshape(B, cap, D // 2), sc.reshape(B, cap, D // 16)


def window(Nq, W, D, seed, wlen=None):
    win = datagen.normal_bf16((Nq * W, D), seed, 41)
    ws = (np.arange(Nq) * W).astype(np.int64)
    wl = np.full(Nq, W, np.int32) if wlen is None else np.asarray(wlen, np.int32)
    return win, ws, wl


def check(out, lse, ref, ref_lse, H):
    err, _ = parity.attention_row_error(out, ref)
    assert err <= parity.ATT_TOL, f"row error {err}"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.all(np.abs(lse[fin] - ref_lse[fin]) <= 1e-3 + 1e-4 * np.abs(ref_lse[fin]))
    return err


def run_csa(fp4, sc, n_blocks, q_offsets, sel, H, D, win=None, ws=None, wl=None, seed=50, max_win=128, scale_fmt=0):
    import torch

    import fp4_kv_cache_csa_b200 as csa

    Nq = int(q_offsets[-1])
    q = datagen.normal_bf16((Nq, H, D), seed, 42)
    scale = 1.0 / np.sqrt(D)
    ref, ref_lse = oracle.csa_attend(fp4, sc, q_offsets, q, sel, win, ws, wl, scale, scale_fmt=scale_fmt)
    cache = make_cache(fp4, sc, n_blocks, 4, scale_fmt=scale_fmt)
    lse = torch.empty(Nq, H, dtype=torch.float32, device="cuda")
    out = csa.csa_decode_attend(cache, dev(q), dev(np.asarray(q_offsets, np.int32)), dev(sel),
                                None if win is None else dev(win), None if ws is None else dev(ws),
                                None if wl is None else dev(wl), max_win=max_win, softmax_scale=scale, lse=lse)
    status = csa.csa_read_device_status(cache)
    return check(host(out), host(lse), ref, ref_lse, H), status


def random_sel(n_vis, k, Nq, seed, pad_from=None):
    rng = np.random.default_rng(seed)
    sel = np.full((Nq, k), -1, np.int32)
    for i in range(Nq):
        take = min(k, n_vis[i]) if pad_from is None else min(pad_from[i], n_vis[i])
        sel[i, :take] = np.sort(rng.choice(n_vis[i], take, replace=False))
    return sel


def test_tiny_d128_h16():
    fp4, sc = cache_bytes(1, 1024, 128, 1)
    sel = random_sel([1024], 64, 1, 2)
    win, ws, wl = window(1, 128, 128, 3)
    err, st = run_csa(fp4, sc, [1024], np.array([0, 1], np.int32), sel, 16, 128, win, ws, wl)
    assert st == 0


def test_b2_d512_h64_k512():
    fp4, sc = cache_bytes(2, 16384, 512, 4)
    sel = random_sel([16384, 9000], 512, 2, 5)
    win, ws, wl = window(2, 128, 512, 6)
    err, st = run_csa(fp4, sc, [16384, 9000], np.array([0, 1, 2], np.int32), sel, 64, 512, win, ws, wl)
    assert st == 0


def test_long_selection_is_split_and_merged():
    # 4096 selected + window = 33 tiles per query for 2 queries: every query spans many CTAs
    fp4, sc = cache_bytes(2, 8192, 512, 7)
    sel = random_sel([8192, 8192], 4096, 2, 8)
    win, ws, wl = window(2, 128, 512, 9)
    run_csa(fp4, sc, [8192, 8192], np.array([0, 1, 2], np.int32), sel, 64, 512, win, ws, wl)


def test_padding_partial_window_and_window_only():
    fp4, sc = cache_bytes(3, 4096, 512, 10)
    sel = random_sel([4096, 50, 4096], 1024, 3, 11, pad_from=[700, 50, 0])  # -1 padded rows
    win, ws, wl = window(3, 128, 512, 12, wlen=[77, 128, 5])
    run_csa(fp4, sc, [4096, 50, 4096], np.array([0, 1, 2, 3], np.int32), sel, 64, 512, win, ws, wl)


def test_no_window_and_empty_query():
    fp4, sc = cache_bytes(2, 1024, 512, 13)
    sel = random_sel([1024, 1024], 256, 2, 14, pad_from=[256, 0])
    run_csa(fp4, sc, [1024, 1024], np.array([0, 1, 2], np.int32), sel, 64, 512)


def test_out_of_range_index_is_flagged_and_skipped():
    import fp4_kv_cache_csa_b200 as csa

    fp4, sc = cache_bytes(1, 2048, 512, 15)
    sel = random_sel([1000], 128, 1, 16)
    bad = sel.copy()
    bad[0, 5] = 1500  # beyond n_blocks = 1000
    skipped = sel.copy()
    skipped[0, 5] = -1
    win, ws, wl = window(1, 128, 512, 17)
    q = datagen.normal_bf16((1, 64, 512), 18, 42)
    ref, ref_lse = oracle.csa_attend(fp4, sc, np.array([0, 1], np.int32), q, skipped, win, ws, wl, 512 ** -0.5)
    cache = make_cache(fp4, sc, [1000], 4)
    import torch
    lse = torch.empty(1, 64, dtype=torch.float32, device="cuda")
    out = csa.csa_decode_attend(cache, dev(q), dev(np.array([0, 1], np.int32)), dev(bad), dev(win), dev(ws), dev(wl),
                                lse=lse)
    assert csa.csa_read_device_status(cache) & csa.CSA_DEV_BAD_INDEX
    check(host(out), host(lse), ref, ref_lse, 64)


def test_scale_spread_rows():
    # scale bytes spread over 40 binades: the per-entry fp16 normalisation must keep every row exact
    fp4, sc = cache_bytes(1, 2048, 512, 19, lo=100, hi=140)
    sel = random_sel([2048], 512, 1, 20)
    win, ws, wl = window(1, 128, 512, 21)
    run_csa(fp4, sc, [2048], np.array([0, 1], np.int32), sel, 64, 512, win, ws, wl)


# ---------------------------------------------------------------- HCA

def run_hca(fp4, sc, n_blocks, q_offsets, q_pos, H, D, m, win=None, ws=None, wl=None, seed=60, scale_fmt=0):
    import torch

    import fp4_kv_cache_csa_b200 as csa

    Nq = int(q_offsets[-1])
    q = datagen.normal_bf16((Nq, H, D), seed, 43)
    scale = 1.0 / np.sqrt(D)
    ref, ref_lse = oracle.hca_attend(fp4, sc, n_blocks, q_offsets, q_pos, q, win, ws, wl, scale, m=m,
                                     scale_fmt=scale_fmt)
    cache = make_cache(fp4, sc, n_blocks, m, scale_fmt=scale_fmt)
    lse = torch.empty(Nq, H, dtype=torch.float32, device="cuda")
    out = csa.hca_decode_attend(cache, dev(q), dev(np.asarray(q_offsets, np.int32)), dev(np.asarray(q_pos, np.int32)),
                                None if win is None else dev(win), None if ws is None else dev(ws),
                                None if wl is None else dev(wl), softmax_scale=scale, lse=lse)
    assert csa.csa_read_device_status(cache) == 0
    return check(host(out), host(lse), ref, ref_lse, H)


def test_hca_dense_8192_entries():
    fp4, sc = cache_bytes(2, 8192, 512, 22, lo=120, hi=123)
    win, ws, wl = window(2, 128, 512, 23)
    run_hca(fp4, sc, [8192, 8192], np.array([0, 1, 2], np.int32), np.array([1048575, 700000], np.int32), 64, 512,
            128, win, ws, wl)


def test_hca_window_only_and_d128():
    fp4, sc = cache_bytes(2, 256, 128, 24, lo=120, hi=123)
    win, ws, wl = window(2, 128, 128, 25, wlen=[128, 60])
    run_hca(fp4, sc, [256, 256], np.array([0, 1, 2], np.int32), np.array([100, 32767], np.int32), 16, 128, 128,
            win, ws, wl)


def test_csa_with_all_blocks_equals_hca():
    # k >= n_blocks: CSA over every block is dense attention (same inputs, both GPU paths)
    import torch

    import fp4_kv_cache_csa_b200 as csa

    fp4, sc = cache_bytes(1, 640, 512, 26)
    win, ws, wl = window(1, 128, 512, 27)
    q = dev(datagen.normal_bf16((1, 64, 512), 28, 1))
    cache = make_cache(fp4, sc, [640], 4)
    sel = dev(np.arange(640, dtype=np.int32)[None])
    a = host(csa.csa_decode_attend(cache, q, dev(np.array([0, 1], np.int32)), sel, dev(win), dev(ws), dev(wl)))
    b = host(csa.hca_decode_attend(cache, q, dev(np.array([0, 1], np.int32)), dev(np.array([2559], np.int32)),
                                   dev(win), dev(ws), dev(wl)))
    assert parity.attention_row_error(a, b)[0] <= 1e-5


# ---------------------------------------------------------------- E4M3 scale per 16 elements

E4 = oracle.SCALE_E4M3_16


def test_e4m3x16_csa_d512_h64():
    fp4, sc = cache_bytes_e4m3x16(2, 16384, 512, 70)
    sel = random_sel([16384, 9000], 1024, 2, 71, pad_from=[1024, 333])
    win, ws, wl = window(2, 128, 512, 72, wlen=[128, 41])
    err, st = run_csa(fp4, sc, [16384, 9000], np.array([0, 1, 2], np.int32), sel, 64, 512, win, ws, wl,
                      scale_fmt=E4)
    assert st == 0


def test_e4m3x16_csa_d128_h16_split():
    # 2048 selected entries per query: each query spans several CTAs and is merged
    fp4, sc = cache_bytes_e4m3x16(1, 4096, 128, 73)
    sel = random_sel([4096, 4096, 4096], 2048, 3, 74)
    win, ws, wl = window(3, 128, 128, 75)
    err, st = run_csa(fp4, sc, [4096], np.array([0, 3], np.int32), sel, 16, 128, win, ws, wl, scale_fmt=E4)
    assert st == 0


def test_e4m3x16_full_scale_range_is_exact_in_fp16():
    # scale bytes over every positive finite E4M3 value (2^-9 .. 448, subnormals included):
    # every E2M1 x E4M3 product is exact in fp16, with no per-row normalisation
    fp4, sc = cache_bytes_e4m3x16(1, 2048, 512, 76, lo=0x01, hi=0x7E)
    sel = random_sel([2048], 512, 1, 77)
    win, ws, wl = window(1, 128, 512, 78)
    run_csa(fp4, sc, [2048], np.array([0, 1], np.int32), sel, 64, 512, win, ws, wl, scale_fmt=E4)


def test_e4m3x16_hca_dense():
    fp4, sc = cache_bytes_e4m3x16(2, 8192, 512, 79)
    win, ws, wl = window(2, 128, 512, 80)
    run_hca(fp4, sc, [8192, 5000], np.array([0, 1, 2], np.int32), np.array([1048575, 700000], np.int32), 64, 512,
            128, win, ws, wl, scale_fmt=E4)


@pytest.mark.parametrize("D,H", [(128, 16), (512, 64)])
def test_more_queries_than_ctas(D, H):
    # prefill-shaped calls: more queries than CTAs, ragged selection lengths (0 to 3 tiles of
    # 128 entries) and windows, so many queries straddle a CTA boundary and are merged by the
    # boundary-indexed merge grid; every query is compared with the oracle
    B, cap, Nq = 2, 2048, 400
    fp4, sc = cache_bytes(B, cap, D, 60)
    counts = [230, 170]
    q_offsets = np.array([0, counts[0], Nq], np.int32)
    rng = np.random.default_rng(61)
    k = 384
    take = rng.integers(0, k + 1, Nq)
    take[::37] = 0
    sel = random_sel([cap] * Nq, k, Nq, 62, pad_from=take)
    wlen = rng.integers(0, 129, Nq)
    win, ws, wl = window(Nq, 128, D, 63, wlen=wlen)
    err, st = run_csa(fp4, sc, [cap, cap], q_offsets, sel, H, D, win, ws, wl, seed=64)
    assert st == 0
