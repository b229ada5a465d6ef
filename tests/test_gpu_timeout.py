"""Failure detection without a GPU fault: a bounded wait inside the attention kernel runs out.

Every mbarrier wait in the attention kernel is bounded; when one runs out the
kernel flags CSA_DEV_TIMEOUT in the cache's status word, waits (with the long
limit) for its own bulk copy and for every MMA it issued, frees its tensor
memory and returns, so the context stays usable. A wait that completes cannot
be made to run out (the barrier wait instruction itself sleeps until the phase
completes), so this test builds a variant of the library in which nothing ever
completes the first wait of a CTA: the copy of its query tile is announced to
the barrier but never sent (`-DCSA_TEST_UNSENT_Q_COPY`), and the limit is cut to
about half a millisecond (`-DCSA_WAIT_CYCLES`). The variant is built into the
test's temporary directory and loaded beside the shipped library; it is never
installed."""
import ctypes

import numpy as np
import pytest

import oracle
from fp4_kv_cache_csa_b200 import datagen
from gpu_util import dev, host, make_cache
import parity
from test_gpu_attend import cache_bytes, window

pytestmark = pytest.mark.gpu


def test_attention_wait_runs_out_then_the_library_still_works(tmp_path):
    import torch

    import fp4_kv_cache_csa_b200 as csa
    from fp4_kv_cache_csa_b200 import build as csa_build

    path = csa_build.build(force=True, defines=["CSA_WAIT_CYCLES=1000000", "CSA_TEST_UNSENT_Q_COPY"], lib_path=str(tmp_path / "libcsa_shortwait.so"),
                           build_dir=str(tmp_path / "build"))
    short = csa.declare(ctypes.CDLL(path))

    B, cap, D, H, m = 2, 640, 512, 64, 128
    fp4, sc = cache_bytes(B, cap, D, 80)
    n_blocks = [600, 257]
    qo = np.arange(B + 1, dtype=np.int32)
    qp = (np.asarray(n_blocks) * m - 1).astype(np.int32)
    q = datagen.normal_bf16((B, H, D), 80, 42)
    win, ws, wl = window(B, 128, D, 81)
    scale = 1.0 / np.sqrt(D)
    cache = make_cache(fp4, sc, n_blocks, m)
    args = (cache, dev(q), dev(qo), dev(qp), dev(win), dev(ws), dev(wl))

    shipped = csa.load_library()
    csa._lib = short
    try:
        csa.hca_decode_attend(*args, max_win=128, softmax_scale=scale)
        status = csa.csa_read_device_status(cache)
    finally:
        csa._lib = shipped
    assert status & csa.CSA_DEV_TIMEOUT

    # the context survived: the shipped library on the same inputs is correct and clean
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    out = csa.hca_decode_attend(*args, max_win=128, softmax_scale=scale, lse=lse)
    assert csa.csa_read_device_status(cache) == 0
    ref, ref_lse = oracle.hca_attend(fp4, sc, np.asarray(n_blocks, np.int32), qo, qp, q, win, ws, wl, scale, m=m)
    err, _ = parity.attention_row_error(host(out), ref)
    assert err <= parity.ATT_TOL
    assert np.all(np.abs(host(lse) - ref_lse) <= 1e-3 + 1e-4 * np.abs(ref_lse))
