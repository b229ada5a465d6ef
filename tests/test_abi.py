"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/csa.h declares, and rejects bad arguments on the host with the
documented status codes (nothing is launched, so no device is touched)."""
import ctypes
import os
import re

import pytest

import fp4_kv_cache_csa_b200 as csa
from fp4_kv_cache_csa_b200 import build as csa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_WORKSPACE = 0, 1, 2, 3, 4, 5


@pytest.fixture(scope="module")
def lib():
    csa_build.build()
    return csa.load_library()


def header_functions():
    text = open(os.path.join(ROOT, "include", "csa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert set(names) == set(csa.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n
    assert lib.csa_version() == 103
    assert lib.csa_status_string(0) == b"ok"
    assert lib.csa_status_string(99) == b"unknown status"


def fake_cache(**kw):
    # host addresses that are never dereferenced (every call below fails validation first)
    d = dict(batch=2, dim=512, block=4, capacity=1024, fp4=0x10000, scale=0x20000, idx_key=0x30000,
             idx_dim=128, idx_dtype=1, n_blocks=0x40000, status=0, scale_fmt=0)
    d.update(kw)
    c = csa._CCache(d["batch"], d["dim"], d["block"], d["capacity"], d["fp4"], d["scale"], d["idx_key"],
                    d["idx_dim"], d["idx_dtype"], d["n_blocks"], d["status"] or None, d["scale_fmt"],
                    d.get("idx_key_scale") or None)
    return c


def compress(lib, c, kv=0x50000, idx=0x60000, gate=0x70000, offs=0x80000, n=16):
    return lib.csa_compress_quantize(ctypes.byref(c) if c is not None else None, kv, idx, gate, offs, n, None)


def test_mxfp4_key_validation(lib):
    # MXFP4 indexer keys need their scale plane (4-byte aligned); the indexer pairs each head with
    # the key groups in its MMA columns, so at most 4 indexer heads are supported with them
    assert compress(lib, fake_cache(idx_dtype=2)) == ERR_NULL
    assert compress(lib, fake_cache(idx_dtype=2, idx_key_scale=0x90002)) == ERR_ALIGN
    c = fake_cache(idx_dtype=2, idx_key_scale=0x90000)
    assert compress(lib, fake_cache(idx_dtype=3, idx_key_scale=0x90000)) == ERR_SHAPE
    args = (0x90000, 0xA0000, 2, 8, 0xB0000, 0xC0000, 64, 0xD0000, 0x100000, 1 << 40, None)
    assert lib.csa_index_topk(ctypes.byref(c), *args) == ERR_UNSUPPORTED
    args4 = (0x90000, 0xA0000, 2, 4, 0xB0000, 0xC0000, 64, 0xD0000, 0, 0, None)
    assert lib.csa_index_topk(ctypes.byref(c), *args4) == ERR_WORKSPACE  # 4 heads pass the checks


def test_compress_validation(lib):
    assert compress(lib, None) == ERR_NULL
    assert compress(lib, fake_cache(fp4=0)) == ERR_NULL
    assert compress(lib, fake_cache(), kv=0) == ERR_NULL
    assert compress(lib, fake_cache(), idx=0) == ERR_NULL            # cache has keys, no key tokens
    assert compress(lib, fake_cache(idx_key=0), idx=0x60000) == ERR_NULL
    assert compress(lib, fake_cache(block=0)) == ERR_SHAPE
    assert compress(lib, fake_cache(block=129)) == ERR_SHAPE
    assert compress(lib, fake_cache(dim=100)) == ERR_SHAPE
    assert compress(lib, fake_cache(dim=1024)) == ERR_UNSUPPORTED
    assert compress(lib, fake_cache(idx_dim=96)) == ERR_UNSUPPORTED
    assert compress(lib, fake_cache(capacity=(1 << 19) + 1)) == ERR_UNSUPPORTED
    assert compress(lib, fake_cache(fp4=0x10008)) == ERR_ALIGN
    assert compress(lib, fake_cache(scale=0x20004)) == ERR_ALIGN
    assert compress(lib, fake_cache(scale_fmt=2)) == ERR_SHAPE
    assert compress(lib, fake_cache(scale_fmt=-1)) == ERR_SHAPE
    assert compress(lib, fake_cache(), kv=0x50008) == ERR_ALIGN
    assert compress(lib, fake_cache(), n=-1) == ERR_SHAPE


def test_index_topk_validation(lib):
    c = fake_cache()
    ws = lib.csa_index_topk_workspace(ctypes.byref(c), 32, 1024)
    assert ws > 32 * 1024 * 4  # at least the score rows
    assert lib.csa_index_topk_workspace(ctypes.byref(c), 0, 1024) == 0

    def call(cache=c, q=0x90000, w=0xA0000, nq=32, hi=4, offs=0xB0000, pos=0xC0000, k=1024, sel=0xD0000,
             wsp=0x1000000, wsb=None):
        return lib.csa_index_topk(ctypes.byref(cache), q, w, nq, hi, offs, pos, k, sel, wsp,
                                  ws if wsb is None else wsb, None)

    assert call(cache=fake_cache(idx_key=0)) == ERR_NULL
    assert call(q=0) == ERR_NULL
    assert call(nq=0) == ERR_SHAPE
    assert call(k=0) == ERR_SHAPE
    assert call(hi=9) == ERR_UNSUPPORTED
    assert call(k=5000) == ERR_UNSUPPORTED
    assert call(q=0x90008) == ERR_ALIGN
    assert call(wsp=0) == ERR_WORKSPACE
    assert call(wsb=ws - 1) == ERR_WORKSPACE
    assert call(wsp=0x1000010) == ERR_ALIGN


def test_index_workspace_is_bounded(lib):
    # the size query asks for all queries' workspace when it stays under 768 MiB, else for the
    # most queries that fit (the call runs the rest in further chunks); GEMM calls get at least
    # one wave of query tiles (4736 queries' score rows)
    def ws(nq, **kw):
        return lib.csa_index_topk_workspace(ctypes.byref(fake_cache(**kw)), nq, 512)

    wave = 148 * 32
    for dt, extra in ((0, {}), (2, {"idx_key_scale": 0x90000})):  # 4 x 8192 prefill tokens over 18432 blocks
        w = ws(32768, batch=4, capacity=18432, idx_dtype=dt, **extra)
        assert 4 * 18432 * wave < w <= (768 << 20)
    w = ws(32, batch=32, capacity=262144, idx_dtype=1)  # decode at 1M: one pass over everything
    assert w > 32 * 12 * 262144
    w = ws(8192, batch=1, capacity=262144, idx_dtype=0)  # 8192 prefill tokens over a 1M-token cache
    assert 4 * 262144 * wave < w < 4 * 262144 * 8192
    w = ws(8192, batch=1, capacity=262144, idx_dtype=1)  # e4m3 keys: streamed, chunks of 128 queries
    assert 128 * 12 * 262144 < w < 256 * 12 * 262144
    # a call accepts less than the size query's answer, down to one chunk of 128 queries
    c = fake_cache(batch=2, capacity=1024, idx_dtype=0)
    args = (0x90000, 0xA0000, 1024, 4, 0xB0000, 0xC0000, 256, 0xD0000, 0x1000000)
    assert lib.csa_index_topk(ctypes.byref(c), *args, 4 * 1024 * 100, None) == ERR_WORKSPACE


def test_size_query_always_suffices_and_one_chunk_is_the_floor(lib):
    # Without a GPU a call that passes every host check fails only at its device query
    # (CSA_ERR_CUDA), so the workspace check's verdict can be read without launching.
    # On a machine with a GPU it would launch on these fake pointers: skipped there.
    import torch

    if torch.cuda.is_available():
        pytest.skip("needs a machine without a GPU (the call would launch)")
    ERR_CUDA = 6

    def call(c, nq, hi, wsb):
        return lib.csa_index_topk(ctypes.byref(c), 0x90000, 0xA0000, nq, hi, 0xB0000, 0xC0000, 256, 0xD0000,
                                  0x1000000, wsb, None)

    # the GEMM + row selection layout of one 128-query chunk: per-query ranges
    # (4 + 4 + 8 + 12 bytes, each array 256-aligned, gprefix one longer) and score rows
    def rows_floor(cap):
        a = lambda x: (x + 255) // 256 * 256
        return a(4 * 128) + a(4 * 128) + a(8 * 129) + a(12 * 128) + a(4 * cap * 128)

    for cap in (1000, 1024, 18432):
        c = fake_cache(batch=2, capacity=cap, idx_dtype=0)  # bf16 keys, 2048 queries: prefill-shaped
        floor = rows_floor(cap)
        assert call(c, 2048, 4, floor - 1) == ERR_WORKSPACE
        assert call(c, 2048, 4, floor) == ERR_CUDA
    for dt, extra in ((0, {}), (1, {}), (2, {"idx_key_scale": 0x90000})):
        for cap in (64, 3001, 40960, 40961, 262144):
            for nq in (1, 32, 127, 128, 129, 4000, 40000):
                c = fake_cache(batch=2, capacity=cap, idx_dtype=dt, **extra)
                w = lib.csa_index_topk_workspace(ctypes.byref(c), nq, 256)
                for hi in ((1, 2, 3, 4) if dt == 2 else (1, 2, 3, 4, 5, 8)):
                    assert call(c, nq, hi, w) == ERR_CUDA, (dt, cap, nq, hi)


def test_attend_validation(lib):
    c = fake_cache()

    def call(cache=c, q=0x90000, nq=4, heads=64, offs=0xB0000, sel=0xD0000, k=64, win=0xE0000, ws_=0xF0000,
             wl=0xF1000, maxw=128, out=0x1000000, lse=0):
        return lib.csa_decode_attend(ctypes.byref(cache), q, nq, heads, offs, sel, k, win, ws_, wl, maxw, 0.1, out,
                                     lse or None, 0x2000000, 1 << 30, None)

    assert call(q=0) == ERR_NULL
    assert call(out=0) == ERR_NULL
    assert call(win=0) == ERR_NULL          # window pointers are all-or-none
    assert call(nq=0) == ERR_SHAPE
    assert call(maxw=-1) == ERR_SHAPE
    assert call(heads=65) == ERR_UNSUPPORTED
    assert call(cache=fake_cache(dim=256)) == ERR_UNSUPPORTED
    assert call(q=0x90008) == ERR_ALIGN
    assert lib.hca_decode_attend(ctypes.byref(c), 0x90000, 4, 64, 0xB0000, None, None, None, None, 128, 0.1,
                                 0x1000000, None, 0x2000000, 1 << 30, None) != OK


def test_pool_and_reindex_validation(lib):
    c = fake_cache()
    ws = lib.csa_index_pool_workspace(ctypes.byref(c), 32, 1024, 8, 2000)
    assert ws > lib.csa_index_topk_workspace(ctypes.byref(c), 32, 1024)
    assert lib.csa_index_pool_workspace(ctypes.byref(c), 32, 1024, 6, 2000) == 0   # group not a power of two
    assert lib.csa_index_pool_workspace(ctypes.byref(c), 32, 1024, 64, 2000) == 0  # group above 32
    wr = lib.csa_index_reindex_workspace(ctypes.byref(c), 32, 8, 2000)
    assert wr >= 32 * 8 * 2000 * 4  # the score rows over the pool positions

    def pool(cache=c, q=0x90000, k=1024, grp=8, pb=2000, out=0xE0000, wsp=0x1000000, wsb=None):
        return lib.csa_index_topk_pool(ctypes.byref(cache), q, 0xA0000, 32, 4, 0xB0000, 0xC0000, k, 0xD0000, grp, pb,
                                       out, wsp, ws if wsb is None else wsb, None)

    def reindex(q=0x90000, grp=8, pb=2000, pl=0xE0000, wsp=0x1000000, wsb=None):
        return lib.csa_index_topk_reindex(ctypes.byref(c), q, 0xA0000, 32, 4, 0xB0000, 0xC0000, 1024, 0xD0000, grp,
                                          pb, pl, wsp, wr if wsb is None else wsb, None)

    assert pool(out=0) == ERR_NULL
    assert pool(q=0) == ERR_NULL
    assert pool(grp=3) == ERR_SHAPE
    assert pool(pb=0) == ERR_SHAPE
    assert pool(pb=5000) == ERR_UNSUPPORTED
    assert pool(out=0xE0002) == ERR_ALIGN
    assert pool(wsb=ws - 1) == ERR_WORKSPACE
    assert pool(cache=fake_cache(idx_key=0)) == ERR_NULL
    assert reindex(pl=0) == ERR_NULL
    assert reindex(grp=5) == ERR_SHAPE
    assert reindex(wsb=wr - 1) == ERR_WORKSPACE
    assert reindex(wsp=0x1000010) == ERR_ALIGN


def test_read_status_needs_status_word(lib):
    v = ctypes.c_int32(0)
    assert lib.csa_read_device_status(ctypes.byref(fake_cache()), None, ctypes.byref(v)) == ERR_NULL


def test_missing_library_raises():
    saved = csa._lib
    try:
        csa._lib = None
        with pytest.raises(csa.CsaError):
            csa.load_library("/nonexistent/libcsa.so")
    finally:
        csa._lib = saved


def test_cache_struct_layout_matches_the_header(tmp_path):
    # the ctypes mirror of csa_cache has the C compiler's field offsets and size
    src = tmp_path / "layout.c"
    fields = [f[0] for f in csa._CCache._fields_]
    body = "".join(f'printf("%zu\\n", offsetof(csa_cache, {f}));' for f in fields)
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "csa.h"\n'
                   f'int main(void) {{ {body} printf("%zu\\n", sizeof(csa_cache)); return 0; }}\n')
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    want = [getattr(csa._CCache, f).offset for f in fields] + [ctypes.sizeof(csa._CCache)]
    assert got == want


def test_mxf4_probe_argument_checks(lib):
    # the MMA probe validates on the host before touching the device
    flops = ctypes.c_int64(0)
    assert lib.csa_probe_mxf4_mma(10, None, None, ctypes.byref(flops)) == ERR_NULL
    assert lib.csa_probe_mxf4_mma(10, ctypes.c_void_p(256), None, None) == ERR_NULL
    assert lib.csa_probe_mxf4_mma(0, ctypes.c_void_p(256), None, ctypes.byref(flops)) == ERR_SHAPE
    assert lib.csa_probe_mxf4_mma(10, ctypes.c_void_p(258), None, ctypes.byref(flops)) == ERR_ALIGN
