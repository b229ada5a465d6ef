"""Plain CPU reference ("oracle") for CSA / HCA / window attention over an MXFP4 KV cache.

TEST INFRASTRUCTURE ONLY. The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The CUDA library never
imports, links or runs anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``csa_oracle.c`` (plain loops, double precision; see the
header for the sources on the pages and the precision rules). This module only
compiles it with gcc and marshals numpy arrays through ctypes.

bf16 tensors are numpy ``uint16`` arrays of bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_HDR = os.path.join(_HERE, "csa_oracle.h")
_LIB_PATH = os.path.join(_HERE, "_liboracle.so")
_lib = None

IDX_BF16 = 0
IDX_E4M3 = 1
IDX_MXFP4 = 2  # E2M1 codes [.., dI/2] + one E8M0 scale per 32 channels [.., dI/32]

# scale formats of the FP4 cache: E8M0 per 32 elements (OCP MXFP4), E4M3 per 16
SCALE_E8M0_32 = 0
SCALE_E4M3_16 = 1


def group_size(scale_fmt: int) -> int:
    return 32 if scale_fmt == SCALE_E8M0_32 else 16


def build(force: bool = False) -> str:
    """Compile csa_oracle.c into _liboracle.so (gcc, OpenMP, no fast-math, no FMA contraction)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.orc_bf16_decode.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_decode.restype = D
        lib.orc_bf16_encode.argtypes = [ctypes.c_float]
        lib.orc_bf16_encode.restype = ctypes.c_uint16
        lib.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e2m1_decode.restype = D
        lib.orc_e2m1_encode.argtypes = [D]
        lib.orc_e2m1_encode.restype = ctypes.c_uint8
        lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_decode.restype = D
        lib.orc_e4m3_encode.argtypes = [D]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_mxfp4_quantize_group.argtypes = [P, P, P]
        lib.orc_mxfp4_quantize_group.restype = None
        lib.orc_e4m3x16_quantize_group.argtypes = [P, P, P]
        lib.orc_e4m3x16_quantize_group.restype = None
        lib.orc_compress.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P]
        lib.orc_compress.restype = I
        lib.orc_index_scores.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P]
        lib.orc_index_scores.restype = None
        lib.orc_topk.argtypes = [I, I, I, P, P, P]
        lib.orc_topk.restype = None
        lib.orc_index_pool.argtypes = [I, I, I, I, P, P, P]
        lib.orc_index_pool.restype = None
        lib.orc_reindex_topk.argtypes = [I, I, I, I, I, P, P, P, P]
        lib.orc_reindex_topk.restype = None
        lib.orc_csa_attend.argtypes = [I, I, I, I, I, I, P, P, I, P, P, P, P, P, P, D, P, P]
        lib.orc_csa_attend.restype = None
        lib.orc_hca_attend.argtypes = [I, I, I, I, I, I, P, P, I, P, P, P, P, P, P, P, D, P, P]
        lib.orc_hca_attend.restype = None
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return _load().orc_num_threads()


# ---- number formats --------------------------------------------------------

def bf16_decode(bits: int) -> float:
    return _load().orc_bf16_decode(int(bits))


def bf16_encode(x: float) -> int:
    return int(_load().orc_bf16_encode(float(x)))


def e2m1_decode(code: int) -> float:
    return _load().orc_e2m1_decode(int(code))


def e2m1_encode(x: float) -> int:
    return int(_load().orc_e2m1_encode(float(x)))


def e4m3_decode(code: int) -> float:
    return _load().orc_e4m3_decode(int(code))


def e4m3_encode(x: float) -> int:
    return int(_load().orc_e4m3_encode(float(x)))


def mxfp4_quantize_group(v):
    """32 float32 values -> (codes[32] one per byte, scale byte)."""
    v = _c(v, np.float32)
    assert v.shape == (32,)
    codes = np.zeros(32, np.uint8)
    sb = np.zeros(1, np.uint8)
    _load().orc_mxfp4_quantize_group(_ptr(v), _ptr(codes), _ptr(sb))
    return codes, int(sb[0])


def e4m3x16_quantize_group(v):
    """16 float32 values -> (codes[16] one per byte, E4M3 scale byte)."""
    v = _c(v, np.float32)
    assert v.shape == (16,)
    codes = np.zeros(16, np.uint8)
    sb = np.zeros(1, np.uint8)
    _load().orc_e4m3x16_quantize_group(_ptr(v), _ptr(codes), _ptr(sb))
    return codes, int(sb[0])


def e4m3x16_dequantize(fp4_rows, scale_rows):
    """Dequantize [..., D/2] packed codes + [..., D/16] E4M3 scale bytes to float64 [..., D]:
    value = E2M1(code) * E4M3(scale byte of its 16-element group)."""
    fp4_rows = np.asarray(fp4_rows, np.uint8)
    scale_rows = np.asarray(scale_rows, np.uint8)
    codes = np.stack([fp4_rows & 0xF, fp4_rows >> 4], axis=-1).reshape(*fp4_rows.shape[:-1], fp4_rows.shape[-1] * 2)
    table = np.array([e2m1_decode(c) for c in range(16)], np.float64)
    stable = np.array([e4m3_decode(c) for c in range(256)], np.float64)
    s = np.repeat(stable[scale_rows], 16, axis=-1)
    assert s.shape[-1] == codes.shape[-1]
    return table[codes] * s


def fp4_dequantize(fp4_rows, scale_rows, scale_fmt=SCALE_E8M0_32):
    if scale_fmt == SCALE_E8M0_32:
        return mxfp4_dequantize(fp4_rows, scale_rows)
    return e4m3x16_dequantize(fp4_rows, scale_rows)


def mxfp4_dequantize(fp4_rows, scale_rows):
    """Dequantize [..., D/2] packed codes + [..., D/32] scale bytes to float64 [..., D].

    Plain restatement of the format for tests: element 2i is the low nibble of
    byte i, value = E2M1(code) * 2^(scale - 127).
    """
    fp4_rows = np.asarray(fp4_rows, np.uint8)
    scale_rows = np.asarray(scale_rows, np.uint8)
    lo = fp4_rows & 0xF
    hi = fp4_rows >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(*fp4_rows.shape[:-1], fp4_rows.shape[-1] * 2)
    table = np.array([e2m1_decode(c) for c in range(16)], np.float64)
    D = codes.shape[-1]
    X = scale_rows.astype(np.int64) - 127
    Xe = np.repeat(X, 32, axis=-1)
    assert Xe.shape[-1] == D
    return np.ldexp(table[codes], Xe)


# ---- the method ------------------------------------------------------------

def compress(kv_tok, idx_tok, w_g, tok_offsets, n_blocks, *, m, cap, idx_dtype=IDX_BF16,
             scale_fmt=SCALE_E8M0_32, fp4=None, scale=None, idx_key=None, idx_key_scale=None,
             return_pooled=False):
    """Gated m-token pooling + FP4 quantization (rows a1, a2), scales per scale_fmt.

    kv_tok [T, D] uint16 (bf16 bits), idx_tok [T, dI] uint16 or None, w_g [D] float32,
    tok_offsets [B+1] int32, n_blocks [B] int32 (copied, returned updated).
    Returns dict(fp4, scale, idx_key, idx_key_scale (MXFP4 keys only), n_blocks[, pooled]).
    """
    kv_tok = _c(kv_tok, np.uint16)
    T, D = kv_tok.shape
    tok_offsets = _c(tok_offsets, np.int32)
    B = tok_offsets.shape[0] - 1
    n_blocks = np.array(n_blocks, np.int32, copy=True)
    dI = 0 if idx_tok is None else idx_tok.shape[1]
    idx_tok = _c(idx_tok, np.uint16)
    w_g = _c(w_g, np.float32)
    kb = {IDX_BF16: 2 * dI, IDX_E4M3: dI, IDX_MXFP4: dI // 2}[idx_dtype]
    fp4 = np.zeros((B, cap, D // 2), np.uint8) if fp4 is None else fp4
    scale = np.zeros((B, cap, D // group_size(scale_fmt)), np.uint8) if scale is None else scale
    assert scale.shape == (B, cap, D // group_size(scale_fmt))
    if idx_tok is not None and idx_key is None:
        idx_key = np.zeros((B, cap, kb), np.uint8)
    if idx_tok is not None and idx_dtype == IDX_MXFP4 and idx_key_scale is None:
        idx_key_scale = np.zeros((B, cap, dI // 32), np.uint8)
    pooled = np.zeros((B, cap, D), np.float32) if return_pooled else None
    pooled_idx = np.zeros((B, cap, dI), np.float32) if (return_pooled and idx_tok is not None) else None
    st = _load().orc_compress(B, D, dI, m, idx_dtype, scale_fmt, cap, _ptr(kv_tok), _ptr(idx_tok), _ptr(w_g),
                              _ptr(tok_offsets), _ptr(n_blocks), _ptr(fp4), _ptr(scale),
                              _ptr(idx_key) if idx_tok is not None else None,
                              _ptr(idx_key_scale) if idx_dtype == IDX_MXFP4 else None, _ptr(pooled),
                              _ptr(pooled_idx))
    out = dict(fp4=fp4, scale=scale, idx_key=idx_key, n_blocks=n_blocks, status=st)
    if idx_dtype == IDX_MXFP4:
        out["idx_key_scale"] = idx_key_scale
    if return_pooled:
        out["pooled"] = pooled
        out["pooled_idx"] = pooled_idx
    return out


def index_scores(idx_key, n_blocks, q_offsets, q_pos, q_idx, w, *, m, idx_dtype=IDX_BF16, idx_key_scale=None):
    """Indexer scores (row a3). idx_key [B, cap, key_bytes] uint8 (MXFP4: codes [B, cap, dI/2] and
    idx_key_scale [B, cap, dI/32]), q_idx [Nq, H_I, dI] uint16, w [Nq, H_I] float32.
    Returns (scores [Nq, cap] float32, n_vis [Nq] int32)."""
    idx_key = _c(idx_key, np.uint8)
    B, cap, _ = idx_key.shape
    q_idx = _c(q_idx, np.uint16)
    Nq, H_I, dI = q_idx.shape
    if idx_dtype == IDX_MXFP4:
        idx_key_scale = _c(idx_key_scale, np.uint8)
        assert idx_key.shape == (B, cap, dI // 2) and idx_key_scale.shape == (B, cap, dI // 32)
    scores = np.empty((Nq, cap), np.float32)
    n_vis = np.zeros(Nq, np.int32)
    _load().orc_index_scores(B, Nq, H_I, dI, idx_dtype, m, cap, _ptr(idx_key),
                             _ptr(idx_key_scale) if idx_dtype == IDX_MXFP4 else None, _ptr(_c(n_blocks, np.int32)),
                             _ptr(_c(q_offsets, np.int32)), _ptr(_c(q_pos, np.int32)), _ptr(q_idx),
                             _ptr(_c(w, np.float32)), _ptr(scores), _ptr(n_vis))
    return scores, n_vis


def topk(scores, n_vis, k):
    """Top-k block selection (row a4): ascending indices, -1 padded."""
    scores = _c(scores, np.float32)
    Nq, cap = scores.shape
    sel = np.empty((Nq, k), np.int32)
    _load().orc_topk(Nq, cap, k, _ptr(scores), _ptr(_c(n_vis, np.int32)), _ptr(sel))
    return sel


def index_pool(scores, n_vis, *, G, P):
    """Hierarchical indexer pool: the P best blocks of G entries by block-max score (ascending, -1 padded)."""
    scores = _c(scores, np.float32)
    Nq, cap = scores.shape
    pool = np.empty((Nq, P), np.int32)
    _load().orc_index_pool(Nq, cap, G, P, _ptr(scores), _ptr(_c(n_vis, np.int32)), _ptr(pool))
    return pool


def reindex_topk(scores, n_vis, pool, *, G, k):
    """Reindex-mode top-k restricted to the pool's entries (ascending, -1 padded)."""
    scores = _c(scores, np.float32)
    Nq, cap = scores.shape
    pool = _c(pool, np.int32)
    P = pool.shape[1]
    sel = np.empty((Nq, k), np.int32)
    _load().orc_reindex_topk(Nq, cap, G, P, k, _ptr(scores), _ptr(_c(n_vis, np.int32)), _ptr(pool), _ptr(sel))
    return sel


def index_topk(idx_key, n_blocks, q_offsets, q_pos, q_idx, w, *, m, k, idx_dtype=IDX_BF16, idx_key_scale=None):
    scores, n_vis = index_scores(idx_key, n_blocks, q_offsets, q_pos, q_idx, w, m=m, idx_dtype=idx_dtype,
                                 idx_key_scale=idx_key_scale)
    return topk(scores, n_vis, k), scores, n_vis


def csa_attend(fp4, scale, q_offsets, q, sel_idx, win_kv, win_start, win_len, softmax_scale, *,
               scale_fmt=SCALE_E8M0_32):
    """Joint softmax attention over the selected compressed entries + window (rows a5, a6).
    Returns (out [Nq, H, D] float64, lse [Nq, H] float64)."""
    fp4 = _c(fp4, np.uint8)
    scale = _c(scale, np.uint8)
    B, cap, half = fp4.shape
    D = half * 2
    q = _c(q, np.uint16)
    Nq, H, _ = q.shape
    sel_idx = _c(sel_idx, np.int32)
    k = sel_idx.shape[1]
    out = np.empty((Nq, H, D), np.float64)
    lse = np.empty((Nq, H), np.float64)
    win_kv = _c(win_kv if win_kv is not None else np.zeros((1, D), np.uint16), np.uint16)
    assert scale.shape == (B, cap, D // group_size(scale_fmt))
    _load().orc_csa_attend(B, Nq, H, D, cap, k, _ptr(fp4), _ptr(scale), scale_fmt, _ptr(_c(q_offsets, np.int32)),
                           _ptr(q), _ptr(sel_idx), _ptr(win_kv), _ptr(_c(win_start, np.int64)),
                           _ptr(_c(win_len, np.int32)), float(softmax_scale), _ptr(out), _ptr(lse))
    return out, lse


def hca_attend(fp4, scale, n_blocks, q_offsets, q_pos, q, win_kv, win_start, win_len, softmax_scale, *, m,
               scale_fmt=SCALE_E8M0_32):
    """Dense attention over every visible compressed entry + window (row a7)."""
    fp4 = _c(fp4, np.uint8)
    scale = _c(scale, np.uint8)
    B, cap, half = fp4.shape
    D = half * 2
    q = _c(q, np.uint16)
    Nq, H, _ = q.shape
    out = np.empty((Nq, H, D), np.float64)
    lse = np.empty((Nq, H), np.float64)
    win_kv = _c(win_kv if win_kv is not None else np.zeros((1, D), np.uint16), np.uint16)
    assert scale.shape == (B, cap, D // group_size(scale_fmt))
    _load().orc_hca_attend(B, Nq, H, D, m, cap, _ptr(fp4), _ptr(scale), scale_fmt, _ptr(_c(n_blocks, np.int32)),
                           _ptr(_c(q_offsets, np.int32)), _ptr(_c(q_pos, np.int32)), _ptr(q),
                           _ptr(win_kv), _ptr(_c(win_start, np.int64)), _ptr(_c(win_len, np.int32)),
                           float(softmax_scale), _ptr(out), _ptr(lse))
    return out, lse
