"""Python binding of libcsa: CSA / HCA / window attention over an MXFP4 KV cache on B200.

Argument marshalling only. Every step of the method runs in the CUDA kernels of
libcsa.so (built in-tree by ``python -m fp4_kv_cache_csa_b200.build``); PyTorch
is used for device memory and streams. Importing this module does not load the
library; the first call does, and raises ``CsaError`` if it is missing -- there
is no CPU fallback.

The function names mirror the C ABI in include/csa.h:
    csa_compress_quantize, csa_index_topk, csa_decode_attend, hca_decode_attend,
    csa_read_device_status (+ the workspace-size queries).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_IDX_BF16 = 0
CSA_IDX_E4M3 = 1
CSA_IDX_MXFP4 = 2

CSA_SCALE_E8M0_32 = 0  # one E8M0 scale byte per 32 elements (OCP MXFP4)
CSA_SCALE_E4M3_16 = 1  # one E4M3 scale byte per 16 elements

CSA_DEV_TOKEN_COUNT = 0x1
CSA_DEV_CAPACITY = 0x2
CSA_DEV_BAD_INDEX = 0x4
CSA_DEV_BAD_WINDOW = 0x8
CSA_DEV_TIMEOUT = 0x10

EXPORTED = (
    "csa_status_string", "csa_version", "csa_compress_quantize", "csa_index_topk_workspace", "csa_index_topk",
    "csa_attend_workspace", "csa_decode_attend", "hca_decode_attend", "csa_read_device_status",
    "csa_index_topk_noalloc", "csa_index_pool_workspace", "csa_index_topk_pool", "csa_index_reindex_workspace",
    "csa_index_topk_reindex", "csa_index_reindex_layers_workspace", "csa_index_topk_reindex_layers",
    "csa_probe_mxf4_mma",
)


class CsaError(RuntimeError):
    pass


class _CCache(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("dim", ctypes.c_int32), ("block", ctypes.c_int32), ("capacity", ctypes.c_int32),
        ("fp4", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("idx_key", ctypes.c_void_p),
        ("idx_dim", ctypes.c_int32), ("idx_dtype", ctypes.c_int32),
        ("n_blocks", ctypes.c_void_p), ("status", ctypes.c_void_p), ("scale_fmt", ctypes.c_int32),
        ("idx_key_scale", ctypes.c_void_p),
    ]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libcsa.so and declare the C signatures. Raises CsaError if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise CsaError(f"libcsa.so not found at {path}: build it with `python -m fp4_kv_cache_csa_b200.build`")
    _lib = declare(ctypes.CDLL(path))
    return _lib


def declare(lib):
    """Declare the C signatures of a loaded libcsa (the library itself or a test variant of it)."""
    P, I, S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    CP = ctypes.POINTER(_CCache)
    lib.csa_status_string.argtypes = [I]
    lib.csa_status_string.restype = ctypes.c_char_p
    lib.csa_version.argtypes = []
    lib.csa_version.restype = I
    lib.csa_compress_quantize.argtypes = [CP, P, P, P, P, I, P]
    lib.csa_compress_quantize.restype = I
    lib.csa_index_topk_workspace.argtypes = [CP, I, I]
    lib.csa_index_topk_workspace.restype = S
    lib.csa_index_topk.argtypes = [CP, P, P, I, I, P, P, I, P, P, S, P]
    lib.csa_index_topk.restype = I
    lib.csa_index_topk_noalloc.argtypes = [CP, P, P, I, I, P, P, I, P, P]
    lib.csa_index_topk_noalloc.restype = I
    lib.csa_index_pool_workspace.argtypes = [CP, I, I, I, I]
    lib.csa_index_pool_workspace.restype = S
    lib.csa_index_topk_pool.argtypes = [CP, P, P, I, I, P, P, I, P, I, I, P, P, S, P]
    lib.csa_index_topk_pool.restype = I
    lib.csa_index_reindex_workspace.argtypes = [CP, I, I, I]
    lib.csa_index_reindex_workspace.restype = S
    lib.csa_index_topk_reindex.argtypes = [CP, P, P, I, I, P, P, I, P, I, I, P, P, S, P]
    lib.csa_index_topk_reindex.restype = I
    lib.csa_index_reindex_layers_workspace.argtypes = [CP, I, I, I, I]
    lib.csa_index_reindex_layers_workspace.restype = S
    lib.csa_index_topk_reindex_layers.argtypes = [CP, P, P, I, I, I, P, P, I, P, I, I, P, P, S, P]
    lib.csa_index_topk_reindex_layers.restype = I
    lib.csa_attend_workspace.argtypes = [CP, I, I]
    lib.csa_attend_workspace.restype = S
    lib.csa_decode_attend.argtypes = [CP, P, I, I, P, P, I, P, P, P, I, ctypes.c_float, P, P, P, S, P]
    lib.csa_decode_attend.restype = I
    lib.hca_decode_attend.argtypes = [CP, P, I, I, P, P, P, P, P, I, ctypes.c_float, P, P, P, S, P]
    lib.hca_decode_attend.restype = I
    lib.csa_read_device_status.argtypes = [CP, P, ctypes.POINTER(I)]
    lib.csa_read_device_status.restype = I
    lib.csa_probe_mxf4_mma.argtypes = [I, P, P, ctypes.POINTER(ctypes.c_int64)]
    lib.csa_probe_mxf4_mma.restype = I
    return lib


def _check(status: int, what: str):
    if status != 0:
        msg = load_library().csa_status_string(status).decode()
        raise CsaError(f"{what}: {msg} (status {status})")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class Cache:
    """One compressed cache (one layer): device tensors owned by the caller (see include/csa.h).

    fp4 [B, cap, D/2] uint8, scale [B, cap, D/32] uint8 (E8M0) or [B, cap, D/16] uint8 (E4M3),
    idx_key [B, cap, dI] bf16 / uint8 (e4m3) or [B, cap, dI/2] uint8 (MXFP4 codes, with
    idx_key_scale [B, cap, dI/32] uint8) or None, n_blocks [B] int32, status [1] int32 or None.
    """
    fp4: object
    scale: object
    n_blocks: object
    block: int
    idx_key: object = None
    idx_dtype: int = CSA_IDX_BF16
    status: object = None
    scale_fmt: int = CSA_SCALE_E8M0_32
    idx_key_scale: object = None

    @property
    def batch(self) -> int:
        return self.fp4.shape[0]

    @property
    def capacity(self) -> int:
        return self.fp4.shape[1]

    @property
    def dim(self) -> int:
        return self.fp4.shape[2] * 2

    @property
    def idx_dim(self) -> int:
        if self.idx_key is None:
            return 0
        return self.idx_key.shape[2] * (2 if self.idx_dtype == CSA_IDX_MXFP4 else 1)

    def c_struct(self) -> _CCache:
        return _CCache(self.batch, self.dim, self.block, self.capacity, _ptr(self.fp4), _ptr(self.scale),
                       _ptr(self.idx_key), self.idx_dim, self.idx_dtype, _ptr(self.n_blocks), _ptr(self.status),
                       self.scale_fmt, _ptr(self.idx_key_scale))

    @staticmethod
    def allocate(batch: int, capacity: int, dim: int, block: int, idx_dim: int = 0, idx_dtype: int = CSA_IDX_BF16,
                 device="cuda", scale_fmt: int = CSA_SCALE_E8M0_32):
        """Zero-filled cache tensors on `device` (torch allocation; the library allocates nothing)."""
        import torch

        idx = idx_scale = None
        if idx_dim and idx_dtype == CSA_IDX_MXFP4:
            idx = torch.zeros(batch, capacity, idx_dim // 2, dtype=torch.uint8, device=device)
            idx_scale = torch.zeros(batch, capacity, idx_dim // 32, dtype=torch.uint8, device=device)
        elif idx_dim:
            dt = torch.bfloat16 if idx_dtype == CSA_IDX_BF16 else torch.uint8
            idx = torch.zeros(batch, capacity, idx_dim, dtype=dt, device=device)
        return Cache(fp4=torch.zeros(batch, capacity, dim // 2, dtype=torch.uint8, device=device),
                     scale=torch.zeros(batch, capacity, dim // (32 if scale_fmt == CSA_SCALE_E8M0_32 else 16),
                                       dtype=torch.uint8, device=device),
                     n_blocks=torch.zeros(batch, dtype=torch.int32, device=device), block=block,
                     idx_key=idx, idx_dtype=idx_dtype, status=torch.zeros(1, dtype=torch.int32, device=device),
                     scale_fmt=scale_fmt, idx_key_scale=idx_scale)


def csa_version() -> int:
    return load_library().csa_version()


def csa_compress_quantize(cache: Cache, kv_tok, idx_tok, gate_w, tok_offsets, stream=None):
    """Rows a1+a2: pool every m new tokens of each request into one block and store it (FP4 + indexer key)."""
    lib = load_library()
    c = cache.c_struct()
    _check(lib.csa_compress_quantize(ctypes.byref(c), _ptr(kv_tok), _ptr(idx_tok), _ptr(gate_w), _ptr(tok_offsets),
                                     int(kv_tok.shape[0]), _stream(stream)), "csa_compress_quantize")


def csa_index_topk_workspace(cache: Cache, n_queries: int, topk: int) -> int:
    return int(load_library().csa_index_topk_workspace(ctypes.byref(cache.c_struct()), n_queries, topk))


def csa_index_topk_noalloc(cache: Cache, q_idx, w, q_offsets, q_pos, topk: int, sel_idx, stream=None):
    """csa_index_topk with the library's fixed 32 MiB device scratch instead of a workspace, for
    callers that cannot allocate device memory (see include/csa.h). sel_idx must be passed in."""
    lib = load_library()
    c = cache.c_struct()
    _check(lib.csa_index_topk_noalloc(ctypes.byref(c), _ptr(q_idx), _ptr(w), int(q_idx.shape[0]),
                                      int(q_idx.shape[1]), _ptr(q_offsets), _ptr(q_pos), topk, _ptr(sel_idx),
                                      _stream(stream)), "csa_index_topk_noalloc")
    return sel_idx


def csa_attend_workspace(cache: Cache, n_queries: int, heads: int) -> int:
    return int(load_library().csa_attend_workspace(ctypes.byref(cache.c_struct()), n_queries, heads))


def _workspace(nbytes: int, workspace, device):
    import torch

    if workspace is not None:
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def csa_index_topk(cache: Cache, q_idx, w, q_offsets, q_pos, topk: int, sel_idx=None, workspace=None, stream=None):
    """Rows a3+a4: indexer scores of every visible block and the top-k blocks per query (ascending, -1 padded)."""
    import torch

    lib = load_library()
    n_queries, idx_heads = int(q_idx.shape[0]), int(q_idx.shape[1])
    if sel_idx is None:
        sel_idx = torch.empty(n_queries, topk, dtype=torch.int32, device=q_idx.device)
    need = csa_index_topk_workspace(cache, n_queries, topk)
    workspace = _workspace(need, workspace, q_idx.device)
    c = cache.c_struct()
    _check(lib.csa_index_topk(ctypes.byref(c), _ptr(q_idx), _ptr(w), n_queries, idx_heads, _ptr(q_offsets),
                              _ptr(q_pos), topk, _ptr(sel_idx), _ptr(workspace), workspace.numel(), _stream(stream)),
           "csa_index_topk")
    return sel_idx


def csa_index_pool_workspace(cache: Cache, n_queries: int, topk: int, pool_group: int = 8,
                             pool_blocks: int = 2000) -> int:
    return int(load_library().csa_index_pool_workspace(ctypes.byref(cache.c_struct()), n_queries, topk, pool_group,
                                                       pool_blocks))


def csa_index_reindex_workspace(cache: Cache, n_queries: int, pool_group: int = 8, pool_blocks: int = 2000) -> int:
    return int(load_library().csa_index_reindex_workspace(ctypes.byref(cache.c_struct()), n_queries, pool_group,
                                                          pool_blocks))


def csa_index_topk_pool(cache: Cache, q_idx, w, q_offsets, q_pos, topk: int, pool_group: int = 8,
                        pool_blocks: int = 2000, sel_idx=None, pool_blk=None, workspace=None, stream=None):
    """A Full-mode layer's indexer: its top-k (as csa_index_topk) and the candidate pool of the
    hierarchical indexer (the pool_blocks best groups of pool_group blocks by their best score)."""
    import torch

    lib = load_library()
    n_queries, idx_heads = int(q_idx.shape[0]), int(q_idx.shape[1])
    if sel_idx is None:
        sel_idx = torch.empty(n_queries, topk, dtype=torch.int32, device=q_idx.device)
    if pool_blk is None:
        pool_blk = torch.empty(n_queries, pool_blocks, dtype=torch.int32, device=q_idx.device)
    need = csa_index_pool_workspace(cache, n_queries, topk, pool_group, pool_blocks)
    workspace = _workspace(need, workspace, q_idx.device)
    c = cache.c_struct()
    _check(lib.csa_index_topk_pool(ctypes.byref(c), _ptr(q_idx), _ptr(w), n_queries, idx_heads, _ptr(q_offsets),
                                   _ptr(q_pos), topk, _ptr(sel_idx), pool_group, pool_blocks, _ptr(pool_blk),
                                   _ptr(workspace), workspace.numel(), _stream(stream)), "csa_index_topk_pool")
    return sel_idx, pool_blk


def csa_index_topk_reindex(cache: Cache, q_idx, w, q_offsets, q_pos, topk: int, pool_blk, pool_group: int = 8,
                           sel_idx=None, workspace=None, stream=None):
    """A Reindex-mode layer's indexer: its own query scored only against the pool's blocks."""
    import torch

    lib = load_library()
    n_queries, idx_heads = int(q_idx.shape[0]), int(q_idx.shape[1])
    pool_blocks = int(pool_blk.shape[1])
    if sel_idx is None:
        sel_idx = torch.empty(n_queries, topk, dtype=torch.int32, device=q_idx.device)
    need = csa_index_reindex_workspace(cache, n_queries, pool_group, pool_blocks)
    workspace = _workspace(need, workspace, q_idx.device)
    c = cache.c_struct()
    _check(lib.csa_index_topk_reindex(ctypes.byref(c), _ptr(q_idx), _ptr(w), n_queries, idx_heads, _ptr(q_offsets),
                                      _ptr(q_pos), topk, _ptr(sel_idx), pool_group, pool_blocks, _ptr(pool_blk),
                                      _ptr(workspace), workspace.numel(), _stream(stream)), "csa_index_topk_reindex")
    return sel_idx


def csa_index_reindex_layers_workspace(cache: Cache, n_queries: int, n_layers: int, pool_group: int,
                                       pool_blocks: int) -> int:
    return int(load_library().csa_index_reindex_layers_workspace(ctypes.byref(cache.c_struct()), n_queries, n_layers,
                                                                 pool_group, pool_blocks))


def csa_index_topk_reindex_layers(cache: Cache, q_idx, w, q_offsets, q_pos, topk: int, pool_blk, pool_group: int = 8,
                                  sel_idx=None, workspace=None, stream=None):
    """Several Reindex-mode layers over one pool in one call. q_idx [Nq, L, H_I, dI] bf16,
    w [Nq, L, H_I] float32; returns sel_idx [Nq, L, topk]."""
    import torch

    lib = load_library()
    n_queries, n_layers, idx_heads = (int(x) for x in q_idx.shape[:3])
    pool_blocks = int(pool_blk.shape[1])
    if sel_idx is None:
        sel_idx = torch.empty(n_queries, n_layers, topk, dtype=torch.int32, device=q_idx.device)
    need = csa_index_reindex_layers_workspace(cache, n_queries, n_layers, pool_group, pool_blocks)
    workspace = _workspace(need, workspace, q_idx.device)
    c = cache.c_struct()
    _check(lib.csa_index_topk_reindex_layers(ctypes.byref(c), _ptr(q_idx), _ptr(w), n_queries, n_layers, idx_heads,
                                             _ptr(q_offsets), _ptr(q_pos), topk, _ptr(sel_idx), pool_group,
                                             pool_blocks, _ptr(pool_blk), _ptr(workspace), workspace.numel(),
                                             _stream(stream)), "csa_index_topk_reindex_layers")
    return sel_idx


def csa_decode_attend(cache: Cache, q, q_offsets, sel_idx, win_kv=None, win_start=None, win_len=None,
                      max_win: int = 128, softmax_scale: Optional[float] = None, out=None, lse=None,
                      workspace=None, stream=None):
    """Rows a5+a6+a8: joint softmax attention over the selected compressed entries and the window."""
    import torch

    lib = load_library()
    n_queries, heads, D = (int(x) for x in q.shape)
    if softmax_scale is None:
        softmax_scale = D ** -0.5
    if out is None:
        out = torch.empty(n_queries, heads, D, dtype=torch.float32, device=q.device)
    need = csa_attend_workspace(cache, n_queries, heads)
    workspace = _workspace(need, workspace, q.device)
    c = cache.c_struct()
    _check(lib.csa_decode_attend(ctypes.byref(c), _ptr(q), n_queries, heads, _ptr(q_offsets), _ptr(sel_idx),
                                 int(sel_idx.shape[1]), _ptr(win_kv), _ptr(win_start), _ptr(win_len), max_win,
                                 float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "csa_decode_attend")
    return out


def hca_decode_attend(cache: Cache, q, q_offsets, q_pos, win_kv=None, win_start=None, win_len=None,
                      max_win: int = 128, softmax_scale: Optional[float] = None, out=None, lse=None,
                      workspace=None, stream=None):
    """Row a7 (+a8): dense attention over every visible compressed entry and the window."""
    import torch

    lib = load_library()
    n_queries, heads, D = (int(x) for x in q.shape)
    if softmax_scale is None:
        softmax_scale = D ** -0.5
    if out is None:
        out = torch.empty(n_queries, heads, D, dtype=torch.float32, device=q.device)
    need = csa_attend_workspace(cache, n_queries, heads)
    workspace = _workspace(need, workspace, q.device)
    c = cache.c_struct()
    _check(lib.hca_decode_attend(ctypes.byref(c), _ptr(q), n_queries, heads, _ptr(q_offsets), _ptr(q_pos),
                                 _ptr(win_kv), _ptr(win_start), _ptr(win_len), max_win, float(softmax_scale),
                                 _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)),
           "hca_decode_attend")
    return out


def csa_probe_mxf4_mma(iters: int, status, stream=None) -> int:
    """Launch the block-scaled MXFP4 MMA probe (one CTA per SM); returns its dense FLOPs.
    `status` is a device int32 tensor that receives CSA_DEV_TIMEOUT if completion is not seen."""
    lib = load_library()
    flops = ctypes.c_int64(0)
    _check(lib.csa_probe_mxf4_mma(int(iters), _ptr(status), _stream(stream), ctypes.byref(flops)), "csa_probe_mxf4_mma")
    return int(flops.value)


def csa_read_device_status(cache: Cache, stream=None) -> int:
    """Synchronize, return and clear the device status bits (CSA_DEV_*)."""
    lib = load_library()
    v = ctypes.c_int32(0)
    c = cache.c_struct()
    _check(lib.csa_read_device_status(ctypes.byref(c), _stream(stream), ctypes.byref(v)), "csa_read_device_status")
    return int(v.value)
