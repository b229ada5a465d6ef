"""Seeded synthetic inputs shared by the tests and the benchmark.

This module only draws random numbers and stores them in the library's input
formats (bf16 bit patterns, E4M3 bytes, raw cache bytes). It holds none of the
method's arithmetic: no pooling, gating, quantization, scoring, selection or
attention. Conversions to bf16 / float8_e4m3fn use PyTorch's own casts.

Workload shapes (all per layer; D = latent dim shared by K and V, m = block size,
W = window, H_I x d_I = indexer heads x dim, k = top-k):

  csa_tiny_4k    1 request, 4096-token context, 16 heads, D=128, m=4 (1024 blocks),
                 W=128, indexer 4x64 bf16, k=64; N(0,1) data, gate weights N(0, 0.02^2)
  csa_b8_64k     8 requests x 65536 tokens, 64 heads, D=512, m=4 (16384 blocks),
                 indexer 4x128 bf16, k=512, W=128; N(0,1) with a per-channel
                 LogNormal(0, 0.5) scale on every activation tensor
  csa_b32_1m     32 requests, context uniform in [524288, 1048576] tokens,
                 m=4 (<= 262144 blocks), D=512, 64 heads, indexer 4x128 e4m3 keys,
                 k=1024, W=128; N(0,1) data
  hca_b64_1m     64 requests x 1048576 tokens, m=128 (8192 blocks), D=512, 64 heads,
                 W=128, dense over every block
  prefill_b4_8k  4 requests, 8192 new tokens appended to 65536 existing ones,
                 m=4 (18432 blocks), D=512, 64 heads, indexer 4x128, k=512, W=128
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

SEED = 0x5EED0C5A


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    ctx_min: int
    ctx_max: int
    heads: int
    dim: int
    block: int
    window: int
    idx_heads: int
    idx_dim: int
    idx_dtype: int  # 0 bf16, 1 e4m3
    topk: int
    channel_lognormal: float = 0.0


WORKLOADS = {
    "csa_tiny_4k": Workload("csa_tiny_4k", 1, 4096, 4096, 16, 128, 4, 128, 4, 64, 0, 64),
    "csa_b8_64k": Workload("csa_b8_64k", 8, 65536, 65536, 64, 512, 4, 128, 4, 128, 0, 512, 0.5),
    "csa_b32_1m": Workload("csa_b32_1m", 32, 524288, 1048576, 64, 512, 4, 128, 4, 128, 1, 1024),
    "hca_b64_1m": Workload("hca_b64_1m", 64, 1048576, 1048576, 64, 512, 128, 128, 0, 0, 0, 0),
    # ctx_min = tokens already in the cache, ctx_max = after the 8192 new ones
    "prefill_b4_8k": Workload("prefill_b4_8k", 4, 65536, 65536 + 8192, 64, 512, 4, 128, 4, 128, 0, 512),
}


def generator(*ids: int) -> np.random.Generator:
    """Counter-based Philox4x32 stream keyed by (SEED, *ids)."""
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([SEED, *ids])))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16) with PyTorch's round-to-nearest-even cast."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    """float32 -> float8_e4m3fn bytes with PyTorch's cast (inputs must be within +-448)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def normal_bf16(shape, *ids, std: float = 1.0, channel_lognormal: float = 0.0) -> np.ndarray:
    """N(0, std^2) values as bf16 bits; optionally times a per-channel LogNormal(0, s) scale."""
    g = generator(*ids)
    x = g.standard_normal(shape, dtype=np.float32) * np.float32(std)
    if channel_lognormal:
        c = generator(*ids, 1).lognormal(0.0, channel_lognormal, size=shape[-1]).astype(np.float32)
        x = x * c
    return to_bf16_bits(x)


def normal_f32(shape, *ids, std: float = 1.0) -> np.ndarray:
    return (generator(*ids).standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def context_lengths(wl: Workload, *ids: int) -> np.ndarray:
    """Per-request context lengths: uniform integers in [ctx_min, ctx_max]."""
    if wl.ctx_min == wl.ctx_max:
        return np.full(wl.batch, wl.ctx_min, np.int64)
    return generator(*ids).integers(wl.ctx_min, wl.ctx_max, size=wl.batch, endpoint=True).astype(np.int64)


def random_cache_bytes(n_rows: int, dim: int, *ids: int, scale_lo: int = 123, scale_hi: int = 126):
    """Raw MXFP4 cache rows drawn directly as bytes: uniform code bytes and E8M0
    scale bytes uniform in [scale_lo, scale_hi] (the range a pooled N(0,1)
    block lands in). Returns (fp4 [n, dim/2] u8, scale [n, dim/32] u8)."""
    g = generator(*ids)
    fp4 = g.integers(0, 256, size=(n_rows, dim // 2), dtype=np.uint8)
    sc = g.integers(scale_lo, scale_hi, size=(n_rows, dim // 32), endpoint=True, dtype=np.uint8)
    return fp4, sc


def random_cache_bytes_e4m3x16(n_rows: int, dim: int, *ids: int, scale_lo: int = 0x1C, scale_hi: int = 0x2C):
    """Raw FP4 cache rows with one E4M3 scale byte per 16 elements, drawn as
    bytes: uniform code bytes and scale bytes uniform in [scale_lo, scale_hi]
    (0x1C .. 0x2C spans the scales a pooled N(0,1) group lands in). Returns
    (fp4 [n, dim/2] u8, scale [n, dim/16] u8)."""
    g = generator(*ids)
    fp4 = g.integers(0, 256, size=(n_rows, dim // 2), dtype=np.uint8)
    sc = g.integers(scale_lo, scale_hi, size=(n_rows, dim // 16), endpoint=True, dtype=np.uint8)
    return fp4, sc


def decode_inputs(wl: Workload, n_queries_per_req: int = 1, *, seed_base: int = 100):
    """Per-query decode tensors: q [Nq, H, D] bf16, q_idx [Nq, H_I, d_I] bf16,
    w [Nq, H_I] f32 (N(0,1)/sqrt(H_I))."""
    Nq = wl.batch * n_queries_per_req
    q = normal_bf16((Nq, wl.heads, wl.dim), seed_base, 1, channel_lognormal=wl.channel_lognormal)
    out = {"q": q}
    if wl.idx_heads:
        out["q_idx"] = normal_bf16((Nq, wl.idx_heads, wl.idx_dim), seed_base, 2,
                                   channel_lognormal=wl.channel_lognormal)
        out["w"] = normal_f32((Nq, wl.idx_heads), seed_base, 3, std=1.0 / np.sqrt(wl.idx_heads))
    return out
