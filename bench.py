#!/usr/bin/env python
"""Benchmark: CSA + HCA decode over an MXFP4 KV cache at 512K-1M context on B200.

One step = one decode token for every request of the batch through one CSA layer
and one HCA layer (the CSA/HCA alternation), i.e. every row of the hot path:
  a1+a2  csa_compress_quantize: the 4 newest tokens -> one CSA block (MXFP4 + e4m3 key),
         the 128 newest tokens -> one HCA block
  a3+a4  csa_index_topk over every visible CSA block (k = 1024)
  a5+a6+a8 csa_decode_attend: selected blocks + 128-token bf16 window, one joint softmax
  a7     hca_decode_attend: every HCA block + the window
Workload (default, per GPU): 32 requests, context lengths uniform in [512K, 1M]
tokens (multiples of 128), D = 512 shared latent, 64 query heads, indexer 4 x 128
with e4m3 keys, k = 1024, W = 128. Synthetic data (seeded torch RNG on the GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). With N > 1 every rank runs its own independent
batch (weak scaling, no data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B, D, H, M_CSA, M_HCA, W = 32, 512, 64, 4, 128, 128
H_I, D_I, TOPK = 4, 128, 1024
POOL_GROUP, POOL_BLOCKS = 8, 2000  # hierarchical indexer pool: ~2000 blocks of 8 entries
REINDEX_LAYERS = 3  # Reindex layers timed together in one call (after the Full layer that keeps the pool)
CTX_MIN, CTX_MAX = 524288, 1048576
CAP_CSA, CAP_HCA = CTX_MAX // M_CSA, CTX_MAX // M_HCA
OUR_KERNELS_PER_STEP = 12  # compress 2x(pool, commit); index: scan (own schedule), merge; attend 2x(schedule, main, merge)
SEED = 0x5EED0C5A


SCALE_FMT = 0  # 0: one E8M0 scale per 32 elements (MXFP4, the headline format); 1: one E4M3 scale per 16
SCALE_FMT_NAMES = {"e8m0x32": 0, "e4m3x16": 1}


def set_batch(n: int):
    global B
    B = int(n)


def set_prefill_requests(n: int):
    """Requests of the prefill workload (4; fewer only for profiling a smaller case)."""
    Prefill.B = int(n)


def set_scale_fmt(name: str):
    global SCALE_FMT
    SCALE_FMT = SCALE_FMT_NAMES[name]


def scale_group() -> int:
    return 32 if SCALE_FMT == 0 else 16


def scale_fmt_name() -> str:
    return {v: k for k, v in SCALE_FMT_NAMES.items()}[SCALE_FMT]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------------------- workload
def context_lengths(rank: int) -> np.ndarray:
    from fp4_kv_cache_csa_b200 import datagen

    g = datagen.generator(1000 + rank)
    return (g.integers(CTX_MIN // 128, CTX_MAX // 128, size=32, endpoint=True) * 128).astype(np.int64)[:B]


class Workload:
    """Device-resident caches and per-step inputs for one rank."""

    def __init__(self, rank: int, device):
        import torch

        import fp4_kv_cache_csa_b200 as csa

        self.T = context_lengths(rank)
        n_csa = self.T // M_CSA           # blocks after this step's append
        n_hca = self.T // M_HCA
        self.n_csa, self.n_hca = n_csa, n_hca
        gen = torch.Generator(device=device)
        gen.manual_seed(SEED + rank)
        self.csa = csa.Cache.allocate(B, CAP_CSA, D, M_CSA, D_I, csa.CSA_IDX_E4M3, device, scale_fmt=SCALE_FMT)
        self.hca = csa.Cache.allocate(B, CAP_HCA, D, M_HCA, 0, csa.CSA_IDX_BF16, device, scale_fmt=SCALE_FMT)
        # scale bytes in the range pooled N(0,1) groups land in: E8M0 123..126, E4M3 0x1C..0x2C
        s_lo, s_hi = (123, 127) if SCALE_FMT == 0 else (0x1C, 0x2D)
        for cache, n in ((self.csa, n_csa), (self.hca, n_hca)):
            for b in range(B):
                nb = int(n[b])
                cache.fp4[b, :nb].random_(0, 256, generator=gen)
                cache.scale[b, :nb].random_(s_lo, s_hi, generator=gen)
                if cache.idx_key is not None:
                    k = torch.randn(nb, D_I, device=device, generator=gen) * 0.5
                    cache.idx_key[b, :nb] = k.to(torch.float8_e4m3fn).view(torch.uint8)
        self.base_csa = torch.tensor(n_csa - 1, dtype=torch.int32, device=device)
        self.base_hca = torch.tensor(n_hca - 1, dtype=torch.int32, device=device)
        bf = torch.bfloat16
        self.kv4 = torch.randn(B * M_CSA, D, device=device, generator=gen).to(bf)
        self.idx4 = torch.randn(B * M_CSA, D_I, device=device, generator=gen).to(bf)
        self.kv128 = torch.randn(B * M_HCA, D, device=device, generator=gen).to(bf)
        self.gate_w = (torch.randn(D, device=device, generator=gen) * 0.02).float()
        self.offs4 = torch.arange(0, B * M_CSA + 1, M_CSA, dtype=torch.int32, device=device)
        self.offs128 = torch.arange(0, B * M_HCA + 1, M_HCA, dtype=torch.int32, device=device)
        self.q_csa = torch.randn(B, H, D, device=device, generator=gen).to(bf)
        self.q_hca = torch.randn(B, H, D, device=device, generator=gen).to(bf)
        self.q_idx = torch.randn(B, H_I, D_I, device=device, generator=gen).to(bf)
        self.w = (torch.randn(B, H_I, device=device, generator=gen) / math.sqrt(H_I)).float()
        self.q_offsets = torch.arange(B + 1, dtype=torch.int32, device=device)
        self.q_pos = torch.tensor(self.T - 1, dtype=torch.int32, device=device)
        self.win = torch.randn(B * W, D, device=device, generator=gen).to(bf)
        self.win_start = torch.arange(0, B * W, W, dtype=torch.int64, device=device)
        self.win_len = torch.full((B,), W, dtype=torch.int32, device=device)
        self.sel = torch.empty(B, TOPK, dtype=torch.int32, device=device)
        self.out_csa = torch.empty(B, H, D, dtype=torch.float32, device=device)
        self.out_hca = torch.empty(B, H, D, dtype=torch.float32, device=device)
        self.lse = torch.empty(B, H, dtype=torch.float32, device=device)
        self.ws_idx = torch.empty(csa.csa_index_topk_workspace(self.csa, B, TOPK), dtype=torch.uint8, device=device)
        nws = max(csa.csa_attend_workspace(self.csa, B, H), csa.csa_attend_workspace(self.hca, B, H))
        self.ws_att = torch.empty(nws, dtype=torch.uint8, device=device)
        self.scale = D ** -0.5
        # CSA2: a Reindex-mode layer's own indexer query over the Full layer's pool
        self.q_idx_re = torch.randn(B, H_I, D_I, device=device, generator=gen).to(bf)
        self.w_re = (torch.randn(B, H_I, device=device, generator=gen) / math.sqrt(H_I)).float()
        self.sel_pool = torch.empty(B, TOPK, dtype=torch.int32, device=device)
        self.sel_re = torch.empty(B, TOPK, dtype=torch.int32, device=device)
        self.pool = torch.empty(B, POOL_BLOCKS, dtype=torch.int32, device=device)
        self.ws_pool = torch.empty(csa.csa_index_pool_workspace(self.csa, B, TOPK, POOL_GROUP, POOL_BLOCKS),
                                   dtype=torch.uint8, device=device)
        self.ws_re = torch.empty(csa.csa_index_reindex_workspace(self.csa, B, POOL_GROUP, POOL_BLOCKS),
                                 dtype=torch.uint8, device=device)
        # three Reindex layers over the same pool in one call
        self.q_idx_re3 = torch.randn(B, REINDEX_LAYERS, H_I, D_I, device=device, generator=gen).to(bf)
        self.w_re3 = (torch.randn(B, REINDEX_LAYERS, H_I, device=device, generator=gen) / math.sqrt(H_I)).float()
        self.sel_re3 = torch.empty(B, REINDEX_LAYERS, TOPK, dtype=torch.int32, device=device)
        self.ws_re3 = torch.empty(csa.csa_index_reindex_layers_workspace(self.csa, B, REINDEX_LAYERS, POOL_GROUP,
                                                                         POOL_BLOCKS), dtype=torch.uint8, device=device)

    def stage_index_pool(self):
        import fp4_kv_cache_csa_b200 as csa

        csa.csa_index_topk_pool(self.csa, self.q_idx, self.w, self.q_offsets, self.q_pos, TOPK, POOL_GROUP,
                                POOL_BLOCKS, sel_idx=self.sel_pool, pool_blk=self.pool, workspace=self.ws_pool)

    def stage_index_reindex(self):
        import fp4_kv_cache_csa_b200 as csa

        csa.csa_index_topk_reindex(self.csa, self.q_idx_re, self.w_re, self.q_offsets, self.q_pos, TOPK, self.pool,
                                   POOL_GROUP, sel_idx=self.sel_re, workspace=self.ws_re)

    def stage_index_reindex_layers(self):
        import fp4_kv_cache_csa_b200 as csa

        csa.csa_index_topk_reindex_layers(self.csa, self.q_idx_re3, self.w_re3, self.q_offsets, self.q_pos, TOPK,
                                          self.pool, POOL_GROUP, sel_idx=self.sel_re3, workspace=self.ws_re3)

    def bytes_reindex(self) -> float:
        """Keys of the pool's entries (about POOL_GROUP * POOL_BLOCKS per request), query, output."""
        pooled = np.minimum(self.n_csa, POOL_GROUP * POOL_BLOCKS).astype(np.float64)
        return float(np.sum(pooled)) * D_I + B * (H_I * D_I * 2 + H_I * 4 + TOPK * 4 + POOL_BLOCKS * 4)

    def stages(self):
        return (self.stage_compress, self.stage_index, self.stage_attend_csa, self.stage_attend_hca)

    # the stages of one step; every launch is one of libcsa's kernels, a memset or the n_blocks reset copy
    def stage_compress(self):
        import fp4_kv_cache_csa_b200 as csa

        self.csa.n_blocks.copy_(self.base_csa)
        self.hca.n_blocks.copy_(self.base_hca)
        csa.csa_compress_quantize(self.csa, self.kv4, self.idx4, self.gate_w, self.offs4)
        csa.csa_compress_quantize(self.hca, self.kv128, None, self.gate_w, self.offs128)

    def stage_index(self):
        import fp4_kv_cache_csa_b200 as csa

        csa.csa_index_topk(self.csa, self.q_idx, self.w, self.q_offsets, self.q_pos, TOPK, sel_idx=self.sel,
                           workspace=self.ws_idx)

    def stage_attend_csa(self):
        import fp4_kv_cache_csa_b200 as csa

        csa.csa_decode_attend(self.csa, self.q_csa, self.q_offsets, self.sel, self.win, self.win_start, self.win_len,
                              max_win=W, softmax_scale=self.scale, out=self.out_csa, lse=self.lse,
                              workspace=self.ws_att)

    def stage_attend_hca(self):
        import fp4_kv_cache_csa_b200 as csa

        csa.hca_decode_attend(self.hca, self.q_hca, self.q_offsets, self.q_pos, self.win, self.win_start,
                              self.win_len, max_win=W, softmax_scale=self.scale, out=self.out_hca,
                              workspace=self.ws_att)

    # algorithmic HBM bytes: what the method must move at least once per step
    def key_bytes(self) -> float:
        return float(np.sum(self.n_csa)) * D_I

    def bytes_index(self) -> float:
        keys = float(np.sum(self.n_csa)) * D_I
        return keys + B * (H_I * D_I * 2 + H_I * 4 + TOPK * 4)

    def bytes_csa_layer(self) -> float:
        """The CSA layer's read/write set at decode: indexer keys, the selected entries, window, q, out."""
        entry = D // 2 + D // scale_group()
        sel = float(np.sum(np.minimum(self.n_csa, TOPK))) * entry
        return self.bytes_index() + sel + B * (W * D * 2 + H * D * 2 + H * D * 4)

    def bytes_step(self) -> float:
        entry = D // 2 + D // scale_group()
        sel = float(np.sum(np.minimum(self.n_csa, TOPK))) * entry
        hca = float(np.sum(self.n_hca)) * entry
        win = 2.0 * B * W * D * 2
        q = 2.0 * B * H * D * 2
        out = 2.0 * B * H * D * 4
        comp = B * (M_CSA * (D + D_I) * 2 + entry + D_I) + B * (M_HCA * D * 2 + entry)
        return self.bytes_index() + sel + hca + win + q + out + comp

    def step_inputs(self):
        """Per-step inputs a caller streams in (new tokens, queries) and the outputs it reads back."""
        ins = [self.kv4, self.idx4, self.kv128, self.q_csa, self.q_hca, self.q_idx, self.w]
        outs = [self.out_csa, self.out_hca]
        return ins, outs


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of this rank's GPU, read (never set) through NVML every
    2 ms by a separate sampler process (a thread of this process would wait for the
    interpreter lock while the timed loop runs), so that even a short timed region has samples;
    falls back to `nvidia-smi --query-gpu ... -lms 100`. The timed region is marked with
    mark_start() / mark_end() (CLOCK_MONOTONIC after a device synchronize) and the summary uses
    the samples inside it."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    SCRIPT = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
uuid, pci, period = sys.argv[1], sys.argv[2], float(sys.argv[3])
try:
    h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
except Exception:
    h = pynvml.nvmlDeviceGetHandleByPciBusId(pci)
reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
    pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
print("ready", flush=True)
while True:
    t = time.monotonic()
    print(t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx, int(reasons(h)), flush=True)
    time.sleep(period)
"""

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.device_index, self.period = device_index, period_s
        self.samples = []  # (t, sm_mhz, max_mhz, reasons bitmask)
        self.t0 = self.t1 = None
        self.proc = None
        self.source = None

    def start(self):
        import torch

        props = torch.cuda.get_device_properties(self.device_index)
        uuid = f"GPU-{props.uuid}"
        pci = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", self.SCRIPT, uuid, pci, str(self.period)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            first = self.proc.stdout.readline()
            if not first.startswith("ready"):
                raise OSError("nvml sampler did not start")
            self.source = "nvml"

            def parse(line):
                p = line.split()
                if len(p) == 4:
                    self.samples.append((float(p[0]), float(p[1]), float(p[2]), int(p[3])))
        except OSError:
            if self.proc:
                self.proc.kill()
            q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            try:
                self.proc = subprocess.Popen(["nvidia-smi", f"--id={pci}", f"--query-gpu={q}",
                                              "--format=csv,noheader,nounits", "-lms", "100"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
                return
            self.source = "nvidia-smi"

            def parse(line):
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 6 and p[0].replace(".", "").isdigit():
                    bits = sum(b for (_, b), v in zip(self.REASONS, p[2:6]) if v.lower().startswith("active"))
                    mx = float(p[1]) if p[1].replace(".", "").isdigit() else 1965.0
                    self.samples.append((time.monotonic(), float(p[0]), mx, bits))

        def loop():
            for line in self.proc.stdout:
                parse(line)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def stop(self):
        if self.proc:
            time.sleep(3 * self.period)  # the sampler's reading of the region's end
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if getattr(self, "thread", None):
            self.thread.join(timeout=5)

    def summary(self):
        inside = [x for x in self.samples if self.t0 is not None and self.t0 <= x[0] <= self.t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": self.source}
        reasons = sorted({name for x in inside for name, bit in self.REASONS if x[3] & bit})
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": max(x[2] for x in inside),
                "reasons": reasons, "samples": len(inside), "source": self.source,
                "window_ms": (self.t1 - self.t0) * 1e3}


# ----------------------------------------------------------------------------- oracle baseline
def cpu_baseline(n_requests: int = 2):
    """The oracle (plain C, double precision, OpenMP over independent units) doing the step's work for a
    bounded sample of requests: compress of the new CSA and HCA blocks, indexer + top-k over the full
    visible key cache, CSA attention, HCA attention. Returns (tokens/s, cores, sample description)."""
    import oracle
    from fp4_kv_cache_csa_b200 import datagen

    T = context_lengths(0)[:n_requests]
    total = 0.0
    for r in range(n_requests):
        n_csa, n_hca = int(T[r] // M_CSA), int(T[r] // M_HCA)
        keys = datagen.to_e4m3_bytes(datagen.normal_f32((1, n_csa, D_I), 2000 + r, 1, std=0.5))
        gen_cache = datagen.random_cache_bytes if SCALE_FMT == 0 else datagen.random_cache_bytes_e4m3x16
        fp4, sc = gen_cache(n_csa, D, 2000 + r, 2)
        hfp4, hsc = gen_cache(n_hca, D, 2000 + r, 3)
        kv4 = datagen.normal_bf16((M_CSA, D), 2000 + r, 4)
        idx4 = datagen.normal_bf16((M_CSA, D_I), 2000 + r, 5)
        kv128 = datagen.normal_bf16((M_HCA, D), 2000 + r, 6)
        wg = datagen.normal_f32((D,), 2000 + r, 7, std=0.02)
        q = datagen.normal_bf16((1, H, D), 2000 + r, 8)
        q_idx = datagen.normal_bf16((1, H_I, D_I), 2000 + r, 9)
        w = datagen.normal_f32((1, H_I), 2000 + r, 10, std=0.5)
        win = datagen.normal_bf16((W, D), 2000 + r, 11)
        fp4 = fp4.reshape(1, n_csa, D // 2)
        sc = sc.reshape(1, n_csa, D // scale_group())
        hfp4 = hfp4.reshape(1, n_hca, D // 2)
        hsc = hsc.reshape(1, n_hca, D // scale_group())
        qo, qp = np.array([0, 1], np.int32), np.array([T[r] - 1], np.int32)
        ws, wl = np.array([0], np.int64), np.array([W], np.int32)
        t0 = time.perf_counter()
        oracle.compress(kv4, idx4, wg, np.array([0, M_CSA], np.int32), np.array([n_csa - 1], np.int32), m=M_CSA,
                        cap=n_csa, idx_dtype=1, scale_fmt=SCALE_FMT, fp4=fp4, scale=sc, idx_key=keys)
        oracle.compress(kv128, None, wg, np.array([0, M_HCA], np.int32), np.array([n_hca - 1], np.int32), m=M_HCA,
                        cap=n_hca, scale_fmt=SCALE_FMT, fp4=hfp4, scale=hsc)
        sel, _, _ = oracle.index_topk(keys, np.array([n_csa], np.int32), qo, qp, q_idx, w, m=M_CSA, k=TOPK,
                                      idx_dtype=1)
        oracle.csa_attend(fp4, sc, qo, q, sel, win, ws, wl, D ** -0.5, scale_fmt=SCALE_FMT)
        oracle.hca_attend(hfp4, hsc, np.array([n_hca], np.int32), qo, qp, q, win, ws, wl, D ** -0.5, m=M_HCA,
                          scale_fmt=SCALE_FMT)
        total += time.perf_counter() - t0
    return n_requests / total, oracle.num_threads(), \
        f"{n_requests} of the {B} requests of one step (contexts {', '.join(str(int(t)) for t in T)} tokens)"


# ----------------------------------------------------------------------------- main
class Prefill:
    """prefill_b4_8k: 4 requests with 16384 cached blocks (seeded bytes) receive 8192 new
    tokens each (2048 blocks); every new token is a query at its own position, causal at
    block granularity, with the 128 raw tokens ending at it as its window. Timed apart
    from the decode step, with its own caches."""

    B, T0, NEW, TOPK = 4, 65536, 8192, 512

    def __init__(self, device, idx_dtype=0):
        import torch

        import fp4_kv_cache_csa_b200 as csa

        B, T0, NEW = self.B, self.T0, self.NEW
        self.n0, self.cap = T0 // M_CSA, (T0 + NEW) // M_CSA
        gen = torch.Generator(device=device)
        gen.manual_seed(SEED + 4)
        bf = torch.bfloat16
        self.cache = csa.Cache.allocate(B, self.cap, D, M_CSA, D_I, idx_dtype, device, scale_fmt=SCALE_FMT)
        s_lo, s_hi = (123, 127) if SCALE_FMT == 0 else (0x1C, 0x2D)
        self.cache.fp4[:, :self.n0].random_(0, 256, generator=gen)
        self.cache.scale[:, :self.n0].random_(s_lo, s_hi, generator=gen)
        if idx_dtype == csa.CSA_IDX_MXFP4:  # E2M1 codes and E8M0 scales as the pooling writes them
            self.cache.idx_key[:, :self.n0].random_(0, 256, generator=gen)
            self.cache.idx_key_scale[:, :self.n0].random_(122, 127, generator=gen)
        else:
            self.cache.idx_key[:, :self.n0] = (torch.randn(B, self.n0, D_I, device=device, generator=gen) * 0.5).to(bf)
        self.base = torch.full((B,), self.n0, dtype=torch.int32, device=device)
        Nq = B * NEW
        self.Nq = Nq
        self.kv = torch.randn(Nq, D, device=device, generator=gen).to(bf)
        self.idx = torch.randn(Nq, D_I, device=device, generator=gen).to(bf)
        self.gate_w = (torch.randn(D, device=device, generator=gen) * 0.02).float()
        self.offs = torch.arange(0, Nq + 1, NEW, dtype=torch.int32, device=device)
        self.q_pos = torch.arange(T0, T0 + NEW, dtype=torch.int32, device=device).repeat(B)
        self.q_idx = torch.randn(Nq, H_I, D_I, device=device, generator=gen).to(bf)
        self.w = (torch.randn(Nq, H_I, device=device, generator=gen) / math.sqrt(H_I)).float()
        self.q = torch.randn(Nq, H, D, device=device, generator=gen).to(bf)
        rows = NEW + W - 1  # the 127 raw tokens before the new ones, then the new ones
        self.win = torch.empty(B * rows, D, dtype=bf, device=device)
        for b in range(B):
            self.win[b * rows:b * rows + W - 1] = torch.randn(W - 1, D, device=device, generator=gen).to(bf)
            self.win[b * rows + W - 1:(b + 1) * rows] = self.kv[b * NEW:(b + 1) * NEW]
        i = torch.arange(Nq, device=device)
        self.win_start = (i // NEW * rows + i % NEW).to(torch.int64)
        self.win_len = torch.full((Nq,), W, dtype=torch.int32, device=device)
        self.sel = torch.empty(Nq, self.TOPK, dtype=torch.int32, device=device)
        self.out = torch.empty(Nq, H, D, dtype=torch.float32, device=device)
        self.ws_idx = torch.empty(csa.csa_index_topk_workspace(self.cache, Nq, self.TOPK), dtype=torch.uint8,
                                  device=device)
        self.ws_att = torch.empty(csa.csa_attend_workspace(self.cache, Nq, H), dtype=torch.uint8, device=device)

    def stages(self):
        return (self.stage_compress, self.stage_index, self.stage_attend)

    def stage_compress(self):
        import fp4_kv_cache_csa_b200 as csa

        self.cache.n_blocks.copy_(self.base)
        csa.csa_compress_quantize(self.cache, self.kv, self.idx, self.gate_w, self.offs)

    def stage_index(self):
        import fp4_kv_cache_csa_b200 as csa

        csa.csa_index_topk(self.cache, self.q_idx, self.w, self.offs, self.q_pos, self.TOPK, sel_idx=self.sel,
                           workspace=self.ws_idx)

    def stage_attend(self):
        import fp4_kv_cache_csa_b200 as csa

        csa.csa_decode_attend(self.cache, self.q, self.offs, self.sel, self.win, self.win_start, self.win_len,
                              max_win=W, softmax_scale=D ** -0.5, out=self.out, workspace=self.ws_att)

    def index_flops(self) -> float:
        """Indexer contraction, causal: sum over queries of n_vis * H_I * d_I * 2."""
        t = np.arange(self.NEW, dtype=np.float64)
        n_vis = np.floor((self.T0 + t + 1) / M_CSA)
        return float(self.B * np.sum(n_vis)) * H_I * D_I * 2


def measure_prefill(device, stream, flush, steps: int = 3):
    """Per-stage CUDA-event times of the prefill workload (cold L2 before each pass)."""
    import torch

    import fp4_kv_cache_csa_b200 as csa

    pf = Prefill(device)
    torch.cuda.synchronize()  # the inputs were written on the default stream
    with torch.cuda.stream(stream):
        for fn in pf.stages():  # warm-up pass
            fn()
    stream.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    with torch.cuda.stream(stream):
        for k in range(steps):
            flush.zero_()
            for s_, fn in enumerate(pf.stages()):
                ev[k][s_].record(stream)
                fn()
            ev[k][3].record(stream)
    stream.synchronize()
    st = np.array([[ev[k][s_].elapsed_time(ev[k][s_ + 1]) for s_ in range(3)] for k in range(steps)]).mean(axis=0)
    status = csa.csa_read_device_status(pf.cache, stream)
    res = {"workload": f"prefill_b{pf.B}_8k", "queries": pf.Nq, "ms": float(st.sum()),
           "stage_ms": {"compress": float(st[0]), "index_topk": float(st[1]), "attend": float(st[2])},
           "index_gflop": pf.index_flops() / 1e9,
           "index_tflops": pf.index_flops() / (st[1] * 1e-3) / 1e12,
           "index_workspace_mb": pf.ws_idx.numel() / 1e6, "device_status": int(status)}
    del pf
    torch.cuda.empty_cache()
    return res


def measure_mxf4_peak(device, stream, iters: int = 4000, reps: int = 5):
    """Dense TFLOP/s of the block-scaled MXFP4 MMA (kind::mxf4, M 128 x N 256 x K 64) issued
    back to back on every SM from resident tiles (the library's MMA probe), best of `reps`;
    (None, reason) if the probe reports a timeout."""
    import torch

    import fp4_kv_cache_csa_b200 as csa

    status = torch.zeros(1, dtype=torch.int32, device=device)
    best = None
    with torch.cuda.stream(stream):
        flops = csa.csa_probe_mxf4_mma(iters // 4, status, stream)  # warm-up
        for _ in range(reps):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            flops = csa.csa_probe_mxf4_mma(iters, status, stream)
            b_.record(stream)
            b_.synchronize()
            t = flops / (a_.elapsed_time(b_) * 1e-3) / 1e12
            best = t if best is None else max(best, t)
    stream.synchronize()
    if int(status.item()) != 0:
        return None, "probe timeout"
    return best, "measured (block-scaled MMA probe, every SM, resident tiles)"


def measure_prefill_index_mxfp4(device, stream, flush, steps: int = 3):
    """The prefill_b4_8k indexer stage with MXFP4 indexer keys: the block-scaled tensor-core
    GEMM (kind::mxf4) writes the score rows, then the same selection as with bf16 keys."""
    import torch

    import fp4_kv_cache_csa_b200 as csa

    pf = Prefill(device, idx_dtype=csa.CSA_IDX_MXFP4)
    torch.cuda.synchronize()  # the inputs were written on the default stream
    with torch.cuda.stream(stream):
        pf.stage_compress()
        pf.stage_index()
    stream.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    with torch.cuda.stream(stream):
        for k in range(steps):
            flush.zero_()
            ev[k][0].record(stream)
            pf.stage_index()
            ev[k][1].record(stream)
    stream.synchronize()
    ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    status = csa.csa_read_device_status(pf.cache, stream)
    fp4_peak, kind = measure_mxf4_peak(device, stream)
    if fp4_peak is None:  # fall back to the measured bf16 peak x the nominal ratio
        bf16_peak, bkind = measured_bf16_tflops()
        fp4_peak, kind = 4.0 * bf16_peak, f"{bkind} bf16 x 4 (nominal MXFP4 : bf16 ratio; {kind})"
    flops = pf.index_flops()
    res = {"workload": f"prefill_b{pf.B}_8k", "idx_dtype": "mxfp4", "queries": pf.Nq, "index_ms": ms,
           "index_gflop": flops / 1e9, "index_tflops": flops / (ms * 1e-3) / 1e12,
           "mxfp4_peak_tflops": fp4_peak, "peak_kind": kind,
           "frac_of_mxfp4_peak": flops / (ms * 1e-3) / 1e12 / fp4_peak,
           "score_bytes": 4.0 * pf.index_flops() / (H_I * D_I * 2), "index_workspace_mb": pf.ws_idx.numel() / 1e6,
           "device_status": int(status)}
    del pf
    torch.cuda.empty_cache()
    return res


class ConfigRun:
    """One of the other decode workloads, timed apart from the step: its own caches (drawn
    bytes, as in the step), one CSA layer (indexer + top-k + attention) or one HCA layer."""

    def __init__(self, device, name, B_, T, H_, D_, m, d_i, idx_dtype, k, lognormal=0.0):
        import torch

        import fp4_kv_cache_csa_b200 as csa

        self.name, self.B, self.T, self.H, self.D, self.m, self.d_i, self.k = name, B_, T, H_, D_, m, d_i, k
        self.n = T // m
        gen = torch.Generator(device=device)
        gen.manual_seed(SEED + 7 + B_)
        bf = torch.bfloat16

        def act(*shape, std=1.0):
            x = torch.randn(*shape, device=device, generator=gen) * std
            if lognormal:
                x = x * torch.exp(torch.randn(shape[-1], device=device, generator=gen) * lognormal)
            return x

        self.cache = csa.Cache.allocate(B_, self.n, D_, m, d_i, idx_dtype, device, scale_fmt=SCALE_FMT)
        s_lo, s_hi = (123, 127) if SCALE_FMT == 0 else (0x1C, 0x2D)
        self.cache.fp4.random_(0, 256, generator=gen)
        self.cache.scale.random_(s_lo, s_hi, generator=gen)
        self.cache.n_blocks.fill_(self.n)
        if d_i:
            keys = act(B_, self.n, d_i, std=0.5)
            self.cache.idx_key.copy_(keys.to(bf) if idx_dtype == csa.CSA_IDX_BF16
                                     else keys.to(torch.float8_e4m3fn).view(torch.uint8))
            self.q_idx = act(B_, H_I, d_i).to(bf)
            self.w = (torch.randn(B_, H_I, device=device, generator=gen) / math.sqrt(H_I)).float()
            self.sel = torch.empty(B_, k, dtype=torch.int32, device=device)
            self.ws_idx = torch.empty(csa.csa_index_topk_workspace(self.cache, B_, k), dtype=torch.uint8,
                                      device=device)
        self.q = act(B_, H_, D_).to(bf)
        self.win = act(B_ * W, D_).to(bf)
        self.win_start = torch.arange(0, B_ * W, W, dtype=torch.int64, device=device)
        self.win_len = torch.full((B_,), W, dtype=torch.int32, device=device)
        self.q_offsets = torch.arange(B_ + 1, dtype=torch.int32, device=device)
        self.q_pos = torch.full((B_,), T - 1, dtype=torch.int32, device=device)
        self.out = torch.empty(B_, H_, D_, dtype=torch.float32, device=device)
        self.ws_att = torch.empty(csa.csa_attend_workspace(self.cache, B_, H_), dtype=torch.uint8, device=device)

    def stages(self):
        import fp4_kv_cache_csa_b200 as csa

        if not self.d_i:  # HCA layer
            return (lambda: csa.hca_decode_attend(self.cache, self.q, self.q_offsets, self.q_pos, self.win,
                                                  self.win_start, self.win_len, max_win=W,
                                                  softmax_scale=self.D ** -0.5, out=self.out,
                                                  workspace=self.ws_att),)
        return (lambda: csa.csa_index_topk(self.cache, self.q_idx, self.w, self.q_offsets, self.q_pos, self.k,
                                           sel_idx=self.sel, workspace=self.ws_idx),
                lambda: csa.csa_decode_attend(self.cache, self.q, self.q_offsets, self.sel, self.win,
                                              self.win_start, self.win_len, max_win=W,
                                              softmax_scale=self.D ** -0.5, out=self.out, workspace=self.ws_att))

    def bytes_flops(self):
        """Algorithmic HBM bytes and dense-contraction FLOPs of one layer step."""
        entry = self.D // 2 + self.D // scale_group()
        per_req = self.B * (W * self.D * 2 + self.H * self.D * 2 + self.H * self.D * 4)
        if not self.d_i:
            ents = self.n
            b = self.B * ents * entry + per_req
        else:
            ents = min(self.n, self.k)
            kb = 2 if self.cache.idx_dtype == 0 else 1
            b = self.B * (self.n * self.d_i * kb + ents * entry + H_I * self.d_i * 2 + H_I * 4 + self.k * 4) + per_req
        flops = 4.0 * self.B * self.H * (ents + W) * self.D
        return float(b), flops


def measure_configs(device, stream, flush, steps: int = 20):
    """Per-layer decode times of the other workloads (CUDA graphs, cold L2 before each replay)."""
    import torch

    import fp4_kv_cache_csa_b200 as csa

    hbm, hbm_kind = measured_peaks()
    tflops, tf_kind = measured_bf16_tflops()
    runs = (("csa_tiny_4k", dict(B_=1, T=4096, H_=16, D_=128, m=4, d_i=64, idx_dtype=csa.CSA_IDX_BF16, k=64)),
            ("csa_b8_64k", dict(B_=8, T=65536, H_=64, D_=512, m=4, d_i=128, idx_dtype=csa.CSA_IDX_BF16, k=512,
                                lognormal=0.5)),
            ("hca_b64_1m", dict(B_=64, T=1048576, H_=64, D_=512, m=128, d_i=0, idx_dtype=csa.CSA_IDX_BF16, k=0)))
    res = {}
    for name, kw in runs:
        cr = ConfigRun(device, name, **kw)
        torch.cuda.synchronize()  # the caches were written on the default stream
        fns = cr.stages()
        with torch.cuda.stream(stream):
            for fn in fns:
                fn()
            stream.synchronize()
            graphs = []
            for fn in fns:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    fn()
                graphs.append(g)
            for _ in range(3):
                flush.zero_()
                for g in graphs:
                    g.replay()
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(graphs) + 1)] for _ in range(steps)]
            for k in range(steps):
                flush.zero_()
                for s_, g in enumerate(graphs):
                    ev[k][s_].record(stream)
                    g.replay()
                ev[k][len(graphs)].record(stream)
        stream.synchronize()
        st = np.array([[ev[k][j].elapsed_time(ev[k][j + 1]) for j in range(len(graphs))]
                       for k in range(steps)]).mean(axis=0)
        ms = float(st.sum())
        b, fl = cr.bytes_flops()
        t_hbm, t_tc = b / (hbm * 1e9), fl / (tflops * 1e12)
        bound = "hbm" if t_hbm >= t_tc else "tensor"
        res[name] = {"batch": cr.B, "ctx": cr.T, "entries_per_request": cr.n, "ms": ms,
                     "stage_ms": dict(zip(("hca_attend",) if not cr.d_i else ("index_topk", "csa_attend"),
                                          (float(x) for x in st))),
                     "tokens_per_s": cr.B / (ms * 1e-3), "algorithmic_bytes": b, "flops": fl,
                     "achieved_gbs": b / (ms * 1e-3) / 1e9, "achieved_tflops": fl / (ms * 1e-3) / 1e12,
                     "bound": bound, "roofline_frac": max(t_hbm, t_tc) / (ms * 1e-3),
                     "peaks": {"hbm_gbs": hbm, "hbm_kind": hbm_kind, "bf16_tflops": tflops, "bf16_kind": tf_kind},
                     "device_status": int(csa.csa_read_device_status(cr.cache, stream))}
        del graphs, cr
        torch.cuda.empty_cache()
    return res


def measure_index_mxfp4(device, stream, flush, wl, steps: int = 20):
    """The step's indexer call (same requests, queries and k) over a cache whose indexer keys are
    MXFP4 (E2M1 codes + one E8M0 scale per 32 channels: 68 bytes per key instead of 128)."""
    import torch

    import fp4_kv_cache_csa_b200 as csa

    gen = torch.Generator(device=device)
    gen.manual_seed(SEED + 11)
    cache = csa.Cache(fp4=wl.csa.fp4, scale=wl.csa.scale, n_blocks=wl.csa.n_blocks.clone(), block=M_CSA,
                      idx_key=torch.empty(B, CAP_CSA, D_I // 2, dtype=torch.uint8, device=device),
                      idx_dtype=csa.CSA_IDX_MXFP4, status=torch.zeros(1, dtype=torch.int32, device=device),
                      scale_fmt=SCALE_FMT,
                      idx_key_scale=torch.empty(B, CAP_CSA, D_I // 32, dtype=torch.uint8, device=device))
    cache.idx_key.random_(0, 256, generator=gen)
    cache.idx_key_scale.random_(122, 128, generator=gen)  # pooled N(0, 0.5^2) keys land in 2^-5 .. 2^0
    cache.n_blocks.copy_(torch.tensor(wl.n_csa, dtype=torch.int32, device=device))
    sel = torch.empty(B, TOPK, dtype=torch.int32, device=device)
    ws = torch.empty(csa.csa_index_topk_workspace(cache, B, TOPK), dtype=torch.uint8, device=device)
    fn = lambda: csa.csa_index_topk(cache, wl.q_idx, wl.w, wl.q_offsets, wl.q_pos, TOPK, sel_idx=sel, workspace=ws)
    torch.cuda.synchronize()  # the cache was written on the default stream
    with torch.cuda.stream(stream):
        fn()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        for _ in range(3):
            flush.zero_()
            g.replay()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for k in range(steps):
            flush.zero_()
            ev[k][0].record(stream)
            g.replay()
            ev[k][1].record(stream)
    stream.synchronize()
    ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    key_bytes = float(np.sum(wl.n_csa)) * (D_I // 2 + D_I // 32)
    b = key_bytes + B * (H_I * D_I * 2 + H_I * 4 + TOPK * 4)
    hbm, kind = measured_peaks()
    res = {"ms": ms, "tokens_per_s": B / (ms * 1e-3), "key_bytes_per_block": D_I // 2 + D_I // 32,
           "algorithmic_bytes": b, "achieved_gbs": b / (ms * 1e-3) / 1e9, "frac_of_hbm_peak": b / (ms * 1e-3) / 1e9 / hbm,
           "peak_kind": kind, "device_status": int(csa.csa_read_device_status(cache, stream))}
    del g
    return res


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", 6650.0)), "measured"
    return 6650.0, "fallback"


def measured_bf16_tflops():
    """Dense bf16 tensor peak: the burst figure of MEASURED_PEAKS.json, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# DRAM traffic of one indexer call (scan with its own schedule, then the merge): the
# read + write bytes that one ncu capture of the call at 8 requests of the same workload
# counted, and the key bytes of that call; scaled to this run by key bytes. Valid only
# for the indexer source it was taken on (hash below); otherwise reported as null.
INDEX_TRAFFIC_CAPTURE = {"bytes": 210.507e6 + 0.442e6 + 1.329e6, "key_bytes": 210.427904e6, "source_hash": "b4b338c7134dd890"}


def index_traffic(key_bytes: float):
    import hashlib

    h = hashlib.sha256()
    for f in ("indexer.cu", "common.cuh"):
        with open(os.path.join(ROOT, "fp4_kv_cache_csa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != INDEX_TRAFFIC_CAPTURE["source_hash"]:
        return None
    return INDEX_TRAFFIC_CAPTURE["bytes"] * key_bytes / INDEX_TRAFFIC_CAPTURE["key_bytes"] / 1e9  # GB per call


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(values, world: int, device):
    """Each timing as the maximum over the ranks (the slowest replica sets the pace)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(ms_per_step: float, world: int):
    """Replicas: every rank decodes its own B requests per step (weak scaling), so the job's
    tokens per step are B * world and its rate is set by the slowest rank's step time."""
    tokens = B * world
    return tokens, tokens / (ms_per_step * 1e-3)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    n_req = 2
    # one "step" of the oracle = the step's work for n_req requests
    times = []
    for _ in range(args.warmup + args.steps):
        v, cores, sample = cpu_baseline(n_req)
        times.append(n_req / v)
    t = statistics.mean(times[args.warmup:])
    value = n_req / t
    line = {"impl": "reference", "metric": "CSA decode tokens/s and achieved HBM TB/s at 1M ctx (MXFP4 KV), vs roofline",
            "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": "csa_hca_decode_b32_ctx512k-1m", "global_batch": B, "seq_len": CTX_MAX,
                       "parallelism": "replicas", "scale_fmt": scale_fmt_name(),
                       "l2": "inputs larger than L2 (full key cache streamed)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill_b4_8k measurement")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the csa_tiny_4k / csa_b8_64k / hca_b64_1m measurements")
    ap.add_argument("--batch", type=int, default=B, help="requests per GPU (default 32; smaller only for profiling)")
    ap.add_argument("--prefill-requests", type=int, default=Prefill.B,
                    help="requests of the prefill workload (default 4; fewer only for profiling)")
    ap.add_argument("--scale-fmt", default="e8m0x32", choices=sorted(SCALE_FMT_NAMES),
                    help="FP4 scale format of both caches (default: E8M0 per 32 elements, MXFP4)")
    args = ap.parse_args()
    set_batch(args.batch)
    set_prefill_requests(args.prefill_requests)
    set_scale_fmt(args.scale_fmt)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import fp4_kv_cache_csa_b200 as csa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    csa.load_library()

    wl = Workload(rank, device)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device)
    graphs = []
    with torch.cuda.stream(stream):
        for fn in wl.stages():  # eager pass before capture
            fn()
        stream.synchronize()
        for fn in wl.stages():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            graphs.append(g)
    torch.cuda.synchronize()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)  # > 126 MB L2

    def replay_step(evs=None):
        for s, g in enumerate(graphs):
            if evs is not None:
                evs[s].record(stream)
            g.replay()
        if evs is not None:
            evs[len(graphs)].record(stream)

    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            replay_step()
    stream.synchronize()
    status = csa.csa_read_device_status(wl.csa, stream) | csa.csa_read_device_status(wl.hca, stream)

    # ---- device-resident timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark_start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(graphs) + 1)] for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for k in range(args.steps):
            flush.zero_()  # outside the events: every step starts with a cold L2
            replay_step(ev[k])
    stream.synchronize()
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        dist.barrier()
    clocks.stop()
    st_ms = np.array([[ev[k][s].elapsed_time(ev[k][s + 1]) for s in range(len(graphs))] for k in range(args.steps)])
    step_ms = st_ms.sum(axis=1)
    ms = float(step_ms.mean())

    # ---- CSA2 (not part of the step): a Full layer that also keeps the pool, and
    # a Reindex layer over that pool, each timed alone with a cold L2
    csa2_graphs = []
    csa2_fns = (wl.stage_index_pool, wl.stage_index_reindex, wl.stage_index_reindex_layers)
    with torch.cuda.stream(stream):
        for fn in csa2_fns:
            fn()
        stream.synchronize()
        for fn in csa2_fns:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            csa2_graphs.append(g)
    n2 = max(4, min(args.steps, 50))
    nf = len(csa2_fns)
    ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(nf * n2)]
    with torch.cuda.stream(stream):
        for k in range(nf * n2):
            flush.zero_()
            ev2[k][0].record(stream)
            csa2_graphs[k % nf].replay()
            ev2[k][1].record(stream)
    stream.synchronize()
    csa2_ms = [float(np.mean([ev2[k][0].elapsed_time(ev2[k][1]) for k in range(j, nf * n2, nf)]))
               for j in range(nf)]
    status |= csa.csa_read_device_status(wl.csa, stream)
    del csa2_graphs
    prefill = measure_prefill(device, stream, flush) if not args.no_prefill else None
    prefill_mx = measure_prefill_index_mxfp4(device, stream, flush) if not args.no_prefill else None
    configs = measure_configs(device, stream, flush) if not args.no_configs else None
    index_mxfp4 = measure_index_mxfp4(device, stream, flush, wl) if not args.no_configs else None

    # ---- end-to-end: pinned host inputs in, results out, every step. Two buffer
    # sets (each with its own graphs): step k+1's inputs are copied in and step
    # k-1's results copied out (own streams) while step k computes.
    import copy

    ins, outs = wl.step_inputs()
    wl2 = copy.copy(wl)
    for name in ("kv4", "idx4", "kv128", "q_csa", "q_hca", "q_idx", "w", "out_csa", "out_hca"):
        setattr(wl2, name, getattr(wl, name).clone())
    ins2, outs2 = wl2.step_inputs()
    graphs2 = []
    with torch.cuda.stream(stream):
        for fn in wl2.stages():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            graphs2.append(g)
        for g in graphs2:  # first replay outside the timed loop
            g.replay()
    torch.cuda.synchronize()
    sets = [(ins, outs, graphs), (ins2, outs2, graphs2)]
    h_ins = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t.cpu()) for t in ins] for _ in range(2)]
    h_outs = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in h_ins[0])
    d2h = sum(t.numel() * t.element_size() for t in h_outs[0])
    e2e_n = max(4, min(args.steps, 50))
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    # the host link alone: one step's input copies, then one step's output copies (best of 5)
    link_ms = []
    for src, dst, st_ in ((h_ins[0], ins, up), (outs, h_outs[0], down)):
        best = float("inf")
        for _ in range(5):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(st_)
            with torch.cuda.stream(st_):
                for s_, d_ in zip(src, dst):
                    d_.copy_(s_, non_blocking=True)
            b_.record(st_)
            b_.synchronize()
            best = min(best, a_.elapsed_time(b_))
        link_ms.append(best)
    ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    drained = [torch.cuda.Event() for _ in range(2)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream.synchronize()
    t_start.record(stream)
    up.wait_event(t_start)
    down.wait_event(t_start)
    for k in range(e2e_n):
        b = k % 2
        d_ins, d_outs, gs = sets[b]
        if k >= 2:
            up.wait_event(computed[b])  # step k-2 has finished reading this set's inputs
        with torch.cuda.stream(up):
            for d_, h_ in zip(d_ins, h_ins[b]):
                d_.copy_(h_, non_blocking=True)
        ready[b].record(up)
        stream.wait_event(ready[b])
        if k >= 2:
            stream.wait_event(drained[b])  # step k-2's results are out of this set's outputs
        with torch.cuda.stream(stream):
            for g in gs:
                g.replay()
        computed[b].record(stream)
        down.wait_event(computed[b])
        with torch.cuda.stream(down):
            for h_, d_ in zip(h_outs[b], d_outs):
                h_.copy_(d_, non_blocking=True)
        drained[b].record(down)
    stream.wait_stream(down)
    t_end.record(stream)
    stream.synchronize()
    e2e_ms = t_start.elapsed_time(t_end) / e2e_n
    del graphs2

    ms, e2e_ms, idx_ms, csa_ms = max_over_ranks(
        [ms, e2e_ms, float(st_ms[:, 1].mean()), float((st_ms[:, 1] + st_ms[:, 2]).mean())], world, device)
    tokens, value = job_throughput(ms, world)
    peak, peak_kind = measured_peaks()
    achieved = wl.bytes_index() / (idx_ms * 1e-3) / 1e9  # GB/s of the indexer stage
    hbm_tbs = wl.bytes_step() / (ms * 1e-3) / 1e12

    line = {
        "metric": "CSA decode tokens/s and achieved HBM TB/s at 1M ctx (MXFP4 KV), vs roofline",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32-acc/fp16-mma",
        "data": "synthetic (seeded torch RNG on device)",
        "config": {"workload": "csa_hca_decode_b32_ctx512k-1m", "global_batch": tokens, "seq_len": CTX_MAX,
                   "parallelism": f"replicas x{world}", "per_gpu_batch": B, "topk": TOPK, "heads": H, "dim": D,
                   "scale_fmt": scale_fmt_name(),
                   "l2": "flushed between steps (512 MB write) and inputs larger than L2"},
        "hbm_tbs": hbm_tbs,
        "stage_ms": {"compress": float(st_ms[:, 0].mean()), "index_topk": float(st_ms[:, 1].mean()),
                     "attend_csa": float(st_ms[:, 2].mean()), "attend_hca": float(st_ms[:, 3].mean())},
        # one CSA layer at decode (indexer + top-k + CSA attention) against its own HBM roofline
        "csa_layer": {"ms": csa_ms, "tokens_per_s": tokens / (csa_ms * 1e-3),
                      "algorithmic_bytes": wl.bytes_csa_layer(),
                      "achieved_gbs": wl.bytes_csa_layer() / (csa_ms * 1e-3) / 1e9,
                      "frac_of_hbm_peak": wl.bytes_csa_layer() / (csa_ms * 1e-3) / 1e9 / peak},
        "roofline": {"bound": "hbm", "kernel": "csa_index_topk (scan + merge)", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": index_traffic(wl.key_bytes()), "traffic_unit": "GB per call (ncu, scaled by keys)",
                     "traffic_note": None if index_traffic(wl.key_bytes()) is not None else
                     "null: the indexer source changed after its last ncu capture; no capture of this source"},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_n,
                "overlap": "step k+1 inputs in and step k-1 results out while step k computes",
                "link_h2d_gbs": h2d / (link_ms[0] * 1e-3) / 1e9, "link_d2h_gbs": d2h / (link_ms[1] * 1e-3) / 1e9},
        # CSA2 cross-layer modes (not in the step): Full layer + pool, then a Reindex layer over the pool
        "csa2": {"pool_group": POOL_GROUP, "pool_blocks": POOL_BLOCKS, "full_with_pool_ms": csa2_ms[0],
                 "reindex_ms": csa2_ms[1], "full_ms": idx_ms,
                 "reindex_layers": REINDEX_LAYERS, "reindex_layers_one_call_ms": csa2_ms[2],
                 "reindex_algorithmic_bytes": wl.bytes_reindex(),
                 "reindex_achieved_gbs": wl.bytes_reindex() / (csa2_ms[1] * 1e-3) / 1e9},
        "prefill": None if prefill is None else dict(
            prefill, index_tensor_frac=prefill["index_tflops"] / measured_bf16_tflops()[0],
            index_tensor_peak={"tflops": measured_bf16_tflops()[0], "kind": measured_bf16_tflops()[1] + " bf16 dense"}),
        # the prefill indexer stage with MXFP4 indexer keys (block-scaled tensor-core GEMM)
        "prefill_index_mxfp4": prefill_mx,
        "configs": configs,
        # the same indexer call with MXFP4 indexer keys (not the headline config's e4m3 keys)
        "index_mxfp4_keys": index_mxfp4,
        "gpu_launches": OUR_KERNELS_PER_STEP * args.steps,
        "clocks": clocks.summary(),
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = cpu_baseline()
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
    if world > 1:
        dist.barrier()
    del graphs
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
