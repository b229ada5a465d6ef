"""The bench's algorithmic byte and FLOP counts against closed forms (no GPU).

Every roofline fraction the bench prints divides one of these counts by a
measured time, so each is pinned here to an independent count of what the
workload must move or compute: the visible (query, block) pairs of the
causal prefill summed token by token, the indexer key stream of the drawn 1M
contexts, and the per-request byte lists of the HCA and 64K workloads
(entry = 256 code bytes + 16 E8M0 scale bytes at D = 512)."""
import types

import numpy as np

import bench


def test_prefill_indexer_flops_count_every_visible_pair():
    # 4 requests of 65536 cached + 8192 new tokens, one query per new token, causal at
    # 4-token blocks: the query at new token t sees floor((65536 + t + 1) / 4) blocks
    pairs = sum((65536 + t + 1) // 4 for t in range(8192))
    assert pairs == 142_604_288
    pf = types.SimpleNamespace(B=4, NEW=8192, T0=65536)
    assert bench.Prefill.index_flops(pf) == 4 * pairs * 4 * 128 * 2 == 584_107_163_648


def test_decode_indexer_and_csa_layer_bytes():
    lengths = bench.context_lengths(0)
    assert len(lengths) == 32 and lengths.min() >= 512 * 1024 and lengths.max() <= 1024 * 1024
    assert np.all(lengths % 128 == 0)
    n = lengths // 4
    wl = types.SimpleNamespace(n_csa=n)
    wl.bytes_index = lambda: bench.Workload.bytes_index(wl)
    keys = int(n.sum()) * 128                      # e4m3 keys, 128 bytes each
    per_query = 4 * 128 * 2 + 4 * 4 + 1024 * 4     # bf16 indexer query, head weights, selected indices
    assert bench.Workload.bytes_index(wl) == keys + 32 * per_query
    assert abs(bench.Workload.bytes_index(wl) - 829.067776e6) < 1.0
    # the CSA layer adds the selected entries (every context has more than 1024 blocks),
    # the 128-token bf16 window, the bf16 query and the fp32 output of 64 heads x 512
    layer = keys + 32 * per_query + 32 * (1024 * 272 + 128 * 512 * 2 + 64 * 512 * 2 + 64 * 512 * 4)
    assert bench.Workload.bytes_csa_layer(wl) == layer


def test_hca_and_64k_workload_counts():
    hca = types.SimpleNamespace(D=512, B=64, H=64, n=8192, d_i=0, k=0, cache=None)
    b, f = bench.ConfigRun.bytes_flops(hca)
    per_req = 8192 * 272 + 128 * 512 * 2 + 64 * 512 * 2 + 64 * 512 * 4
    assert b == 64 * per_req == 163_577_856
    assert f == 64 * 64 * (8192 + 128) * 512 * 4     # QK and PV, 2 FLOP per MAC each
    assert abs(f - 69.8e9) < 0.1e9
    c2 = types.SimpleNamespace(D=512, B=8, H=64, n=16384, d_i=128, k=512,
                               cache=types.SimpleNamespace(idx_dtype=0))
    b, f = bench.ConfigRun.bytes_flops(c2)
    per_req = (16384 * 128 * 2 + 512 * 272 + 4 * 128 * 2 + 4 * 4 + 512 * 4
               + 128 * 512 * 2 + 64 * 512 * 2 + 64 * 512 * 4)
    assert b == 8 * per_req
    assert abs(b - 37.3e6) < 0.05e6
    assert f == 8 * 64 * (512 + 128) * 512 * 4
