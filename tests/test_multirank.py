"""The benchmark's multi-rank host logic on CPU: two gloo ranks (no GPU).

Replicas: each rank owns a different seeded batch of requests, the step time is the
maximum over ranks, and the job's throughput counts every rank's requests."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports times r+1, 10*(r+1), ...; every rank must see the maxima
        got = bench.max_over_ranks([rank + 1.0, 10.0 * (rank + 1), 0.5], world, "cpu")
        tokens, value = bench.job_throughput(got[0], world)
        out[rank] = (got, tokens, value, bench.context_lengths(rank).tolist())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest_and_count_every_replica():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    import bench

    for r in range(world):
        got, tokens, value, lengths = res[r]
        assert got == [2.0, 20.0, 0.5]
        assert tokens == bench.B * world
        assert np.isclose(value, bench.B * world / 2.0e-3)
    # each replica decodes its own seeded batch
    assert res[0][3] != res[1][3]
    assert res[0][3] == bench.context_lengths(0).tolist()


def test_one_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
    tokens, value = bench.job_throughput(0.5, 1)
    assert tokens == bench.B and np.isclose(value, bench.B / 0.5e-3)
