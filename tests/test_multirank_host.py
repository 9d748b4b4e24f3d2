"""Host logic of the multi-rank bench path, on CPU: two ranks over gloo.

Each rank owns one layer set (distinct seeds, no data-path collective); the job's
time is the maximum over ranks; the reference arm runs on rank 0 alone."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports durations that make each rank the slowest on one entry
        mine = [10.0 + rank, 20.0 - rank, 5.0 * (rank + 1)]
        got = bench.reduce_times(mine, dist, "cpu")

        class A:
            workload, optimizers, steps, warmup, seed, cpu_budget_s = "muon_single", "muon", 1, 0, 0, 0.2
        ref = bench.run_reference(A, rank, world) if rank != 0 else "skipped"
        q.put((rank, got, bench.rank_seed(0, rank), ref))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_seeds_and_rank0_reference():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, got, seed, ref in out:
        assert got == [11.0, 20.0, 10.0], (rank, got)
        if rank != 0:
            assert ref is None  # the oracle arm prints on rank 0 only
    assert out[0][2] != out[1][2]
    assert bench.per_layer_set(30.0, world) == 15.0


def test_single_process_reduce_is_identity():
    assert bench.reduce_times([3.5, 7.25], None, "cpu") == [3.5, 7.25]
    assert bench.rank_seed(5, 0) == 5
