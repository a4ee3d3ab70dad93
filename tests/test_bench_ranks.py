"""The benchmark's multi-process plumbing on CPU: two gloo ranks, each with its own
device time, agree on the slowest one and on the whole-job throughput (weak scaling:
every rank runs the same steps of its own replica)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(world, times[rank])
        out[rank] = (ms, bench.job_tokens_per_s(world, 100, 8, ms))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_ranks():
    world, port = 2, _free_port()
    times = [3.0, 5.0]                     # ms for 100 steps, per rank
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, port, times, out), nprocs=world, join=True)
    for r in range(world):
        ms, tps = out[r]
        assert ms == 5.0                   # the slowest rank
        assert tps == pytest.approx(2 * 100 * 8 / 0.005)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(1, 1.25) == 1.25
    assert bench.job_tokens_per_s(1, 10, 1, 2.0) == pytest.approx(5000.0)
