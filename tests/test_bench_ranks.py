"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (one process per rank, as
torchrun starts them on a node) take the maximum of their times and report the whole-job
throughput from it.  The hot path runs one replica per rank with no exchange step, so this
barrier-and-maximum logic is all the multi-GPU path adds."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        barrier, max_over_ranks = bench.rank_tools(torch, dist, torch.device("cpu"))
        barrier()
        t = max_over_ranks(times[rank])
        out[rank] = (t, bench.whole_job(1000.0, world, t))
        barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_time():
    world, port = 2, _free_port()
    times = [1.5, 2.5]  # ms per step of each rank
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, times, out), nprocs=world, join=True)
        got = dict(out)
    for r in range(world):
        t, v = got[r]
        assert t == 2.5
        assert v == pytest.approx(2 * 1000.0 / 2.5e-3)


def test_one_rank_needs_no_process_group():
    barrier, max_over_ranks = bench.rank_tools(torch, None, torch.device("cpu"))
    barrier()
    assert max_over_ranks(3.25) == 3.25
    assert bench.whole_job(10.0, 1, 2.0) == pytest.approx(5000.0)
