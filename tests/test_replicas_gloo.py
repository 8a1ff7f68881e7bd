"""The multi-GPU form of the benchmark runs independent replicas (the layer
has no cross-GPU exchange): each rank times its own steps, the job takes the
slowest rank's time, and the whole-job rate counts every rank's tokens.
This checks that host-side logic with two gloo ranks on the CPU."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, times, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        f = bench.max_over_ranks_fn(world, torch.device("cpu"))
        ms = f(times[rank])
        dist.barrier()
        out[rank] = (ms, bench.whole_job_rate(4096, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    port = 29500 + os.getpid() % 2000
    times = [2.5, 3.25]
    with mp.get_context("spawn").Manager() as m:  # no fork of a threaded process
        out = m.dict()
        mp.spawn(_worker, args=(2, port, times, out), nprocs=2, join=True)
        got = dict(out)
    for rank in (0, 1):
        ms, rate = got[rank]
        assert ms == 3.25  # both ranks see the slowest time
        assert rate == pytest.approx(2 * 4096 / 3.25e-3)


def test_one_replica_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    f = bench.max_over_ranks_fn(1, torch.device("cpu"))
    assert f(1.5) == 1.5
    assert bench.whole_job_rate(8, 1, 2.0) == pytest.approx(4000.0)
