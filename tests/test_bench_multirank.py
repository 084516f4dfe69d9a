"""bench.py's multi-rank bookkeeping on CPU: two gloo ranks, max over ranks of
the timings and the whole-job throughput they give (replicas: per-GPU work is
fixed, the job's units add up)."""
import os
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = 100.0 + 50.0 * rank  # rank 1 is the slower one
    got = bench.max_over_ranks(world, ms)
    out[rank] = (got, bench.job_throughput(12100, world, 10, got))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    manager = mp.get_context("spawn").Manager()  # no fork of this (threaded) process
    out = manager.dict()
    port = 29500 + (os.getpid() % 1000)
    mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
    assert out[0][0] == out[1][0] == 150.0
    assert out[0][1] == pytest.approx(12100 * 2 * 10 / 0.150)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1, 42.0) == 42.0
    assert bench.job_throughput(12100, 1, 20, 1000.0) == pytest.approx(12100 * 20)
