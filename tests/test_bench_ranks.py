"""The benchmark's multi-rank host logic on CPU: two gloo ranks agree on the maximum of their
timings, the job throughput counts every replica, and only rank 0 runs the reference arm."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(dist, [1.0 + rank, 10.0 - rank, 3.5], device="cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == [2.0, 10.0, 3.5]


def test_single_process_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, [4, 5.5]) == [4.0, 5.5]


def test_job_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_throughput(1, 1e9, 10, 100.0)
    assert one == pytest.approx(1e11)
    assert bench.job_throughput(4, 1e9, 10, 100.0) == pytest.approx(4 * one)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    import pba_inputs as pi
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(warmup=3, steps=2, seed=0, cpu_seconds=1.0)
    assert bench.run_reference(args, pi.CONFIGS["C1"]) is None
