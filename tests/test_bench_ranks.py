"""The multi-rank plumbing of bench.py on CPU: world size 2 over gloo.

Each rank of a replicas-only run times its own steps; the job's time is the slowest
rank's, and the whole-job rate counts every rank's steps.  No GPU is involved."""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 100.0 + 50.0 * rank            # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms, torch.device("cpu"))
        rate = bench.whole_job_rate(world, 20, total)
        env = bench.dist_env()
        out[rank] = (total, rate, env)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    for r in range(world):
        total, rate, env = out[r]
        assert total == pytest.approx(150.0)          # the slowest rank's time on every rank
        assert rate == pytest.approx(2 * 20 / 0.150)  # all ranks' steps over that time
        assert env == (world, r, r)


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(12.5, torch.device("cpu")) == 12.5
    assert bench.whole_job_rate(1, 10, 1000.0) == pytest.approx(10.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup, gpus = 1, 3, 2

    assert bench.run_reference(Args(), None) is None   # returns before touching the workload
    assert capsys.readouterr().out == ""
