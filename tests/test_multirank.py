"""The N>1 path of bench.py on CPU: two gloo ranks (replicas, no data-path collective).

Covers the cross-rank timing reduction (max over ranks), the whole-job
throughput aggregation and the reference arm's rank-0-only behaviour.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    bench.dist_init(world, backend="gloo")
    try:
        my_ms = 100.0 + 25.0 * rank                  # rank 1 is the slow one
        mx = bench.max_over_ranks(my_ms, world)
        rate = bench.whole_job_rate(world, 16384, 10, mx)
        bench.barrier(world)
        out[rank] = (mx, rate)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_whole_job_rate():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert set(out.keys()) == {0, 1}
    for r in range(world):
        mx, rate = out[r]
        assert mx == 125.0                          # slowest rank's time on every rank
        assert rate == pytest.approx(2 * 16384 * 10 / 0.125)


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1", MASTER_PORT="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_single_rank_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(1, 100, 4, 2000.0) == pytest.approx(200.0)
