"""The multi-process path of bench.py on CPU: two gloo ranks reduce their
step times to the slowest one and count both ranks' tokens, and under a
launcher only rank 0 runs the reference arm (the others exit without work)."""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        def reduce_max(x):
            t = torch.tensor([x], dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())
        local_ms = [2.0, 5.0][rank]
        ms, tps = bench.job_throughput(local_ms, 1000, world, reduce_max)
        out[rank] = (ms, tps)
    finally:
        dist.destroy_process_group()


def test_job_throughput_two_gloo_ranks():
    world, port = 2, _free_port()
    out = tmp.get_context("spawn").Manager().dict()  # no fork of this (threaded) process
    tmp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        ms, tps = out[r]
        assert ms == 5.0                              # the slowest rank's time, on every rank
        assert abs(tps - 2 * 1000 / 5e-3) < 1e-6      # both ranks' tokens


def test_job_throughput_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    ms, tps = bench.job_throughput(4.0, 100, 1, lambda x: (_ for _ in ()).throw(AssertionError("no collective")))
    assert ms == 4.0 and abs(tps - 100 / 4e-3) < 1e-9


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
