"""The bench's multi-GPU host logic on CPU: two gloo ranks.

The hot path has no cross-GPU exchange, so `bench.py --gpus N` runs N
independent replicas; what has to be right is the host side: every rank sees
the slowest rank's timings, the job's throughput counts the work of all ranks,
and the reference arm runs on rank 0 alone while the other ranks exit cleanly.
"""

import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r's timings: total grows with r, e2e shrinks with r
        out[rank] = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 2.5], world, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    # the manager's server process is spawned too: forking a process that
    # already runs threads can deadlock the child
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_max_worker, args=(world, free_port(), out), nprocs=world, join=True)
        got = dict(out)
    assert got == {0: [11.0, 5.0, 2.5], 1: [11.0, 5.0, 2.5]}


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([3.0, 1.0], 1, "cpu") == [3.0, 1.0]


def test_job_throughput_counts_every_rank():
    # 1e12 FLOP per step, 10 steps on each of 2 ranks, slowest rank 1000 ms
    assert bench.job_throughput(1e12, 10, 2, 1000.0) == pytest.approx(2e13)
    assert bench.job_throughput(1e12, 10, 1, 1000.0) == pytest.approx(1e13)


def test_reference_arm_under_torchrun_two_ranks():
    # rank 0 prints one JSON line; rank 1 exits 0 without work
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--workload", "decode64", "--steps", "1", "--warmup", "3",
           "--ref-rows", "1", "--ref-cols", "64"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
