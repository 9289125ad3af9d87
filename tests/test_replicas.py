"""Multi-process (replicas-only) host logic of bench.py on CPU with gloo.

The path shards into independent units and has no exchange step, so N GPUs run
N replicas; what needs checking is the host side: the max-over-ranks timing,
the whole-job aggregate, and that under torchrun only rank 0 prints.
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
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [3.0, 7.5][rank]
    m = bench.max_over_ranks(local_ms, dist)
    q.put((rank, m, bench.whole_job_tflops(1e12, world, 10, m)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    mp.spawn(_worker, args=(2, port, q), nprocs=2, join=True)
    got = sorted(q.get(timeout=30) for _ in range(2))
    for rank, m, v in got:
        assert m == 7.5                      # every rank sees the slowest rank's time
        assert abs(v - 1e12 * 2 * 10 / 7.5e-3 / 1e12) < 1e-9


def test_single_process_is_identity():
    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.whole_job_tflops(2e12, 1, 4, 8.0) == pytest.approx(1000.0)


def test_reference_arm_under_torchrun_prints_once():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
