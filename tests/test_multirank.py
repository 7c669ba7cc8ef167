"""The N > 1 launch path on CPU: world-size-2 `gloo` process groups.

The hot path has no exchange step (every (batch, kv head) group is
independent), so several GPUs run replicas; what the ranks share is the
timing contract of bench.py: every rank reduces its timings and its error
status with a max over ranks at the same points, and under torchrun the
reference arm runs on rank 0 alone while the other ranks exit cleanly.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _reduce_worker(rank: int, world: int, port: int, values, out_dir: str) -> None:
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method="env://")
    try:
        got = bench.max_over_ranks(values[rank], torch.device("cpu"))
        status = bench.max_over_ranks(4 if rank == 1 else 0, torch.device("cpu"))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "status": status}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    import torch.multiprocessing as mp

    values = [1.25, 3.5]
    mp.start_processes(_reduce_worker, args=(2, _free_port(), values, str(tmp_path)), nprocs=2,
                       start_method="spawn", join=True)
    for r in range(2):
        with open(tmp_path / f"rank{r}.json") as f:
            d = json.load(f)
        assert d["max"] == 3.5          # every rank sees the slowest rank's time
        assert d["status"] == 4         # and any rank's error status


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import torch

    import bench

    assert bench.max_over_ranks(2.5, torch.device("cpu")) == 2.5


def test_reference_arm_under_torchrun():
    """Two ranks: rank 0 times the oracle and prints one JSON line, rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "1",
           "--impl", "reference"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
