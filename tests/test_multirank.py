"""The multi-rank (replicas) host logic of bench.py on CPU: two gloo ranks.

Each rank of `bench.py --gpus N` runs its own replica of the decode step; the job's time
is the slowest rank's, taken with an all-reduce, and rank 0 alone prints the JSON line.
"""
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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # ranks see different local step times; every rank must get the largest
        local_ms = [12.5, 20.0][rank]
        ms = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        e2e = bench.max_over_ranks([30.0, 25.0][rank], world, torch.device("cpu"))
        out[rank] = (ms, e2e, bench.whole_job_gbs(world, 1e9, 10, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        ms, e2e, gbs = out[r]
        assert ms == 20.0 and e2e == 30.0
        # 2 ranks x 1 GB x 10 steps in the slowest rank's 20 ms
        assert gbs == pytest.approx(2 * 1e9 * 10 / 0.020 / 1e9)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.whole_job_gbs(1, 4e9, 2, 1000.0) == pytest.approx(8.0)


def test_reference_arm_under_torchrun_prints_once():
    """--impl reference under torchrun: rank 0 times the oracle and prints one line, the
    other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "single_768"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
