"""Host-side logic of the multi-rank bench (replicas only), on CPU with gloo.

The bench runs one independent replica per GPU; the only cross-rank steps
are the max of the step times and the whole-job rate.  These run here as
two gloo ranks, and the reference arm is launched under torch.distributed.run
with two ranks to check that rank 0 alone prints its line.
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.5 + rank, 10.0 - rank, 7.0])
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out),
                           nprocs=world, join=True, start_method="spawn")
        for r in range(world):
            assert out[r] == [2.5, 10.0, 7.0]


def test_job_rate_counts_all_ranks_over_slowest_time():
    # 4 replicas of 32768 tokens in 2 ms -> 65.536 M tokens/s
    assert bench.job_rate(32768, 4, 2.0) == pytest.approx(65.536e6)
    assert bench.job_rate(1, 1, 1.0) == pytest.approx(1000.0)


def test_reference_arm_prints_once_under_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
           "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload",
           "tiny_prefill_f32", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["value"] > 0
