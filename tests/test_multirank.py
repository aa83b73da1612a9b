"""The N > 1 host path of bench.py on the CPU: two ranks over gloo.

The decode has no exchange between batch rows, so several GPUs run replicas
(one batch per rank, weak scaling) and meet only to take the slowest rank's
time.  These tests run that reduction and the whole-job rate with two real
processes, and the reference arm as the driver launches it (torchrun, two
ranks: rank 0 alone works and prints, the other exits 0).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        rate = bench.whole_job_rate(64, world, 100, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "rate": rate}, f)
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_slowest_rank_time_and_whole_job_rate_over_two_gloo_ranks(tmp_path):
    times = [7.25, 9.5]  # rank 1 is the slow one
    mp.start_processes(_rank_main, args=(2, _free_port(), times, str(tmp_path)), nprocs=2, start_method="spawn",
                       join=True)
    for r in range(2):
        with open(tmp_path / f"rank{r}.json") as f:
            got = json.load(f)
        assert got["ms"] == 9.5  # every rank sees the maximum
        assert got["rate"] == pytest.approx(64 * 2 * 100 / 9.5e-3)  # rows of all ranks over the slowest time


def test_one_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.whole_job_rate(64, 1, 10, 2.0) == pytest.approx(64 * 10 / 2e-3)


def test_reference_arm_under_torchrun_two_ranks():
    """As the driver launches it for N = 2: only rank 0 runs the oracle and
    prints one JSON line; the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "small_b3_ctx1001_top256"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2 and res["value"] > 0
    assert res["cpu_baseline"]["kind"] == "oracle"
