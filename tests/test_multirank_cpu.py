"""The multi-process plumbing of bench.py, on CPU with the gloo backend (world size 2).

bench.py runs one replica of the workload per rank (the path has no exchange step), times
each rank on its device and reports the whole job from the slowest rank.  These tests run
that reduction across two gloo ranks, and the reference arm as torchrun launches it with
two processes (rank 0 alone measures and prints).
"""
import json
import os
import socket
import subprocess
import sys
import tempfile

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as td
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    td.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        ms = bench.max_over_ranks(torch.tensor([local_ms], dtype=torch.float64), True)
        rate = bench.whole_job_rate(1000, world, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "rate": rate}, f)
    finally:
        td.barrier()
        td.destroy_process_group()


def test_max_over_two_gloo_ranks():
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(2, _free_port(), d), nprocs=2, join=True, start_method="spawn")
        res = [json.load(open(os.path.join(d, f"rank{r}.json"))) for r in range(2)]
    # both ranks see the slowest rank's time; the job rate counts both replicas' units
    assert res[0]["ms"] == res[1]["ms"] == 15.0
    assert res[0]["rate"] == pytest.approx(1000 * 2 / 15e-3 / 1e6)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(torch.tensor([3.5], dtype=torch.float64), False) == 3.5
    assert bench.whole_job_rate(786432, 1, 0.25) == pytest.approx(786432 / 0.25e-3 / 1e6)


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "fp32_L256"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
