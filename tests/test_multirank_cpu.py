"""The multi-process path of bench.py on the CPU (gloo, world size 2): every rank runs the
same workload (weak scaling), the timed region is the max over ranks, rank 0 alone prints
the JSON line. No GPU is used."""
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


def _ranks_max(rank, world, port, values, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(values[rank], dist, "cpu")
        # a second call in the same order on every rank
        got2 = bench.max_over_ranks(-values[rank], dist, "cpu")
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump([got, got2], f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    values = [3.25, 7.5]
    mp.spawn(_ranks_max, args=(2, free_port(), values, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        got, got2 = json.load(open(tmp_path / f"r{r}.json"))
        assert got == max(values)
        assert got2 == max(-v for v in values)


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(4.0, None, "cpu") == 4.0


def test_whole_job_is_weak_scaling():
    # 2 ranks, each 1e12 units per step, 2 ms per step (the slowest rank)
    assert bench.whole_job(1e12, 2.0, 2) == pytest.approx(1e15)
    assert bench.whole_job(5.0, 1000.0, 1) == pytest.approx(5.0)


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    """bench.py --impl reference under torchrun with 2 ranks: rank 0 alone prints one JSON
    line for the whole job; the other rank exits 0 without work."""
    env = dict(os.environ, SWA_REF_STEP_S="0.2", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
