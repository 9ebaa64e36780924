"""The bench's multi-rank host logic on CPU: two gloo ranks (no GPU).

Covers the max-over-ranks reduction of device times, the whole-job
throughput of weak scaling, distinct activations per rank over the same
weights, and the reference arm under torchrun (rank 0 alone prints)."""
import importlib.util
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


def load_bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = load_bench()
        # rank r measured (10 + r, 20 - r) ms: the job takes the max of each
        got = bench.max_over_ranks([10.0 + rank, 20.0 - rank], "cpu")
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        assert out[0] == out[1] == [11.0, 20.0]


def test_whole_job_throughput_and_rank_inputs():
    bench = load_bench()
    # 2 ranks, 3 steps, 606 MB per rank-step, slowest rank 1.5 ms total
    assert bench.whole_job_gbs(606e6, 2, 3, 1.5) == pytest.approx(2 * 3 * 606e6 / 1.5e-3 / 1e9)
    v = [bench.activation_variant(var, r) for r in range(4) for var in range(8)]
    assert len(set(v)) == len(v)  # every rank and call gets its own activations


def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--cpu-seconds", "1"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
