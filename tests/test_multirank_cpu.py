"""The N > 1 host logic of the benchmark, on CPU with gloo ranks (world size 2).

The eviction path shards by request: every rank runs its own batch and the only
cross-rank steps are the barrier and the max-over-ranks of the timed region.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = 0.010 + 0.005 * rank  # a per-rank step time
        slowest = bench.max_over_ranks(local)
        dist.barrier()
        p = synth.make_problem(0, seed=bench.rank_seed(0, rank))
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "seed": bench.rank_seed(0, rank),
                       "q0_sum": float(p.q0.float().sum()), "shape": list(p.q0.shape),
                       "value": bench.job_throughput(world, p.R, slowest)}, f)
    finally:
        dist.destroy_process_group()


def test_gloo_world2_max_over_ranks_and_batches(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    assert all(abs(r["slowest"] - 0.015) < 1e-12 for r in res)     # the max, on every rank
    assert res[0]["seed"] != res[1]["seed"]                         # independent batches
    assert res[0]["shape"] == res[1]["shape"]                       # of the same shape
    assert res[0]["q0_sum"] != res[1]["q0_sum"]
    assert all(abs(r["value"] - world * 1 / 0.015) < 1e-6 for r in res)  # whole-job blocks/s


def test_single_process_helpers():
    import bench
    assert bench.max_over_ranks(0.25) == 0.25
    assert bench.job_throughput(4, 256, 0.5) == 2048.0


def test_reference_arm_under_torchrun_prints_once():
    """`bench.py --impl reference` under torchrun: rank 0 alone runs the oracle and
    prints one JSON line; the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           "2", "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "0",
           "--gpus", "2", "--steps", "3", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "blocks/s" and d["value"] > 0
    assert d["n_gpus"] == 2 and d["steps"] == 3
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
