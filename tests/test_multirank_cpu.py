"""The N > 1 host logic of the benchmark, on CPU with gloo ranks (world size 2).

The eviction path shards by request: every rank runs its own batch and the only
cross-rank steps are the barrier and the max-over-ranks of the timed region.  The
head-sharded (tensor-parallel) variant adds one all-reduce of the partial
importance, checked here against the oracle's importance over all heads.
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


def test_shard_heads_partitions_the_heads():
    from attention_delta_token_b200.parallel import shard_heads
    for Hq, Hkv, world in ((32, 8, 2), (32, 8, 4), (32, 8, 8), (32, 4, 4), (8, 8, 2)):
        G = Hq // Hkv
        seen_q, seen_k = [], []
        for r in range(world):
            hq, hk = shard_heads(Hq, Hkv, r, world)
            q = list(range(Hq))[hq]
            k = list(range(Hkv))[hk]
            assert q == [h for h in range(Hq) if h // G in k]  # each query head with its kv head
            seen_q += q
            seen_k += k
        assert seen_q == list(range(Hq)) and seen_k == list(range(Hkv))
    with pytest.raises(ValueError):
        shard_heads(32, 8, 0, 3)


def _tp_worker(rank, world, port, out_dir):
    """One rank of a head-sharded group on CPU: its partial importance comes from the
    oracle on its own head slice; the library call that follows the all-reduce is
    replaced by a recorder (no GPU here)."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        from attention_delta_token_b200 import make_dims, parallel
        p = synth.make_problem(0, seed=77, overrides=dict(R=3, Hq=8, Hkv=4))
        hq, hk = parallel.shard_heads(p.Hq, p.Hkv, rank, world)

        def partial(R, B, Hq_l, Hkv_l, d, q0, k0p, k0b, q1, k1p, k1b, cu, scale, **kw):
            i = [oracle.importance(q, kp, cu, kb, Hq=Hq_l, Hkv=Hkv_l, scale=scale)
                 for q, kp, kb in ((q0, k0p, k0b), (q1, k1p, k1b))]
            return torch.tensor(np.stack(i), dtype=torch.float32)

        seen = {}

        def finish(dims, importance, *a, **kw):
            seen["importance"] = importance.clone()

        parallel.partial_importance = partial
        parallel.finish_from_importance = finish
        dims = make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale)
        parallel.evict_head_sharded(
            dims, rank, world, p.q0[:, :, hq].contiguous(), p.k0_prefix[:, hk].contiguous(),
            p.k0_block[:, :, hk].contiguous(), p.q1[:, :, hq].contiguous(),
            p.k1_prefix[:, hk].contiguous(), p.k1_block[:, :, hk].contiguous(), p.cu_prefix,
            p.hidden, p.decoded, p.budget, None, None, None)
        full = [oracle.importance(q, kp, p.cu_prefix, kb, Hq=p.Hq, Hkv=p.Hkv, scale=p.scale)
                for q, kp, kb in ((p.q0, p.k0_prefix, p.k0_block), (p.q1, p.k1_prefix, p.k1_block))]
        np.save(os.path.join(out_dir, f"tp{rank}.npy"), seen["importance"].numpy())
        np.save(os.path.join(out_dir, "tp_full.npy"), np.stack(full))
    finally:
        dist.destroy_process_group()


def test_gloo_world2_head_sharded_importance_sums_to_the_full():
    """I_j sums over heads, so the all-reduced per-rank importances equal the oracle's
    importance over all heads, and every rank holds the same numbers before selecting."""
    import tempfile
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_tp_worker, args=(world, _free_port(), d), nprocs=world, join=True,
                           start_method="spawn")
        got = [np.load(os.path.join(d, f"tp{r}.npy")) for r in range(world)]
        full = np.load(os.path.join(d, "tp_full.npy"))
    np.testing.assert_array_equal(got[0], got[1])
    np.testing.assert_allclose(got[0], full, rtol=2e-6, atol=1e-6)
    assert (full > 0).all()
