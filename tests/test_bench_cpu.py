"""The benchmark's host-side accounting, on CPU: the algorithmic work counts behind
every roofline number, and the workload overrides both arms share."""
import argparse

import numpy as np

import bench
import synth


def _args(**kw):
    base = dict(config=0, requests=0, prefix=None)
    base.update(kw)
    return argparse.Namespace(**base)


def test_algorithmic_counts_tiny_config_by_hand():
    """Config 0: one block, B = 32, L = 96 prefix keys, Hq = 4, Hkv = 2, d = 64, H = 256,
    12 decoded positions, budget 8.  N = L + B = 128 keys per layer."""
    p = synth.make_problem(0)
    c = bench.algorithmic_counts(p)
    N, B, Hq, Hkv, d, H = 128, 32, 4, 2, 64, 256
    attn = 2 * (N * Hkv * d * 2 + B * Hq * d * 2)            # K read once, Q once, per layer
    assert c["attn_bytes"] == attn == 98304
    k = 8                                                    # min(budget, masked = 20)
    rest = B + 4 + 4 * k + 4 + k * H * 2 * 2                 # mask, budget, kept, cu, rows r+w
    assert c["bytes"] == attn + rest + 4
    assert c["flops"] == 2 * (2 * Hq * B * N * d) == 4194304
    assert c["exps"] == 2 * Hq * B * N == 32768
    assert c["kept_rows"] == k and c["decisions"] == 20 and c["blocks"] == 1


def test_algorithmic_counts_variants():
    p = synth.make_problem(0)
    full = bench.algorithmic_counts(p)
    one = bench.algorithmic_counts(p, layers=1)              # ranking by I1 alone
    assert one["flops"] * 2 == full["flops"] and one["exps"] * 2 == full["exps"]
    lse = bench.algorithmic_counts(p, lse0=True)             # layer 0 streams only its B keys
    N, B, Hq, Hkv, d = 128, 32, 4, 2, 64
    assert lse["attn_bytes"] == (N * Hkv * d * 2 + B * Hq * d * 2) + \
        (B * Hkv * d * 2 + B * Hq * d * 2 + B * Hq * 4)
    assert lse["exps"] == Hq * B * N + Hq * B * B


def test_algorithmic_counts_scale_with_heads():
    """A head shard of a tensor-parallel group does 1/S of the attention work."""
    import dataclasses
    p = synth.make_problem(1, overrides=dict(R=3))
    full = bench.algorithmic_counts(p)
    half = bench.algorithmic_counts(dataclasses.replace(p, Hq=p.Hq // 2, Hkv=p.Hkv // 2))
    assert half["attn_bytes"] * 2 == full["attn_bytes"]
    assert half["flops"] * 2 == full["flops"]


def test_workload_overrides():
    cfg = bench.workload_config(_args(config=2))
    assert cfg is synth.CONFIGS[2]
    cfg = bench.workload_config(_args(config=1, requests=4, prefix=[15000, 16000]))
    assert cfg.R == 4 and cfg.prefix == ("uniform", 15000, 16000)
    assert cfg.name == "sdar8b_r32_b32_r4_l15000_16000"
    p = synth.make_problem(cfg, seed=bench.rank_seed(1, 0))
    assert p.R == 4 and (p.prefix_len >= 15000).all() and (p.prefix_len <= 16000).all()
    assert bench.rank_seed(2, 0) == 2 and bench.rank_seed(2, 1) != 2
    assert np.isclose(bench.job_throughput(2, 256, 0.5), 1024.0)


def test_cpu_baseline_reports_all_core_and_single_thread():
    """The oracle's timing on the host: the all-core figure and a one-thread figure on
    a sample of the same workload, with the thread count restored afterwards."""
    import oracle
    p = synth.make_problem(1, overrides=dict(R=4, prefix=("uniform", 0, 200)))
    threads = oracle.num_threads()
    cb = bench.cpu_baseline(p, target_s=0.2)
    assert cb["kind"] == "oracle" and cb["cores"] == threads and cb["value"] > 0
    one = cb["single_thread"]
    assert one["cores"] == 1 and one["value"] > 0 and one["unit"] == "blocks/s"
    assert oracle.num_threads() == threads
