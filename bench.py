#!/usr/bin/env python
"""Throughput of the FOCUS importance-delta token eviction step on B200.

One step = one fused focus_evict call over a batch of blocks: layer-0 and
layer-1 attention importance, delta, MaxPool1D, mask, top-K, compaction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--config C]

Default workload: SDAR-8B shape, 256 requests, B = 32, prefix lengths
U[1024, 4096], Hq = 32, Hkv = 8, d = 128, hidden = 4096 (seeded synthetic bf16).
N > 1 runs under torchrun, one rank per GPU; every rank processes its own batch
(independent requests: weak scaling, no collective on the data path); the
time is the max over ranks.  Prints one JSON line on rank 0.  --tp-shards S
instead splits the heads S ways (the tensor-parallel form: one all-reduce of
the partial importance per step under torchrun with N = S).

--impl reference times the float64 CPU oracle (the checker the tests use) on
the host cores, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "eviction blocks/s at SDAR-8B shape, batch 256, B=32; % of HBM roofline"
UNIT = "blocks/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SOURCES = ["attn_stats.cu", "focus_device.cuh", "focus_kernels.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_stats_traffic.txt")
TRACE_EVERY = 8  # timed steps between two CUDA-event measurements of the attention kernel


# ---------------------------------------------------------------- accounting

def algorithmic_counts(p, layers: int = 2, lse0: bool = False) -> dict:
    """Work the method must do per step (not what an implementation happens to do).

    attention: each of the `layers` layers (2; 1 when ranking by I1 alone) reads
    every prefix and block key once (Hkv x d bf16 per key) and every block query
    once; flops 2*d per (query row, key) per layer; one exp per (query row, key)
    per layer.  With `lse0` (layer 0's row log-sum-exps given) layer 0 reads only its
    B block keys, Q0 and the LSEs.  Select/compact: the mask, budget, kept indices,
    cu_seqlens, and the kept hidden rows read once and written once.
    """
    L = p.prefix_len.astype(np.int64)
    N = L + p.B
    dec = p.decoded.cpu().numpy()
    masked = (dec == 0).sum(1).astype(np.int64)
    k = np.minimum(np.clip(p.budget.cpu().numpy().astype(np.int64), 0, None), masked)
    n0 = np.full_like(N, p.B) if lse0 else N  # keys layer 0 streams
    attn = layers * (p.B * p.Hq * p.d * 2) + N * p.Hkv * p.d * 2
    flops = 2 * p.Hq * p.B * N * p.d
    exps = p.Hq * p.B * N
    if layers == 2:
        attn = attn + n0 * p.Hkv * p.d * 2 + (p.B * p.Hq * 4 if lse0 else 0)
        flops = flops + 2 * p.Hq * p.B * n0 * p.d
        exps = exps + p.Hq * p.B * n0
    rest = p.B + 4 + 4 * k + 4 + k * p.H * 2 * 2
    return dict(attn_bytes=int(attn.sum()), bytes=int(attn.sum() + rest.sum() + 4),
                flops=int(flops.sum()), exps=int(exps.sum()), decisions=int(masked.sum()),
                kept_rows=int(k.sum()), blocks=int(p.R))


def read_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "attention_delta_token_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary, or None when
    the kernel sources changed since the counters were taken."""
    try:
        kv = {}
        for line in open(TRAFFIC_FILE):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("kernel_sources_sha256_16") != attn_source_hash():
            return None
        return int(kv[f"dram_bytes_per_launch[{workload}]"])
    except Exception:
        return None


# ---------------------------------------------------------------- clocks

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


# The sampling loop runs in a child process of its own, so that it keeps its period
# while this process waits for the GPU (a thread here would wait for the interpreter
# lock).  It only reads NVML: SM clock and clock-event reasons, one line per sample,
# until its standard input closes.
_SAMPLER_SRC = r"""
import select, sys, time
import pynvml
pynvml.nvmlInit()
dev, period, out = sys.argv[1], float(sys.argv[2]), sys.argv[3]
h = (pynvml.nvmlDeviceGetHandleByUUID(dev) if dev.startswith("GPU-")
     else pynvml.nvmlDeviceGetHandleByIndex(int(dev)))
with open(out, "w") as f:
    f.write("max %d\n" % pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
    f.flush()
    while True:
        t = time.monotonic()
        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        f.write("%.6f %d %d\n" % (t, sm, rs))
        if select.select([sys.stdin], [], [], period)[0]:
            break
"""


class ClockSampler:
    """Reads SM clock and clock-event reasons through NVML every `period` seconds
    (in a child process) while the timed region runs; `mark_start` / `mark_stop`
    bracket the region the summary covers.  Read-only: it changes no GPU setting."""

    def __init__(self, device_index: int, period: float = 0.0005):
        self.samples = []      # (monotonic time, SM MHz, reason bits)
        self.period = period
        self.sm_max = None
        self.window = [None, None]
        self._proc = None
        self._file = None
        try:
            import pynvml  # noqa: F401  (the child needs it)
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self.dev = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            except Exception:
                self.dev = str(device_index)
            self.ok = True
        except Exception:
            self.ok = False

    def __enter__(self):
        if not self.ok:
            return self
        import subprocess
        import tempfile
        fd, self._file = tempfile.mkstemp(prefix="focus_clocks_", suffix=".txt")
        os.close(fd)
        self._proc = subprocess.Popen(
            [sys.executable, "-c", _SAMPLER_SRC, self.dev, str(self.period), self._file],
            stdin=subprocess.PIPE, stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        t0 = time.monotonic()
        while time.monotonic() - t0 < 20.0:  # until the first sample is written
            if self._proc.poll() is not None:
                break
            with open(self._file) as f:
                if len(f.read().splitlines()) >= 2:
                    break
            time.sleep(0.01)
        return self

    def mark_start(self):
        self.window[0] = time.monotonic()

    def mark_stop(self):
        self.window[1] = time.monotonic()

    def __exit__(self, *a):
        if self._proc is None:
            return
        try:
            self._proc.stdin.close()
            self._proc.wait(timeout=10)
        except Exception:
            self._proc.kill()
        try:
            for line in open(self._file).read().splitlines():
                parts = line.split()
                if parts[0] == "max":
                    self.sm_max = int(parts[1])
                elif len(parts) == 3:
                    self.samples.append((float(parts[0]), int(parts[1]), int(parts[2])))
        except Exception:
            pass
        finally:
            os.unlink(self._file)

    def summary(self) -> dict:
        sel = self.samples
        lo, hi = self.window
        if lo is not None and hi is not None:
            inside = [x for x in self.samples if lo <= x[0] <= hi]
            if inside:
                sel = inside
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": [], "samples": 0}
        sms = [sm for _, sm, _ in sel]
        bits = 0
        for _, _, r in sel:
            bits |= r
        names = [n for b, n in REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(sms)), "sm_max_mhz": self.sm_max,
                "reasons": names, "samples": len(sms)}


# ---------------------------------------------------------------- our arm

def layer0_row_lse(p) -> torch.Tensor:
    """Layer-0 row log-sum-exps [R, B, Hq] over each row's prefix and block keys, in
    float32 on the device: the input an engine's layer-0 attention forward hands over
    (computed here with torch as setup, outside the timed region)."""
    G = p.Hq // p.Hkv
    cu = p.cu_prefix.cpu().numpy()
    out = torch.empty(p.R, p.B, p.Hq, dtype=torch.float32, device=p.q0.device)
    for r in range(p.R):
        keys = torch.cat([p.k0_prefix[int(cu[r]):int(cu[r + 1])], p.k0_block[r]], 0).float()
        q = p.q0[r].float()  # [B, Hq, d]
        for g in range(p.Hkv):
            qs = q[:, g * G:(g + 1) * G].reshape(-1, p.d)
            s = p.scale * (qs @ keys[:, g].T)
            out[r, :, g * G:(g + 1) * G] = torch.logsumexp(s, dim=-1).view(p.B, G)
    return out


def make_outputs(p, cap, dev):
    kept = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)[:cap]
    cu = torch.empty(p.R + 1, dtype=torch.int32, device=dev)
    packed = torch.empty(max(cap, 1), p.H, dtype=torch.bfloat16, device=dev)[:cap]
    return kept, cu, packed


def rank_seed(config: int, rank: int) -> int:
    """Each rank draws its own batch of the same shape (independent requests)."""
    return config + 1000 * rank


def max_over_ranks(x: float, device=None) -> float:
    """The slowest rank's time (all ranks must call this in the same order)."""
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, blocks_per_rank: int, seconds_per_step: float) -> float:
    """Whole-job blocks/s: every rank processes `blocks_per_rank` blocks per step."""
    return world * blocks_per_rank / seconds_per_step


def workload_config(args):
    """The benchmark's workload: a synthetic config with the command line's overrides
    (both arms use the same one)."""
    cfg = synth.CONFIGS[args.config]
    if args.requests:
        cfg = synth.FocusConfig(**{**cfg.__dict__, "R": args.requests,
                                   "name": f"{cfg.name}_r{args.requests}"})
    if args.prefix:
        lo, hi = args.prefix
        cfg = synth.FocusConfig(**{**cfg.__dict__, "prefix": ("uniform", lo, hi),
                                   "name": f"{cfg.name}_l{lo}_{hi}"})
    return cfg


def run_ours(args, rank, world, local_rank):
    import attention_delta_token_b200 as F
    dist = torch.distributed if world > 1 else None
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = workload_config(args)
    tp = args.tp_shards
    # head-sharded ranks all work on the same requests; request-sharded ones on their own
    seed = rank_seed(args.config, 0 if tp > 1 else rank)
    p = synth.make_problem(cfg, seed=seed, device=dev)
    counts = algorithmic_counts(p, layers=1 if args.score else 2, lse0=args.lse0)
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window, args.constraints,
                       args.score)
    ws = F.Workspace(dims, dev)
    cap = F.plan_capacity(p.decoded, p.budget, args.constraints)
    kept, cu, packed = make_outputs(p, cap, dev)
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(t.numel() * t.element_size() for t in p.tensors().values())

    layer0 = (None, None, None) if args.score else (p.q0, p.k0_prefix, p.k0_block)
    tp_ws = None
    if tp > 1:
        # This rank's head slice: focus_partial_importance, the all-reduce of the
        # [2, R, B] sums (NCCL, only with one rank per shard), then the shared selection.
        from attention_delta_token_b200.parallel import shard_heads
        hq, hk = shard_heads(p.Hq, p.Hkv, rank if world > 1 else 0, tp)
        sl = {k: (v[:, :, hq] if k.startswith("q") else v[:, :, hk] if k.endswith("block")
                  else v[:, hk]).contiguous()
              for k, v in p.tensors().items() if k[:2] in ("q0", "q1", "k0", "k1")}
        sdims = F.make_dims(p.R, p.B, p.Hq // tp, p.Hkv // tp, p.d, 8, p.scale, p.pool_window,
                            0, args.score)
        tp_ws = F.Workspace(sdims, dev)
        imp = torch.empty(2, p.R, p.B, dtype=torch.float32, device=dev)
        s_l0 = (None, None, None) if args.score else (sl["q0"], sl["k0_prefix"], sl["k0_block"])
        counts = algorithmic_counts(dataclasses.replace(p, Hq=p.Hq // tp, Hkv=p.Hkv // tp),
                                    layers=1 if args.score else 2)

        if args.tp_exchange == "p2p":
            # the sums travel inside the kernels: pushed into every rank's exchange buffer
            from attention_delta_token_b200.parallel import PeerExchange
            ex = (PeerExchange.symmetric(dims) if world > 1 else PeerExchange.local(dims, dev))

            def step():
                epoch = ex.next_epoch()
                F.focus_partial_importance_push(sdims, *s_l0, sl["q1"], sl["k1_prefix"],
                                                sl["k1_block"], p.cu_prefix, ex.peer_ptrs,
                                                ex.rank, ex.world, epoch, tp_ws)
                F.focus_evict_from_exchange(dims, ex.buffer, ex.world, epoch, p.hidden,
                                            p.decoded, p.budget, kept, cu, packed, ws)
        else:
            def step():
                F.focus_partial_importance(sdims, *s_l0, sl["q1"], sl["k1_prefix"],
                                           sl["k1_block"], p.cu_prefix, imp, tp_ws)
                if world > 1:
                    dist.all_reduce(imp)
                F.focus_evict_from_importance(dims, imp, p.hidden, p.decoded, p.budget, kept,
                                              cu, packed, ws)
    elif args.dynamic_budget:
        # historical decoded-per-step averages: ~10% of a 32-token block per step
        # (Figure 2), drawn uniformly in [0, 0.2 B] per request
        gen = torch.Generator().manual_seed(seed)
        decode_avg = (torch.rand(p.R, generator=gen) * 0.2 * p.B).to(dev)
        budget_out = torch.empty(p.R, dtype=torch.int32, device=dev)
        cap = F.plan_capacity(p.decoded, None, args.constraints, dynamic=True)
        kept, cu, packed = make_outputs(p, cap, dev)

        def step():
            F.focus_evict_ex(dims, q0=p.q0, k0_prefix=p.k0_prefix, k0_block=p.k0_block, q1=p.q1,
                             k1_prefix=p.k1_prefix, k1_block=p.k1_block, cu_prefix=p.cu_prefix,
                             hidden=p.hidden, decoded=p.decoded, decode_avg=decode_avg,
                             budget_alpha=1.5, budget_out=budget_out, kept_idx=kept,
                             cu_seqlens=cu, packed=packed, ws=ws)
    elif args.page_size:
        pg = synth.to_paged(p, args.page_size, seed=seed)

        def step():
            F.focus_evict_paged(dims, p.q0, pg.k0_pages, p.k0_block, p.q1, pg.k1_pages, p.k1_block,
                                pg.page_table, pg.prefix_len, p.hidden, p.decoded, p.budget, kept,
                                cu, packed, ws)
    elif args.lse0:
        torch.backends.cuda.matmul.allow_tf32 = False
        lse0 = layer0_row_lse(p)

        def step():
            F.focus_evict_with_lse0(dims, lse0, p.q0, p.k0_block, p.q1, p.k1_prefix, p.k1_block,
                                    p.cu_prefix, p.hidden, p.decoded, p.budget, kept, cu,
                                    packed, ws)
    else:
        def step():
            F.focus_evict(dims, *layer0, p.q1, p.k1_prefix, p.k1_block,
                          p.cu_prefix, p.hidden, p.decoded, p.budget, kept, cu, packed, ws)

    def barrier():
        torch.cuda.synchronize(dev)
        if dist:
            dist.barrier()

    # ---- device-resident timing
    graph = None
    sampler = ClockSampler(local_rank)
    with sampler:
        for _ in range(args.warmup):
            step()
        barrier()
        if args.graph:
            # the whole step captured once (its kernels keep their programmatic
            # dependent launch edges) and replayed: one launch of host work per step
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=torch.cuda.Stream(dev)):
                step()
            graph.replay()
            barrier()
        # The attention kernel is timed on every TRACE_EVERY-th step: events around it
        # break the launch overlap with the planner, so they are not on every step.
        # A graph replay cannot be traced: then the same number of direct steps are
        # traced right after the timed loop.
        traced = list(range(0, args.steps, TRACE_EVERY))
        ev_a = [torch.cuda.Event(enable_timing=True) for _ in traced]
        ev_b = [torch.cuda.Event(enable_timing=True) for _ in traced]
        for e in ev_a + ev_b:
            e.record(stream)
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        barrier()
        sampler.mark_start()
        start.record(stream)
        for k in range(args.steps):
            if graph is not None:
                graph.replay()
                continue
            if k % TRACE_EVERY == 0:
                F.focus_set_trace_events(ev_a[k // TRACE_EVERY], ev_b[k // TRACE_EVERY])
            step()
            if k % TRACE_EVERY == 0:
                F.focus_set_trace_events(None, None)
        stop.record(stream)
        barrier()
        sampler.mark_stop()
        if graph is not None:
            for i in range(len(traced)):
                F.focus_set_trace_events(ev_a[i], ev_b[i])
                step()
                F.focus_set_trace_events(None, None)
            barrier()
    for w in (ws, tp_ws) if tp_ws is not None else (ws,):
        status = F.focus_read_device_status(w)
        if status != 0:
            raise RuntimeError(f"device status {F.focus_status_string(status)}")
    elapsed = start.elapsed_time(stop) / 1e3
    attn_s = sum(a.elapsed_time(b) for a, b in zip(ev_a, ev_b)) / 1e3 / len(traced)
    elapsed_max = max_over_ranks(elapsed, dev)
    attn_s_max = max_over_ranks(attn_s, dev)
    step_s = elapsed_max / args.steps

    # ---- sustained: the same step repeated for about --sustained-seconds after the timed
    # steps (not part of ms_per_step), so the line also shows the rate once the board has
    # reached its power limit.  Every rank runs the same count (from the max-over-ranks time).
    sustained = None
    if args.sustained_seconds > 0:
        n_sus = max(1, math.ceil(args.sustained_seconds / step_s))
        s_sampler = ClockSampler(local_rank)
        with s_sampler:
            s3 = torch.cuda.Event(enable_timing=True)
            t3 = torch.cuda.Event(enable_timing=True)
            barrier()
            s3.record(stream)
            for _ in range(n_sus):
                if graph is not None:
                    graph.replay()
                else:
                    step()
            t3.record(stream)
            barrier()
        sus_s = max_over_ranks(s3.elapsed_time(t3) / 1e3, dev) / n_sus
        sustained = {"value": p.R / sus_s if tp > 1 else job_throughput(world, p.R, sus_s),
                     "unit": UNIT, "ms_per_step": sus_s * 1e3, "steps": n_sus,
                     "seconds": sus_s * n_sus, "clocks": s_sampler.summary()}
        if F.focus_read_device_status(ws) != 0:
            raise RuntimeError("device status after the sustained run")

    # ---- end to end: pinned host inputs -> device, the C-ABI call, result -> host
    e2e = None
    variant = args.score or args.lse0 or args.page_size or args.dynamic_budget or tp > 1
    if not args.no_e2e and not variant:
        host = {k: v.to("cpu").pin_memory() for k, v in p.tensors().items()}
        dev_t = p.tensors()
        out_kept = torch.empty(kept.shape, dtype=kept.dtype).pin_memory()
        out_cu = torch.empty(cu.shape, dtype=cu.dtype).pin_memory()
        out_packed = torch.empty(packed.shape, dtype=packed.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in (out_kept, out_cu, out_packed))
        n_e2e = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            for k, t in host.items():
                dev_t[k].copy_(t, non_blocking=True)
            step()
            out_kept.copy_(kept, non_blocking=True)
            out_cu.copy_(cu, non_blocking=True)
            out_packed.copy_(packed, non_blocking=True)

        e2e_step()
        barrier()
        s2 = torch.cuda.Event(enable_timing=True)
        t2 = torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        t2.record(stream)
        barrier()
        e2e_s = max_over_ranks(s2.elapsed_time(t2) / 1e3, dev) / n_e2e
        e2e = {"value": job_throughput(world, p.R, e2e_s), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": n_e2e, "ms_per_step": e2e_s * 1e3,
               "path": "pinned host -> cudaMemcpyAsync -> focus_evict -> host"}
        if F.focus_read_device_status(ws) != 0:
            raise RuntimeError("device status after e2e")

    result = None
    if rank == 0:
        peaks, peak_src = read_peaks()
        hbm = float(peaks["hbm_gbs"])
        tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        achieved = counts["attn_bytes"] / attn_s_max / 1e9
        t_hbm = counts["bytes"] / (hbm * 1e9)
        t_tc = counts["flops"] / (tc * 1e12)
        workload = cfg.name
        clocks = sampler.summary()
        sm_hz = (clocks["sm_mhz"] or 1965.0) * 1e6
        t_mufu = counts["exps"] / (16 * 148 * sm_hz)  # one SFU exp per (row, key): 16 per clock per SM
        result = {
            "metric": METRIC,
            "value": p.R / step_s if tp > 1 else job_throughput(world, p.R, step_s), "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "strong" if tp > 1 else "weak",
            "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {
                "workload": workload, "R": p.R, "B": p.B, "Hq": p.Hq, "Hkv": p.Hkv, "d": p.d,
                "hidden": p.H, "prefix": list(cfg.prefix), "total_prefix": p.total_prefix,
                "seed": seed, "kept_rows": counts["kept_rows"],
                "input_bytes_per_step": int(in_bytes),
                "l2": f"no flush: {in_bytes / 2**30:.2f} GiB of inputs per step > 126 MB L2",
                "accumulate": "fp32",
                "parallelism": (f"dp{world} (request-sharded replicas)" if tp <= 1 else
                                f"tp{tp} (head-sharded; partial importance exchanged by "
                                f"{'peer stores inside the kernels' if args.tp_exchange == 'p2p' else 'NCCL all-reduce'})"
                                if world > 1 else
                                f"tp{tp} emulated: rank 0's head shard + the shared selection "
                                "timed on one GPU" + (", exchanging with itself through its "
                                "exchange buffer" if args.tp_exchange == "p2p" else
                                ", no all-reduce")),
                "constraints": args.constraints, "score": args.score, "lse0": args.lse0,
                "page_size": args.page_size, "dynamic_budget": args.dynamic_budget,
                "launch": "CUDA graph replay" if args.graph else "direct C-ABI calls",
            },
            "decisions_per_s": world * counts["decisions"] / step_s,
            "roofline": {
                "bound": "hbm", "kernel": "attn_stats_kernel", "achieved": achieved,
                "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": read_traffic(workload) if not variant else None,
                "algorithmic_bytes_per_launch": counts["attn_bytes"],
                "ms_per_launch": attn_s_max * 1e3, "peak_source": f"{peak_src} (hbm_gbs)",
                "launches_timed": len(traced),
                "timed_on": ("direct steps after the graph-replay loop" if args.graph else
                             "every 8th step of the timed loop"),
                "note": f"frac of {peak_src} HBM copy bandwidth",
            },
            "roofline_step": {
                "t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_tc * 1e6,
                "t_mufu_us": t_mufu * 1e6,
                "frac": max(t_hbm, t_tc) / step_s,
                "frac_with_sfu": max(t_hbm, t_tc, t_mufu) / step_s, "bytes": counts["bytes"],
                "flops": counts["flops"], "exps": counts["exps"],
                "peaks": f"{peak_src}: hbm {hbm} GB/s, bf16 {tc} TFLOP/s",
            },
            "clocks": clocks,
            "sustained": sustained,
            # plan, attention statistics, select, (scan,) compact; split into two calls
            # (tp): plan, attention, reduce + plan, select, (scan,) compact
            # (list mode: structural constraints or the dynamic budget add the scan kernel)
            "gpu_launches": ((5 if (args.constraints or args.dynamic_budget) else 4) +
                             (2 if tp > 1 else 0)) * args.steps,
            "e2e": e2e,
            "impl": "ours",
        }
    return result, p


def cpu_baseline(p, target_s: float = 12.0) -> dict:
    """The oracle as it stands, on a bounded sample of the same workload (rank 0, N=1)."""
    import oracle
    threads = oracle.num_threads()
    n0 = max(1, min(p.R, threads // max(1, p.Hkv)))
    cpu_p = p.subset(range(n0)).to("cpu")
    t0 = time.perf_counter()
    oracle.evict(cpu_p)
    t = time.perf_counter() - t0
    n = n0
    if t < target_s / 2 and n0 < p.R:
        n = int(min(p.R, max(n0 + 1, round(n0 * target_s / max(t, 1e-3)))))
        cpu_p = p.subset(range(n)).to("cpu")
        t0 = time.perf_counter()
        oracle.evict(cpu_p)
        t = time.perf_counter() - t0
    single = cpu_baseline_single_thread(p, target_s=target_s / 2)
    return {"value": n / t, "unit": UNIT, "cores": threads, "kind": "oracle",
            "seconds": t,
            "sample": f"requests 0..{n - 1} ({n} of {p.R} blocks) of the same workload; "
                      f"both layers' importance, delta, pooling, mask, top-K, compaction in "
                      f"float64 (OpenMP over request x kv-head pairs)",
            "single_thread": single}


def cpu_baseline_single_thread(p, target_s: float = 6.0) -> dict:
    """The same oracle on one host thread, on the first few requests of the workload
    (2, then as many as fit in about `target_s`)."""
    import oracle
    threads = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        n = min(p.R, 2)
        sub = p.subset(range(n)).to("cpu")
        t0 = time.perf_counter()
        oracle.evict(sub)
        t = time.perf_counter() - t0
        if t < target_s / 2 and n < p.R:
            n = int(min(p.R, max(n + 1, round(n * target_s / max(t, 1e-3)))))
            sub = p.subset(range(n)).to("cpu")
            t0 = time.perf_counter()
            oracle.evict(sub)
            t = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(threads)
    return {"value": n / t, "unit": UNIT, "cores": 1, "seconds": t,
            "sample": f"requests 0..{n - 1} ({n} of {p.R} blocks), one thread"}


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    """The float64 CPU oracle on host cores; each step a bounded sample of the workload."""
    import oracle
    cfg = workload_config(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    p = synth.make_problem(cfg, seed=rank_seed(args.config, 0), device=dev)
    threads = oracle.num_threads()
    n = max(1, min(p.R, threads // max(1, p.Hkv)))
    subsets = {}

    def sample(step_idx):
        start = (step_idx * n) % p.R
        req = [(start + i) % p.R for i in range(n)]
        key = tuple(req)
        if key not in subsets:
            subsets[key] = p.subset(req).to("cpu")
        return subsets[key]

    for w in range(args.warmup):
        oracle.evict(sample(w))
    total = 0.0
    for s in range(args.steps):
        sp = sample(args.warmup + s)
        t0 = time.perf_counter()
        oracle.evict(sp)
        total += time.perf_counter() - t0
    step_s = total / max(1, args.steps)
    value = n / step_s
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": cfg.name, "R": p.R, "B": p.B, "Hq": p.Hq, "Hkv": p.Hkv, "d": p.d,
                   "hidden": p.H, "prefix": list(cfg.prefix), "seed": rank_seed(args.config, 0)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{n} requests per step, cycling through the {p.R}-block "
                                   f"workload; float64, OpenMP over request x kv-head pairs"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=synth.METRIC_CONFIG)
    ap.add_argument("--requests", type=int, default=0,
                    help="override the workload's request count (same shape; for profiling)")
    ap.add_argument("--prefix", type=int, nargs=2, metavar=("LO", "HI"), default=None,
                    help="override the prefix lengths: uniform in [LO, HI] keys (same shape otherwise)")
    ap.add_argument("--constraints", type=int, default=0, choices=[0, 1, 2, 3],
                    help="structural constraints on the retained set (bit 1: predecessors, "
                         "bit 2: masked tokens left of the rightmost candidate)")
    ap.add_argument("--score", type=int, default=0, choices=[0, 1],
                    help="0: rank by I1 - I0 (the method); 1: by I1 alone (layer 0 skipped)")
    ap.add_argument("--lse0", action="store_true",
                    help="layer 0's row log-sum-exps are given (focus_evict_with_lse0)")
    ap.add_argument("--page-size", type=int, default=0,
                    help="read the prefix keys from a paged pool with pages of this many tokens "
                         "(focus_evict_paged)")
    ap.add_argument("--dynamic-budget", action="store_true",
                    help="dynamic retention budget (focus_evict_ex with decode_avg)")
    ap.add_argument("--tp-shards", type=int, default=1,
                    help="head-sharded (tensor-parallel) step over this many head shards: under "
                         "torchrun one rank per shard with an NCCL all-reduce; on one GPU rank "
                         "0's share is timed")
    ap.add_argument("--tp-exchange", choices=["nccl", "p2p"], default="nccl",
                    help="with --tp-shards: NCCL all-reduce between two library calls, or the "
                         "exchange fused into the kernels over peer memory")
    ap.add_argument("--graph", action="store_true",
                    help="replay the step as a captured CUDA graph in the timed loop")
    ap.add_argument("--sustained-seconds", type=float, default=1.0,
                    help="after the timed steps, repeat the step for about this long and report "
                         "its rate and clocks separately (0: skip)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.tp_shards > 1 and (args.lse0 or args.page_size or args.dynamic_budget):
        ap.error("--tp-shards combines with --constraints and --score only")
    if args.graph and args.tp_shards > 1 and (args.tp_exchange == "p2p" or args.gpus > 1):
        ap.error("--graph: the exchange's epoch and the collective must run uncaptured")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if world > 1 and args.tp_shards > 1 and args.tp_shards != world:
        ap.error("--tp-shards under torchrun needs one rank per shard (N = S)")

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=300),
            device_id=torch.device("cuda", local_rank))
    try:
        result, p = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                result["cpu_baseline"] = cpu_baseline(p)
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
