"""Seeded synthetic inputs for the FOCUS eviction step (shared by the tests,
the benchmark and the smoke check).

This module draws inputs only.  It holds none of the method's arithmetic: no
softmax, no importance, no delta, no pooling, no selection.  The one
construction it performs is the planted layer-1 key lift that gives a
selection margin (see ``make_problem``).

The workloads mirror the shapes of the FOCUS pages' SDAR-8B serving runs
("FOCUS: DLLMs Know How to Tame Their Compute Bound": Figure 2 and the
Referee Report summary name SDAR-8B-Chat with block size 32; the shapes below
are the five workload configurations this library is measured on).  The pages'
datasets (ShareGPT, WildChat, GSM8K, ...) are not used; these seeded draws
stand in for them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class FocusConfig:
    """One workload shape and its value distributions."""
    name: str
    R: int                      # requests (blocks) per step
    B: int                      # block size
    Hq: int                     # query heads
    Hkv: int                    # kv heads
    d: int                      # head dim
    H: int                      # hidden size
    prefix: tuple               # ('fixed', L) | ('uniform', lo, hi) | ('loguniform', hi)
    decoded: tuple              # ('exact', n) | ('uniform', lo, hi)
    lift: tuple                 # ('count', n) | ('frac', f) of the masked tokens
    budget: tuple               # ('fixed', K) | ('ceil', f): K = max(1, ceil(f * masked))
    tie_frac: float = 0.0       # fraction of blocks with a duplicated block key
    force_edges: bool = False   # force >=2 empty prefixes, >=2 all-masked, >=2 single-masked
    lift_size: float = 1.5      # logit rise planted on lifted tokens (layer 1)
    pool_window: int = 3


CONFIGS = [
    FocusConfig("tiny_r1_b32_l96", R=1, B=32, Hq=4, Hkv=2, d=64, H=256,
                prefix=("fixed", 96), decoded=("exact", 12), lift=("count", 4),
                budget=("fixed", 8)),
    FocusConfig("sdar8b_r32_b32", R=32, B=32, Hq=32, Hkv=8, d=128, H=4096,
                prefix=("uniform", 512, 2048), decoded=("uniform", 0.0, 0.8),
                lift=("frac", 0.10), budget=("ceil", 0.3)),
    FocusConfig("sdar8b_r256_b32", R=256, B=32, Hq=32, Hkv=8, d=128, H=4096,
                prefix=("uniform", 1024, 4096), decoded=("uniform", 0.0, 0.8),
                lift=("frac", 0.10), budget=("ceil", 0.25)),
    FocusConfig("large_block_r64_b128", R=64, B=128, Hq=32, Hkv=8, d=128, H=4096,
                prefix=("uniform", 1024, 4096), decoded=("uniform", 0.0, 0.9),
                lift=("frac", 0.08), budget=("ceil", 0.2)),
    FocusConfig("ragged_r128_b64", R=128, B=64, Hq=32, Hkv=4, d=128, H=2048,
                prefix=("loguniform", 8192), decoded=("uniform", 0.0, 1.0),
                lift=("frac", 0.10), budget=("ceil", 0.3), tie_frac=0.05, force_edges=True),
]

METRIC_CONFIG = 2  # SDAR-8B shape, 256 requests, B = 32


@dataclass
class FocusProblem:
    """All inputs of one eviction step, plus generation metadata.

    Layouts (row-major):
      q0, q1               [R, B, Hq, d]    bf16
      k0_prefix, k1_prefix [sum L, Hkv, d]  bf16 (request r owns rows cu_prefix[r]..cu_prefix[r+1]-1)
      k0_block, k1_block   [R, B, Hkv, d]   bf16
      hidden               [R, B, H]        bf16
      decoded              [R, B]           uint8 (1 = already decoded)
      budget               [R]              int32
      cu_prefix            [R + 1]          int32
    """
    R: int
    B: int
    Hq: int
    Hkv: int
    d: int
    H: int
    scale: float
    pool_window: int
    prefix_len: np.ndarray
    cu_prefix: torch.Tensor
    q0: torch.Tensor
    k0_prefix: torch.Tensor
    k0_block: torch.Tensor
    q1: torch.Tensor
    k1_prefix: torch.Tensor
    k1_block: torch.Tensor
    hidden: torch.Tensor
    decoded: torch.Tensor
    budget: torch.Tensor
    lifted: np.ndarray
    tie_pairs: list = field(default_factory=list)
    name: str = ""

    @property
    def total_prefix(self) -> int:
        return int(self.prefix_len.sum())

    def tensors(self):
        return dict(q0=self.q0, k0_prefix=self.k0_prefix, k0_block=self.k0_block,
                    q1=self.q1, k1_prefix=self.k1_prefix, k1_block=self.k1_block,
                    hidden=self.hidden, decoded=self.decoded, budget=self.budget,
                    cu_prefix=self.cu_prefix)

    def to(self, device) -> "FocusProblem":
        out = FocusProblem(**{**self.__dict__})
        for k, v in self.tensors().items():
            setattr(out, k, v.to(device))
        return out

    def subset(self, requests) -> "FocusProblem":
        """A problem holding only the listed requests (same data, repacked)."""
        req = [int(r) for r in requests]
        cu = self.cu_prefix.cpu().numpy().astype(np.int64)
        rows = [torch.arange(int(cu[r]), int(cu[r + 1])) for r in req]
        rows = torch.cat(rows) if rows else torch.zeros(0, dtype=torch.long)
        lens = self.prefix_len[req]
        sel = torch.tensor(req, dtype=torch.long)
        dev = self.q0.device
        out = FocusProblem(**{**self.__dict__})
        out.R = len(req)
        out.prefix_len = lens.copy()
        out.cu_prefix = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).to(dev)
        out.q0, out.q1 = self.q0[sel.to(dev)], self.q1[sel.to(dev)]
        out.k0_block, out.k1_block = self.k0_block[sel.to(dev)], self.k1_block[sel.to(dev)]
        out.k0_prefix = self.k0_prefix[rows.to(dev)].contiguous()
        out.k1_prefix = self.k1_prefix[rows.to(dev)].contiguous()
        out.hidden = self.hidden[sel.to(dev)]
        out.decoded = self.decoded[sel.to(self.decoded.device)]
        out.budget = self.budget[sel.to(self.budget.device)]
        out.lifted = self.lifted[req]
        out.tie_pairs = [(req.index(r), a, b) for (r, a, b) in self.tie_pairs if r in req]
        return out


def _draw_prefix(rng, cfg: FocusConfig) -> np.ndarray:
    kind = cfg.prefix[0]
    if kind == "fixed":
        return np.full(cfg.R, cfg.prefix[1], np.int64)
    if kind == "uniform":
        return rng.integers(cfg.prefix[1], cfg.prefix[2] + 1, size=cfg.R).astype(np.int64)
    if kind == "loguniform":
        hi = cfg.prefix[1]
        u = rng.uniform(0.0, math.log(hi + 1), size=cfg.R)
        return np.clip(np.floor(np.exp(u)).astype(np.int64) - 1, 0, hi)
    raise ValueError(kind)


def _bulk(gen, shape, std, device, chunk=1 << 26) -> torch.Tensor:
    """N(0, std^2) draws rounded to bf16, generated in float32 chunks."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = torch.randn(e - s, generator=gen, dtype=torch.float32, device=device)
        if std != 1.0:
            x.mul_(std)
        out[s:e] = x.to(torch.bfloat16)
    return out.view(*shape)


def make_problem(cfg: FocusConfig | int, seed: int | None = None, *, device="cpu",
                 wide_logits: bool = False, overrides: dict | None = None) -> FocusProblem:
    """Seeded inputs of one configuration.

    Draw order (fixed): prefix lengths, decoded sets, budgets, lift sets and
    direction u, duplicate-key ties (numpy PCG64); then Q0, K0 prefix, K0 block,
    Q1, K1 prefix, K1 block, hidden (torch generator on ``device``).

    Q and K elements are N(0, 1/d) (N(0, 1) with ``wide_logits``), rounded to bf16.
    Planted lift (a reading of "a planted layer-1 key lift (+lift_size along a
    shared random unit direction)"): every layer-1 query gets u / scale added,
    and every lifted token's layer-1 block key gets lift_size * u added for all
    kv heads, so each layer-1 logit toward a lifted token rises by about
    lift_size.  A duplicate-key tie copies an earlier masked position's layer-0
    and layer-1 block keys onto a later masked position of the same block.
    Hidden rows are N(0, 1) with element 0 = r and element 1 = j.
    """
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    if overrides:
        cfg = FocusConfig(**{**cfg.__dict__, **overrides})
    if seed is None:
        seed = CONFIGS.index(cfg) if cfg in CONFIGS else 0
    R, B, Hq, Hkv, d, H = cfg.R, cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.H
    rng = np.random.Generator(np.random.PCG64(seed))
    scale = 1.0 / math.sqrt(d)

    # 1. prefix lengths
    L = _draw_prefix(rng, cfg)
    # 2. decoded sets
    decoded = np.zeros((R, B), np.uint8)
    if cfg.decoded[0] == "exact":
        counts = np.full(R, cfg.decoded[1], np.int64)
    else:
        f = rng.uniform(cfg.decoded[1], cfg.decoded[2], size=R)
        counts = np.floor(f * B).astype(np.int64)
    if cfg.force_edges and R >= 6:
        pick = rng.choice(R, size=6, replace=False)
        L[pick[:2]] = 0
        counts[pick[2:4]] = 0          # every position still masked
        counts[pick[4:6]] = B - 1      # a single masked position
    counts = np.clip(counts, 0, B)
    for r in range(R):
        pos = rng.choice(B, size=int(counts[r]), replace=False)
        decoded[r, pos] = 1
    masked = (decoded == 0).sum(axis=1)
    # 3. budgets
    if cfg.budget[0] == "fixed":
        budget = np.full(R, cfg.budget[1], np.int32)
    else:
        budget = np.maximum(1, np.ceil(cfg.budget[1] * masked - 1e-9)).astype(np.int32)
    # 4. lift sets and direction
    lifted = np.zeros((R, B), bool)
    for r in range(R):
        mpos = np.flatnonzero(decoded[r] == 0)
        if cfg.lift[0] == "count":
            n = min(int(cfg.lift[1]), mpos.size)
        else:
            n = int(round(cfg.lift[1] * mpos.size))
            if mpos.size >= 1:
                n = max(n, 1)
        if n:
            lifted[r, rng.choice(mpos, size=n, replace=False)] = True
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    # 5. duplicate-key ties
    tie_pairs = []
    if cfg.tie_frac > 0:
        cand = [r for r in range(R) if masked[r] >= 2]
        n_tie = min(len(cand), max(1, int(round(cfg.tie_frac * R))))
        for r in sorted(rng.choice(cand, size=n_tie, replace=False).tolist()):
            a, b = sorted(rng.choice(np.flatnonzero(decoded[r] == 0), size=2, replace=False).tolist())
            tie_pairs.append((int(r), int(a), int(b)))

    # 6. bulk draws
    gen = torch.Generator(device=device).manual_seed(seed)
    std = 1.0 if wide_logits else 1.0 / math.sqrt(d)
    T = int(L.sum())
    q0 = _bulk(gen, (R, B, Hq, d), std, device)
    k0p = _bulk(gen, (T, Hkv, d), std, device)
    k0b = _bulk(gen, (R, B, Hkv, d), std, device)
    q1 = _bulk(gen, (R, B, Hq, d), std, device)
    k1p = _bulk(gen, (T, Hkv, d), std, device)
    k1b = _bulk(gen, (R, B, Hkv, d), std, device)
    hidden = _bulk(gen, (R, B, H), 1.0, device)

    # planted lift
    ut = torch.from_numpy(u).to(device=device, dtype=torch.float32)
    q1 = (q1.float() + ut / scale).to(torch.bfloat16)
    lt = torch.from_numpy(lifted).to(device)
    k1f = k1b.float()
    k1f[lt] += cfg.lift_size * ut
    k1b = k1f.to(torch.bfloat16)
    for (r, a, b) in tie_pairs:
        k0b[r, b] = k0b[r, a]
        k1b[r, b] = k1b[r, a]
    ar = torch.arange(R, device=device, dtype=torch.float32)
    aj = torch.arange(B, device=device, dtype=torch.float32)
    hidden[:, :, 0] = ar[:, None].to(torch.bfloat16)
    hidden[:, :, 1] = aj[None, :].to(torch.bfloat16)

    cu = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
    return FocusProblem(
        R=R, B=B, Hq=Hq, Hkv=Hkv, d=d, H=H, scale=scale, pool_window=cfg.pool_window,
        prefix_len=L, cu_prefix=torch.from_numpy(cu).to(device),
        q0=q0, k0_prefix=k0p, k0_block=k0b, q1=q1, k1_prefix=k1p, k1_block=k1b,
        hidden=hidden, decoded=torch.from_numpy(decoded).to(device),
        budget=torch.from_numpy(budget).to(device), lifted=lifted, tie_pairs=tie_pairs,
        name=cfg.name + ("_wide" if wide_logits else ""))



@dataclass
class PagedPrefix:
    """The prefix keys of a FocusProblem laid out as a paged KV pool.

    k0_pages, k1_pages [num_pages, page_size, Hkv, d] bf16: the pools of the two
    layers (same page table).  page_table [R, max_pages] int32 (entries past a
    request's pages are -1); prefix_len [R] int32.  Pages are handed out in a
    seeded random order and the unused tail of each request's last page holds
    unrelated random keys, so reading past a prefix shows up in the results.
    """
    k0_pages: torch.Tensor
    k1_pages: torch.Tensor
    page_table: torch.Tensor
    prefix_len: torch.Tensor
    page_size: int

    def to(self, device) -> "PagedPrefix":
        return PagedPrefix(self.k0_pages.to(device), self.k1_pages.to(device),
                           self.page_table.to(device), self.prefix_len.to(device), self.page_size)


def to_paged(p: FocusProblem, page_size: int, seed: int = 0, spare_pages: int = 3) -> PagedPrefix:
    L = p.prefix_len.astype(np.int64)
    pages = (L + page_size - 1) // page_size
    num_pages = int(pages.sum()) + spare_pages
    max_pages = max(1, int(pages.max()) if p.R else 1)
    rng = np.random.Generator(np.random.PCG64(seed))
    perm = rng.permutation(num_pages)
    table = np.full((p.R, max_pages), -1, np.int32)
    cu = p.cu_prefix.cpu().numpy().astype(np.int64)
    dev = p.k0_prefix.device
    gen = torch.Generator(device=dev).manual_seed(seed + 1)
    pools = []
    for kp in (p.k0_prefix, p.k1_prefix):
        pool = (torch.randn(num_pages, page_size, p.Hkv, p.d, generator=gen, device=dev) /
                math.sqrt(p.d)).to(torch.bfloat16)
        pools.append(pool)
    nxt = 0
    for r in range(p.R):
        for t in range(int(pages[r])):
            pg = int(perm[nxt])
            nxt += 1
            table[r, t] = pg
            a = int(cu[r]) + t * page_size
            b = min(int(cu[r + 1]), a + page_size)
            for pool, kp in zip(pools, (p.k0_prefix, p.k1_prefix)):
                pool[pg, :b - a] = kp[a:b]
    return PagedPrefix(pools[0], pools[1], torch.from_numpy(table).to(dev),
                       torch.from_numpy(L.astype(np.int32)).to(dev), page_size)
