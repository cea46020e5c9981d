"""Shared helpers of the parity tests: run the CUDA path through the C ABI and
compare its outputs with the float64 oracle.

Tolerances (bf16 inputs, fp32 accumulation on the GPU, float64 in the oracle):
  I0, I1, delta:  |gpu - oracle| <= 2e-3 + 1e-2 * |oracle|   (allclose convention)
  masked entries: -inf on both sides, exactly
  kept positions: identical, except that a position may differ only where its
                  oracle pooled delta lies within 2e-3 of the k-th largest value
  packed rows:    bit-exact copies of hidden[r, kept]
"""
from __future__ import annotations

import numpy as np
import torch

ATOL = 2e-3
RTOL = 1e-2
TIE_TOL = 2e-3


def run_evict(p, *, outputs=True, capacity=None, stream=None, constraints=0, score=0):
    """focus_evict on a problem whose tensors live on the GPU.  Returns numpy arrays."""
    import attention_delta_token_b200 as F
    dev = p.q1.device
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window, constraints,
                       score)
    ws = F.Workspace(dims, dev)
    cap = F.plan_capacity(p.decoded, p.budget, constraints) if capacity is None else capacity
    kept = torch.full((max(cap, 1),), -1, dtype=torch.int32, device=dev)[:cap]
    cu = torch.full((p.R + 1,), -7, dtype=torch.int32, device=dev)
    packed = torch.zeros((max(cap, 1), p.H), dtype=torch.bfloat16, device=dev)[:cap]
    mk = (lambda: torch.full((p.R, p.B), float("nan"), device=dev)) if outputs else (lambda: None)
    delta, i0, i1 = mk(), mk(), mk()
    l0 = (None, None, None) if score else (p.q0, p.k0_prefix, p.k0_block)
    F.focus_evict(dims, *l0, p.q1, p.k1_prefix, p.k1_block, p.cu_prefix,
                  p.hidden, p.decoded, p.budget, kept, cu, packed, ws, delta_out=delta,
                  i0_out=i0, i1_out=i1, stream=stream)
    status = F.focus_read_device_status(ws, stream)
    n = min(cap, int(cu[-1].item())) if constraints else cap
    out = dict(kept=kept[:n].cpu().numpy(), cu_seqlens=cu.cpu().numpy(),
               packed=packed[:n].view(torch.int16).cpu().numpy().view(np.uint16), status=status)
    if outputs:
        out.update(delta=delta.cpu().numpy().astype(np.float64), i0=i0.cpu().numpy().astype(np.float64),
                   i1=i1.cpu().numpy().astype(np.float64))
    return out


def assert_close_importance(got, want, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - want) - (ATOL + RTOL * np.abs(want))
    bad = np.argwhere(err > 0)
    assert bad.size == 0, (f"{what}: {len(bad)} entries out of tolerance, first at {bad[0].tolist()}: "
                           f"gpu {got[tuple(bad[0])]!r} oracle {want[tuple(bad[0])]!r}")


def assert_close_delta(got, want, what="delta"):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    ninf_w = np.isneginf(want)
    np.testing.assert_array_equal(np.isneginf(got), ninf_w, err_msg=f"{what}: -inf pattern")
    assert_close_importance(np.where(ninf_w, 0.0, got), np.where(ninf_w, 0.0, want), what)


def check_selection(kept_gpu, cu_gpu, pooled_oracle, decoded, budget, requests=None):
    """Checks the kept sets request by request.  Returns (n_exact, n_checked, n_tie_only)."""
    pooled_oracle = np.asarray(pooled_oracle, np.float64)
    decoded = np.asarray(decoded)
    budget = np.asarray(budget)
    R, B = decoded.shape
    reqs = range(R) if requests is None else requests
    exact = tie_only = 0
    for i, r in enumerate(reqs):
        orow = pooled_oracle[i]
        masked = np.flatnonzero(decoded[r] == 0)
        k = min(max(int(budget[r]), 0), masked.size)
        a, b = int(cu_gpu[r]), int(cu_gpu[r + 1])
        assert b - a == k, (r, b - a, k)
        got = kept_gpu[a:b]
        assert (np.diff(got) > 0).all(), (r, got)               # ascending, unique
        assert np.isin(got, masked).all(), (r, got)              # only masked positions
        order = np.lexsort((np.arange(B), -orow))
        want = np.sort(order[:k])
        if np.array_equal(got, want):
            exact += 1
            continue
        kth = orow[order[k - 1]]
        diff = np.setxor1d(got, want)
        assert np.all(np.abs(orow[diff] - kth) <= TIE_TOL), (
            f"request {r}: kept {got.tolist()} vs oracle {want.tolist()}; "
            f"differing positions {diff.tolist()} have pooled delta {orow[diff].tolist()}, k-th {kth}")
        tie_only += 1
    return exact, len(list(reqs)), tie_only


def check_structured(kept_gpu, cu_gpu, kept_oracle, cu_oracle, pooled_oracle, decoded, budget,
                     requests=None):
    """Retained sets under structural constraints.  A request whose candidate set is
    decided by a margin (oracle k-th and (k+1)-th pooled values more than 2e-3 apart)
    must match the oracle exactly; requests inside the tie band only need a valid,
    ascending, unique set.  Returns (n_exact, n_checked)."""
    pooled_oracle = np.asarray(pooled_oracle, np.float64)
    decoded = np.asarray(decoded)
    budget = np.asarray(budget)
    R, B = decoded.shape
    reqs = range(R) if requests is None else requests
    exact = 0
    for i, r in enumerate(reqs):
        got = kept_gpu[cu_gpu[r]:cu_gpu[r + 1]]
        assert (np.diff(got) > 0).all() and ((got >= 0) & (got < B)).all(), (r, got)
        orow = pooled_oracle[i]
        masked = np.flatnonzero(decoded[r] == 0)
        k = min(max(int(budget[r]), 0), masked.size)
        vals = np.sort(orow[masked])[::-1]
        decided = k == 0 or k == masked.size or vals[k - 1] - vals[k] > TIE_TOL
        if decided:
            want = kept_oracle[cu_oracle[i]:cu_oracle[i + 1]]
            np.testing.assert_array_equal(got, want, err_msg=f"retained set of request {r}")
            exact += 1
    return exact, len(list(reqs))


def check_packed(packed, kept, cu, hidden_bits, requests=None):
    """Each packed row is a bit-exact copy of hidden[r, kept]."""
    R = len(cu) - 1
    reqs = range(R) if requests is None else requests
    for r in reqs:
        a, b = int(cu[r]), int(cu[r + 1])
        if b > a:
            np.testing.assert_array_equal(packed[a:b], hidden_bits[r][kept[a:b]],
                                          err_msg=f"packed rows of request {r}")


def hidden_bits(p) -> np.ndarray:
    return p.hidden.detach().cpu().view(torch.int16).numpy().view(np.uint16)
