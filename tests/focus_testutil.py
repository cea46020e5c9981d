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

import math

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


def selection_margin(raw_row, pooled_row, decoded_row, k) -> float:
    """How far the oracle's selection of one request is from a different answer.

    The k-th largest masked pooled value v_k is the cut.  Pooled values are window
    maxima of the raw delta, so equal values at neighbouring positions are copies of
    one raw value; such exact ties are broken by position identically on both sides.
    Two raw positions that both hold exactly v_k (duplicated keys) are a tie of two
    separately computed values: the rule lets their order differ, so the margin is 0.
    Otherwise what can move the cut is another raw value close to v_k, pooled or hidden
    inside a window, so the margin is the distance from v_k to the nearest raw delta of
    the block that differs from it; infinite when k is 0 or every masked position is
    kept.
    """
    masked = np.flatnonzero(np.asarray(decoded_row) == 0)
    if k == 0 or k >= masked.size:
        return float("inf")
    vk = np.sort(np.asarray(pooled_row, np.float64)[masked])[::-1][k - 1]
    raw = np.asarray(raw_row, np.float64)
    if np.count_nonzero(raw == vk) >= 2:
        return 0.0
    other = raw[raw != vk]
    return float(np.min(np.abs(other - vk))) if other.size else float("inf")


def selection_margins(ref, decoded, budget) -> np.ndarray:
    """selection_margin of every request of an oracle result (budget clamped as the
    method clamps it)."""
    decoded = np.asarray(decoded)
    budget = np.asarray(budget)
    out = np.empty(decoded.shape[0])
    for r in range(decoded.shape[0]):
        k = min(max(int(budget[r]), 0), int((decoded[r] == 0).sum()))
        out[r] = selection_margin(ref["delta"][r], ref["pooled"][r], decoded[r], k)
    return out


def check_selection_all(kept_gpu, cu_gpu, ref, decoded, budget, orc):
    """Every request's kept set against the oracle's selection from its pooled delta
    (`ref["pooled"]`, raw delta `ref["delta"]`) under `budget`.  Requests decided by a
    margin (selection_margin > TIE_TOL) must match exactly; the others must satisfy
    the tie rule of check_selection.  Returns a report dict."""
    decoded = np.asarray(decoded)
    budget = np.asarray(budget)
    want, want_cu, _ = orc.select(ref["pooled"], decoded, budget)
    margins = selection_margins(ref, decoded, budget)
    exact, n, tie_only = check_selection(kept_gpu, cu_gpu, ref["pooled"], decoded, budget)
    decided = margins > TIE_TOL
    for r in np.flatnonzero(decided):
        np.testing.assert_array_equal(kept_gpu[cu_gpu[r]:cu_gpu[r + 1]],
                                      want[want_cu[r]:want_cu[r + 1]],
                                      err_msg=f"request {r} (margin {margins[r]:.3g})")
    return dict(requests=n, exact=exact, tie_band=int((~decided).sum()),
                exact_in_tie_band=int(exact - decided.sum()), decided=int(decided.sum()),
                min_margin=float(margins.min()) if n else float("inf"))


def check_structured(kept_gpu, cu_gpu, cand_gpu, cand_cu_gpu, ref, decoded, budget, constraints,
                     orc):
    """Retained sets under structural constraints, every request.

    cand_gpu / cand_cu_gpu are the GPU's plain top-k candidates on the same inputs
    (a constraints = 0 call: the same delta, so the same candidates); they must pass
    check_selection_all against the oracle's plain selection under `budget`.  The
    retained list must then be the constraint closure of those candidates
    (predecessors, masked positions left of the rightmost one), which the oracle's
    own structured selection computes from a 0/1 indicator of the candidates.
    Requests decided by a margin must also equal the oracle's retained list under
    `budget`.  Returns the candidates' report with the structured exact count added.
    """
    decoded = np.asarray(decoded)
    budget = np.asarray(budget)
    R, B = decoded.shape
    rep = check_selection_all(cand_gpu, cand_cu_gpu, ref, decoded, budget, orc)
    ind = np.where(decoded != 0, -np.inf, 0.0)
    counts = np.zeros(R, np.int32)
    for r in range(R):
        c = cand_gpu[cand_cu_gpu[r]:cand_cu_gpu[r + 1]]
        ind[r, c] = 1.0
        counts[r] = c.size
    closure, closure_cu, _ = orc.select_structured(ind, decoded, counts, constraints)
    np.testing.assert_array_equal(cu_gpu, closure_cu, err_msg="cu_seqlens vs the candidates' closure")
    want, want_cu, _ = orc.select_structured(ref["pooled"], decoded, budget, constraints)
    margins = selection_margins(ref, decoded, budget)
    exact = 0
    for r in range(R):
        got = kept_gpu[cu_gpu[r]:cu_gpu[r + 1]]
        np.testing.assert_array_equal(got, closure[closure_cu[r]:closure_cu[r + 1]],
                                      err_msg=f"request {r}: not the closure of its candidates")
        oref = want[want_cu[r]:want_cu[r + 1]]
        if margins[r] > TIE_TOL:
            np.testing.assert_array_equal(got, oref, err_msg=f"retained set of request {r}")
        exact += int(np.array_equal(got, oref))
    rep["structured_exact"] = exact
    return rep


def check_dynamic_budget(k_gpu, pooled, decoded, decode_avg, alpha=1.5, band=1e-2):
    """The GPU's dynamic budgets against the oracle's reading of Eq. 4,
    K = min(max(ceil(alpha * avg), n, 1), masked) with n the masked positions whose pooled
    delta exceeds their mean plus one population standard deviation.  n is bounded by
    the counts above the threshold moved by +-`band` (values that close to it may be
    counted either way), and ceil(alpha * avg) by its float32 and float64 values; every
    request's budget must lie within the bounds (equal to the oracle's where they
    meet).  Returns the number of requests whose bounds meet."""
    k_gpu = np.asarray(k_gpu)
    decoded = np.asarray(decoded)
    avg = np.asarray(decode_avg, np.float32)
    pinned = 0
    for r in range(decoded.shape[0]):
        m = decoded[r] == 0
        if not m.any():
            assert k_gpu[r] == 0, (r, k_gpu[r])
            pinned += 1
            continue
        D = np.asarray(pooled[r], np.float64)[m]
        thr = D.mean() + D.std()
        n_lo, n_hi = int((D > thr + band).sum()), int((D > thr - band).sum())
        a = max(float(avg[r]), 0.0)
        bases = (math.ceil(alpha * a), math.ceil(float(np.float32(alpha) * np.float32(a))))
        lo = min(max(min(bases), n_lo, 1), int(m.sum()))
        hi = min(max(max(bases), n_hi, 1), int(m.sum()))
        assert lo <= k_gpu[r] <= hi, (r, int(k_gpu[r]), lo, hi)
        pinned += int(lo == hi)
    return pinned


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
