"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Small cases are compared element by element; they span several 128-key tiles,
ragged tails, several 128-row query tiles, both head dims, GQA group sizes
1..16, odd block sizes and empty prefixes.  The five full-size workloads run in
the launch configuration the benchmark times and are compared on every request.
"""
import os

import numpy as np
import pytest
import torch

import synth
from focus_testutil import (assert_close_delta, assert_close_importance, check_dynamic_budget,
                            check_packed, check_selection_all, check_structured, hidden_bits,
                            run_evict)

pytestmark = pytest.mark.gpu

SMALL_CASES = {
    "tiny": (0, {}, False),
    "tiny_wide": (0, {}, True),
    "sdar_r6_ragged": (1, dict(R=6, prefix=("uniform", 0, 700)), False),
    "sdar_r6_ragged_wide": (1, dict(R=6, prefix=("uniform", 0, 700)), True),
    "block128_mt4": (3, dict(R=3, prefix=("uniform", 100, 400)), True),
    "ragged_g8_ties": (4, dict(R=8, prefix=("loguniform", 600)), True),
    "d64_g1_b20": (0, dict(R=5, B=20, Hq=4, Hkv=4, d=64, H=64, prefix=("uniform", 0, 300),
                          decoded=("uniform", 0.0, 0.8), lift=("frac", 0.2),
                          budget=("ceil", 0.3)), True),
    "g16_b16_mt2": (1, dict(R=3, B=16, Hq=32, Hkv=2, prefix=("uniform", 1, 260)), True),
    "b1_g1": (0, dict(R=4, B=1, Hq=8, Hkv=8, d=64, H=64, prefix=("uniform", 0, 200),
                      decoded=("exact", 0), lift=("count", 0), budget=("fixed", 1)), True),
    "no_prefix": (1, dict(R=4, prefix=("fixed", 0)), True),
    "g2_b32_neighbours": (0, dict(R=3, prefix=("uniform", 0, 300)), True),
    "d64_b128": (3, dict(R=2, d=64, Hq=8, Hkv=2, prefix=("uniform", 0, 300)), True),
}


@pytest.fixture(scope="module")
def orc():
    import oracle
    return oracle.default()


def _compare_full(p, out, ref, orc):
    assert out["status"] == 0, out["status"]
    assert_close_importance(out["i0"], ref["i0"], "I0")
    assert_close_importance(out["i1"], ref["i1"], "I1")
    assert_close_delta(out["delta"], ref["pooled"])
    np.testing.assert_array_equal(out["cu_seqlens"], ref["cu_seqlens"])
    check_selection_all(out["kept"], out["cu_seqlens"], ref, p.decoded.cpu().numpy(),
                        p.budget.cpu().numpy(), orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))


@pytest.mark.parametrize("case", sorted(SMALL_CASES))
def test_small_elementwise(case, orc):
    cfg, ov, wide = SMALL_CASES[case]
    p = synth.make_problem(cfg, seed=100 + sorted(SMALL_CASES).index(case), wide_logits=wide,
                           overrides=ov)
    ref = orc.evict(p)
    out = run_evict(p.to("cuda"))
    _compare_full(p, out, ref, orc)


def _report(parity_report, what, rep):
    line = (f"{what}: exact {rep['exact']}/{rep['requests']} kept sets "
            f"(decided by a margin > 2e-3: {rep['decided']}, all exact; tie band: "
            f"{rep['tie_band']}, of which exact {rep['exact_in_tie_band']}); "
            f"smallest margin {rep['min_margin']:.2e}")
    if "structured_exact" in rep:
        line += f"; retained lists equal to the oracle's: {rep['structured_exact']}"
    parity_report.append(line)


@pytest.mark.parametrize("wide", [False, True], ids=["literal", "wide"])
@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_full_config_every_request(cfg, wide, orc, parity_report):
    """The five workloads at full size, in the benchmark's launch configuration, against
    the oracle on every request: I0, I1 and the pooled delta element by element,
    cu_seqlens and packed rows exactly, and every kept set -- exactly where the oracle's
    selection is decided by a margin, else under the tie rule.  Run with the workloads'
    own value scale and with wide logits (Q, K ~ N(0, 1)), where margins are larger."""
    p = synth.make_problem(cfg, wide_logits=wide)
    out = run_evict(p.to("cuda"))
    ref = orc.evict(p)
    assert out["status"] == 0, out["status"]
    assert_close_importance(out["i0"], ref["i0"], "I0")
    assert_close_importance(out["i1"], ref["i1"], "I1")
    assert_close_delta(out["delta"], ref["pooled"])
    np.testing.assert_array_equal(out["cu_seqlens"], ref["cu_seqlens"])
    rep = check_selection_all(out["kept"], out["cu_seqlens"], ref, p.decoded.numpy(),
                              p.budget.numpy(), orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))
    _report(parity_report, f"{synth.CONFIGS[cfg].name} ({'wide' if wide else 'literal'} logits)",
            rep)


def _row_lse_on_device(g):
    """Layer-0 row log-sum-exps [R, B, Hq] of a problem on the GPU, in float64 with torch
    (setup: the input an engine's layer-0 attention forward hands over)."""
    G = g.Hq // g.Hkv
    cu = g.cu_prefix.cpu().numpy()
    out = torch.empty(g.R, g.B, g.Hq, dtype=torch.float64, device=g.q0.device)
    for r in range(g.R):
        keys = torch.cat([g.k0_prefix[int(cu[r]):int(cu[r + 1])], g.k0_block[r]], 0).double()
        q = g.q0[r].double()  # [B, Hq, d]
        for kv in range(g.Hkv):
            qs = q[:, kv * G:(kv + 1) * G].reshape(-1, g.d)
            out[r, :, kv * G:(kv + 1) * G] = torch.logsumexp(
                g.scale * (qs @ keys[:, kv].T), dim=-1).view(g.B, G)
    return out


@pytest.mark.parametrize("variant", ["paged64", "lse0", "score1", "dynamic"])
def test_variants_full_metric_shape_every_request(variant, orc, parity_report):
    """The options of the fused step at the metric shape (256 requests), every request
    against the oracle run with the same option: paged prefix keys (64-token pages), the
    layer-0 row log-sum-exps given, ranking by I1 alone, the dynamic budget."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(2)
    g = p.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    budget = p.budget.numpy()
    if variant == "score1":
        out = run_evict(g, score=1)
        ref = orc.evict(p, score=1)
    elif variant == "dynamic":
        avg = np.random.default_rng(12).uniform(0.0, 0.2 * p.B, size=p.R).astype(np.float32)
        out = _evict_dynamic(p, g, avg, 0)
        ref = orc.evict(p, decode_avg=avg.astype(np.float64))
        check_dynamic_budget(out["budget"], ref["pooled"], p.decoded.numpy(), avg)
        budget = out["budget"]
    else:
        ws = F.Workspace(dims)
        cap = F.plan_capacity(p.decoded, p.budget)
        kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
        packed = torch.zeros(cap, p.H, dtype=torch.bfloat16, device="cuda")
        delta = torch.empty(p.R, p.B, device="cuda")
        if variant == "paged64":
            pg = synth.to_paged(g, 64, seed=2)
            F.focus_evict_paged(dims, g.q0, pg.k0_pages, g.k0_block, g.q1, pg.k1_pages, g.k1_block,
                                pg.page_table, pg.prefix_len, g.hidden, g.decoded, g.budget, kept,
                                cu, packed, ws, delta_out=delta)
            ref = orc.evict(p)
        else:
            lse = _row_lse_on_device(g).float()  # both sides take the same float32 values
            F.focus_evict_with_lse0(dims, lse, g.q0, g.k0_block, g.q1, g.k1_prefix, g.k1_block,
                                    g.cu_prefix, g.hidden, g.decoded, g.budget, kept, cu, packed,
                                    ws, delta_out=delta)
            ref = orc.evict(p, lse0=lse.double().cpu().numpy())
        st = F.focus_read_device_status(ws)
        out = dict(status=st, kept=kept.cpu().numpy(), cu_seqlens=cu.cpu().numpy(),
                   packed=packed.view(torch.int16).cpu().numpy().view(np.uint16),
                   delta=delta.cpu().numpy().astype(np.float64))
    assert out["status"] == 0
    assert_close_delta(out["delta"], ref["pooled"])
    rep = check_selection_all(out["kept"], out["cu_seqlens"], ref, p.decoded.numpy(), budget, orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))
    _report(parity_report, f"sdar8b_r256_b32 ({variant})", rep)


@pytest.mark.parametrize("cfg,ov", [
    (4, dict(R=24, prefix=("loguniform", 900), tie_frac=0.5)),
    (4, dict(R=24, B=48, prefix=("loguniform", 900), tie_frac=1.0)),
    (3, dict(R=16, prefix=("uniform", 100, 600), tie_frac=1.0)),
], ids=["b64", "b48", "b128"])
def test_duplicate_keys_give_equal_columns(cfg, ov):
    """A duplicated block key (same K rows at both layers) gets bit-equal I columns when
    both copies are weighted by the same softmax warpgroup: always for B <= 64 (one
    warpgroup weights the whole block), and within each 64-column half of a larger block.
    Copies in different halves (B > 64) are weighted against each half's own reference max
    and agree to rounding (a relative 1e-5 here); the tie rule covers them."""
    p = synth.make_problem(cfg, seed=77, overrides=ov)
    assert p.tie_pairs
    out = run_evict(p.to("cuda"))
    assert out["status"] == 0
    same = [(r, a, b) for (r, a, b) in p.tie_pairs if p.B <= 64 or (a < 64) == (b < 64)]
    across = [t for t in p.tie_pairs if t not in same]
    assert same and (p.B <= 64 or across)
    for (r, a, b) in same:
        assert out["i0"][r, a] == out["i0"][r, b], (r, a, b)
        assert out["i1"][r, a] == out["i1"][r, b], (r, a, b)
    for (r, a, b) in across:
        for key in ("i0", "i1"):
            np.testing.assert_allclose(out[key][r, a], out[key][r, b], rtol=1e-5, atol=0)


def test_deterministic():
    p = synth.make_problem(1, overrides=dict(R=8), wide_logits=True).to("cuda")
    a, b = run_evict(p), run_evict(p)
    for k in ("i0", "i1", "delta", "kept", "cu_seqlens", "packed"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_deterministic_full_ragged_workload():
    """The ragged workload at full size (4,096 work items over the persistent grid, most of
    them short): two calls give identical bits."""
    p = synth.make_problem(4, wide_logits=True).to("cuda")
    a, b = run_evict(p), run_evict(p)
    for k in ("i0", "i1", "delta", "kept", "cu_seqlens", "packed"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_results_do_not_depend_on_the_schedule():
    """A request's outputs are the same bits whichever schedule processed it: the metric
    workload (4,096 attention items, claimed dynamically by the CTAs) against 32, 48 and 73 of
    its requests run alone (512, 768 and 1,168 items: the static order) and 74 of them (1,184
    items, exactly four per CTA: dynamic again), which also changes which CTA takes which item
    and when."""
    p = synth.make_problem(2, wide_logits=True)
    full = run_evict(p.to("cuda"))
    for req in (list(range(0, 256, 8)), list(range(3, 256, 5))[:48], list(range(73)),
                list(range(100, 174))):
        sub = run_evict(p.subset(req).to("cuda"))
        for key in ("i0", "i1", "delta"):
            np.testing.assert_array_equal(full[key][req], sub[key], err_msg=key)
        cu_f, cu_s = full["cu_seqlens"], sub["cu_seqlens"]
        for t, r in enumerate(req):
            np.testing.assert_array_equal(full["kept"][cu_f[r]:cu_f[r + 1]],
                                          sub["kept"][cu_s[t]:cu_s[t + 1]], err_msg=str(r))
            np.testing.assert_array_equal(full["packed"][cu_f[r]:cu_f[r + 1]],
                                          sub["packed"][cu_s[t]:cu_s[t + 1]], err_msg=str(r))


def test_consecutive_denoising_steps_vs_oracle(orc):
    """One workspace and one set of output buffers across five denoising steps, as an
    engine would use them: after each step a few of the kept (still-masked) tokens become
    decoded and the budgets shrink with the masked counts; every step matches the oracle."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, seed=77, wide_logits=True,
                           overrides=dict(R=12, prefix=("uniform", 0, 900)))
    g = p.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    ws = F.Workspace(dims)
    kept = torch.empty(p.R * p.B, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.empty(p.R * p.B, p.H, dtype=torch.bfloat16, device="cuda")
    delta = torch.empty(p.R, p.B, device="cuda")
    rng = np.random.default_rng(5)
    for step in range(5):
        dec = p.decoded.numpy()
        masked = (dec == 0).sum(1)
        p.budget = torch.from_numpy(np.maximum(1, np.ceil(0.3 * masked)).astype(np.int32))
        p.budget[masked == 0] = 0
        g.decoded, g.budget = p.decoded.cuda(), p.budget.cuda()
        F.focus_evict(dims, g.q0, g.k0_prefix, g.k0_block, g.q1, g.k1_prefix, g.k1_block,
                      g.cu_prefix, g.hidden, g.decoded, g.budget, kept, cu, packed, ws,
                      delta_out=delta)
        assert F.focus_read_device_status(ws) == 0, step
        ref = orc.evict(p)
        cu_h = cu.cpu().numpy()
        n = int(cu_h[-1])
        np.testing.assert_array_equal(cu_h, ref["cu_seqlens"])
        assert_close_delta(delta.cpu().numpy(), ref["pooled"])
        kept_h = kept[:n].cpu().numpy()
        check_selection_all(kept_h, cu_h, ref, p.decoded.numpy(), p.budget.numpy(), orc)
        check_packed(packed[:n].view(torch.int16).cpu().numpy().view(np.uint16), kept_h, cu_h,
                     hidden_bits(p))
        # the next step: up to two kept tokens per request are decoded
        new = p.decoded.clone()
        for r in range(p.R):
            seg = kept_h[cu_h[r]:cu_h[r + 1]]
            if seg.size:
                new[r, rng.choice(seg, size=min(2, seg.size), replace=False)] = 1
        p.decoded = new


def test_standalone_chain_matches_fused():
    """attn_stats x2 -> importance_delta -> topk_select -> compact reproduces
    focus_evict bit for bit (same reduction order everywhere)."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(4, overrides=dict(R=16, prefix=("loguniform", 1500)),
                           wide_logits=True).to("cuda")
    fused = run_evict(p)
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    ws = F.Workspace(dims)
    i0 = torch.empty(p.R, p.B, device="cuda")
    i1 = torch.empty_like(i0)
    F.focus_attn_stats(dims, p.q0, p.k0_prefix, p.cu_prefix, p.k0_block, i0, ws)
    F.focus_attn_stats(dims, p.q1, p.k1_prefix, p.cu_prefix, p.k1_block, i1, ws)
    delta = torch.empty_like(i0)
    raw = torch.empty_like(i0)
    F.focus_importance_delta(dims, i0, i1, p.decoded, delta, raw)
    cap = F.plan_capacity(p.decoded, p.budget)
    kept = torch.empty(cap, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    F.focus_topk_select(dims, delta, p.decoded, p.budget, kept, cu, ws)
    packed = torch.empty(cap, p.H, dtype=torch.bfloat16, device="cuda")
    F.focus_compact(dims, p.hidden, kept, cu, packed, ws)
    assert F.focus_read_device_status(ws) == 0
    np.testing.assert_array_equal(i0.cpu().numpy(), fused["i0"].astype(np.float32))
    np.testing.assert_array_equal(i1.cpu().numpy(), fused["i1"].astype(np.float32))
    np.testing.assert_array_equal(delta.cpu().numpy(), fused["delta"].astype(np.float32))
    np.testing.assert_array_equal((i1 - i0).cpu().numpy(), raw.cpu().numpy())
    np.testing.assert_array_equal(kept.cpu().numpy(), fused["kept"])
    np.testing.assert_array_equal(cu.cpu().numpy(), fused["cu_seqlens"])
    np.testing.assert_array_equal(packed.view(torch.int16).cpu().numpy().view(np.uint16),
                                  fused["packed"])


def test_standalone_steps_vs_oracle(orc):
    """Each stand-alone entry point against the oracle's step of the same name."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, overrides=dict(R=5, prefix=("uniform", 0, 500)), wide_logits=True)
    g = p.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    ws = F.Workspace(dims)
    i0 = torch.empty(p.R, p.B, device="cuda")
    F.focus_attn_stats(dims, g.q0, g.k0_prefix, g.cu_prefix, g.k0_block, i0, ws)
    want = orc.importance(p.q0, p.k0_prefix, p.cu_prefix, p.k0_block, Hq=p.Hq, Hkv=p.Hkv,
                          scale=p.scale)
    assert_close_importance(i0.cpu().numpy(), want, "attn_stats")
    # delta / pool / mask on exact float32 inputs: exact
    rng = np.random.default_rng(3)
    a = rng.normal(size=(p.R, p.B)).astype(np.float32)
    b = rng.normal(size=(p.R, p.B)).astype(np.float32)
    delta = torch.empty(p.R, p.B, device="cuda")
    F.focus_importance_delta(dims, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(),
                             g.decoded, delta)
    _, pooled = orc.delta_pool_mask(a.astype(np.float64), b.astype(np.float64), p.decoded)
    np.testing.assert_array_equal(delta.cpu().numpy(),
                                  pooled.astype(np.float32))  # b - a is exact in fp64 -> fp32 rounding once
    # select on a coarse grid (many exact ties): bit-exact
    vals = (rng.integers(-3, 4, size=(p.R, p.B)) * 0.5).astype(np.float32)
    vals[p.decoded.numpy() != 0] = -np.inf
    cap = F.plan_capacity(p.decoded, p.budget)
    kept = torch.empty(cap, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    F.focus_topk_select(dims, torch.from_numpy(vals).cuda(), g.decoded, g.budget, kept, cu, ws)
    okept, ocu, _ = orc.select(vals.astype(np.float64), p.decoded, p.budget)
    np.testing.assert_array_equal(kept.cpu().numpy(), okept)
    np.testing.assert_array_equal(cu.cpu().numpy(), ocu)
    packed = torch.empty(cap, p.H, dtype=torch.bfloat16, device="cuda")
    F.focus_compact(dims, g.hidden, kept, cu, packed, ws)
    want_packed = orc.compact(p.hidden, okept, ocu)
    np.testing.assert_array_equal(packed.view(torch.int16).cpu().numpy().view(np.uint16), want_packed)
    assert F.focus_read_device_status(ws) == 0


def test_signed_zero_ties_vs_oracle(orc):
    """-0.0 and +0.0 tie (the lower position wins whatever the sign), in the selection
    call and after the delta step, whose I1 - I0 and MaxPool1D produce zeros of both
    signs; kept sets bit-exact against the oracle."""
    import attention_delta_token_b200 as F
    rng = np.random.default_rng(41)
    R, B = 24, 32
    dims = F.make_dims(R, B, 32, 8, 128, 4096)
    ws = F.Workspace(dims)
    dec = (rng.random((R, B)) < 0.25).astype(np.uint8)
    budget = rng.integers(1, B, size=R).astype(np.int32)
    dec_g = torch.from_numpy(dec).cuda()
    bud_g = torch.from_numpy(budget).cuda()
    cap = F.plan_capacity(torch.from_numpy(dec), torch.from_numpy(budget))
    # scores drawn from {-0.5, -0.0, +0.0, +0.5}: most cuts fall inside a run of zeros
    vals = rng.choice(np.array([-0.5, -0.0, 0.0, 0.5], np.float32), size=(R, B))
    vals[dec != 0] = -np.inf
    assert (np.signbit(vals) & (vals == 0)).any() and (~np.signbit(vals) & (vals == 0)).any()
    kept = torch.empty(cap, dtype=torch.int32, device="cuda")
    cu = torch.empty(R + 1, dtype=torch.int32, device="cuda")
    F.focus_topk_select(dims, torch.from_numpy(vals).cuda(), dec_g, bud_g, kept, cu, ws)
    okept, ocu, _ = orc.select(vals.astype(np.float64), dec, budget)
    np.testing.assert_array_equal(cu.cpu().numpy(), ocu)
    np.testing.assert_array_equal(kept.cpu().numpy(), okept)
    # through the delta step: I1 - I0 of equal values is +0.0, of (-0.0) - (+0.0) is -0.0
    i0 = rng.choice(np.array([0.0, -0.0, 0.25], np.float32), size=(R, B))
    i1 = rng.choice(np.array([0.0, -0.0, 0.25], np.float32), size=(R, B))
    delta = torch.empty(R, B, device="cuda")
    F.focus_importance_delta(dims, torch.from_numpy(i0).cuda(), torch.from_numpy(i1).cuda(),
                             dec_g, delta)
    _, pooled = orc.delta_pool_mask(i0.astype(np.float64), i1.astype(np.float64), dec)
    np.testing.assert_array_equal(delta.cpu().numpy(), pooled.astype(np.float32))  # -0 == +0
    F.focus_topk_select(dims, delta, dec_g, bud_g, kept, cu, ws)
    okept, ocu, _ = orc.select(pooled, dec, budget)
    np.testing.assert_array_equal(cu.cpu().numpy(), ocu)
    np.testing.assert_array_equal(kept.cpu().numpy(), okept)
    assert F.focus_read_device_status(ws) == 0


def test_zero_budget_and_all_decoded(orc):
    p = synth.make_problem(1, overrides=dict(R=4, prefix=("uniform", 0, 300)))
    p.budget = torch.tensor([0, -5, 3, 40], dtype=torch.int32)
    dec = p.decoded.clone()
    dec[2] = 1  # request 2 fully decoded: nothing to keep
    p.decoded = dec
    ref = orc.evict(p)
    out = run_evict(p.to("cuda"))
    _compare_full(p, out, ref, orc)
    assert out["cu_seqlens"][1] == 0 and out["cu_seqlens"][2] == 0


def test_nothing_kept_anywhere(orc):
    """Every budget zero: the packed batch is empty (capacity 0), cu_seqlens is all zeros, the
    importance is still computed and matches the oracle."""
    p = synth.make_problem(1, overrides=dict(R=5, prefix=("uniform", 0, 300)))
    p.budget = torch.zeros(p.R, dtype=torch.int32)
    out = run_evict(p.to("cuda"))
    assert out["status"] == 0
    np.testing.assert_array_equal(out["cu_seqlens"], np.zeros(p.R + 1, np.int32))
    assert out["kept"].size == 0 and out["packed"].shape[0] == 0
    ref = orc.evict(p)
    assert_close_importance(out["i1"], ref["i1"], "I1")
    assert_close_delta(out["delta"], ref["pooled"])


def test_capacity_overflow_reports_and_stays_in_bounds():
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, overrides=dict(R=4, prefix=("uniform", 0, 300))).to("cuda")
    need = F.plan_capacity(p.decoded, p.budget)
    assert need >= 3
    out = run_evict(p, capacity=need - 2)
    assert out["status"] == 3  # FOCUS_ERR_CAPACITY
    assert out["cu_seqlens"][-1] == need


def test_malformed_cu_prefix_reports():
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, overrides=dict(R=3, prefix=("uniform", 10, 100))).to("cuda")
    bad = p.cu_prefix.clone()
    bad[2] = bad[3] + 5  # beyond total_prefix and decreasing
    p.cu_prefix = bad
    out = run_evict(p)
    assert out["status"] == 6  # FOCUS_ERR_DEVICE_CHECK


@pytest.mark.parametrize("factor", [0.0, 0.5, 2.0])
def test_softmax_scale_other_than_default(factor, orc):
    """softmax_scale is an argument: zero (every row's softmax uniform over its keys), half
    and twice 1/sqrt(d), against the oracle with the same scale."""
    import dataclasses
    p = synth.make_problem(1, seed=61, wide_logits=True, overrides=dict(R=5, prefix=("uniform", 0, 500)))
    p = dataclasses.replace(p, scale=p.scale * factor)
    ref = orc.evict(p)
    out = run_evict(p.to("cuda"))
    _compare_full(p, out, ref, orc)
    if factor == 0.0:  # uniform rows: I_j = B Hq / N_r for every block column
        N = p.prefix_len + p.B
        np.testing.assert_allclose(out["i1"], (p.B * p.Hq / N)[:, None] * np.ones((1, p.B)),
                                   rtol=1e-5)


def test_non_finite_inputs_are_reported_and_contained(orc):
    """A NaN in one request's layer-1 queries (out of contract) makes that request's
    importance non-finite: the call reports FOCUS_ERR_DEVICE_CHECK, cu_seqlens keeps its
    count-based values, and every other request still matches the oracle."""
    p = synth.make_problem(1, seed=55, wide_logits=True, overrides=dict(R=6, prefix=("uniform", 100, 600)))
    bad = 2
    q1 = p.q1.clone()
    q1[bad, 0, 0, 0] = float("nan")
    p.q1 = q1
    out = run_evict(p.to("cuda"))
    assert out["status"] == 6  # FOCUS_ERR_DEVICE_CHECK
    good = [r for r in range(p.R) if r != bad]
    sub = p.subset(good)
    ref = orc.evict(sub)
    _, cu_all, _ = orc.select(np.zeros((p.R, p.B)), p.decoded, p.budget)
    np.testing.assert_array_equal(out["cu_seqlens"], cu_all)
    assert_close_importance(out["i0"], orc.evict(p)["i0"], "I0 (layer 0 has no NaN)")
    assert_close_delta(out["delta"][good], ref["pooled"])
    kept, cu, packed = [], [0], []
    for r in good:
        a, b = int(out["cu_seqlens"][r]), int(out["cu_seqlens"][r + 1])
        kept.append(out["kept"][a:b])
        packed.append(out["packed"][a:b])
        cu.append(cu[-1] + (b - a))
    check_selection_all(np.concatenate(kept), np.array(cu), ref, sub.decoded.numpy(),
                        sub.budget.numpy(), orc)
    check_packed(np.concatenate(packed), np.concatenate(kept), np.array(cu), hidden_bits(sub))


def test_bounded_wait_times_out_and_reports():
    """A kernel waiting on a barrier that never completes gives up after its limit,
    reports FOCUS_DEV_TIMEOUT in the status word, and leaves the context usable."""
    import attention_delta_token_b200 as F
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(1, dtype=torch.int64, device="cuda")
    limit = 50_000_000  # 50 ms
    F.focus_selftest_wait_timeout(status, elapsed, limit)
    torch.cuda.synchronize()
    assert int(status.item()) == 4  # FOCUS_DEV_TIMEOUT, and the barrier never completed
    assert limit <= int(elapsed.item()) < limit + 200_000_000
    # the context still runs the eviction step correctly
    p = synth.make_problem(0).to("cuda")
    out = run_evict(p)
    assert out["status"] == 0


STRUCTURED_CASES = {
    "sdar_r8_wide": (1, dict(R=8, prefix=("uniform", 0, 600)), True),
    "ragged_r10_ties": (4, dict(R=10, prefix=("loguniform", 500)), True),
    "block128_r3": (3, dict(R=3, prefix=("uniform", 100, 300)), True),
    "tiny": (0, {}, False),
}


@pytest.mark.parametrize("constraints", [1, 2, 3])
@pytest.mark.parametrize("case", sorted(STRUCTURED_CASES))
def test_structural_constraints_vs_oracle(case, constraints, orc):
    """Retained sets with the structural constraints ("What carries the argument"):
    candidates plus predecessors and/or masked tokens left of the rightmost one.  Every
    request's list is the closure of the GPU's own top-k candidates (checked against the
    oracle's selection), and equals the oracle's list where a margin decides it."""
    cfg, ov, wide = STRUCTURED_CASES[case]
    p = synth.make_problem(cfg, seed=300 + constraints, wide_logits=wide, overrides=ov)
    ref = orc.evict(p, constraints=constraints)
    g = p.to("cuda")
    out = run_evict(g, constraints=constraints)
    cand = run_evict(g)
    assert out["status"] == 0 and cand["status"] == 0
    np.testing.assert_array_equal(out["delta"], cand["delta"])  # same delta, same candidates
    assert_close_importance(out["i0"], ref["i0"], "I0")
    assert_close_importance(out["i1"], ref["i1"], "I1")
    assert_close_delta(out["delta"], ref["pooled"])
    check_structured(out["kept"], out["cu_seqlens"], cand["kept"], cand["cu_seqlens"], ref,
                     p.decoded.numpy(), p.budget.numpy(), constraints, orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))


def test_structural_topk_select_exact(orc):
    """Stand-alone focus_topk_select with constraints on exact (grid) values: the
    retained lists and cu_seqlens equal the oracle's bit for bit, ties included."""
    import attention_delta_token_b200 as F
    rng = np.random.default_rng(21)
    p = synth.make_problem(4, overrides=dict(R=40, prefix=("fixed", 0)))
    vals = (rng.integers(-3, 4, size=(p.R, p.B)) * 0.5).astype(np.float32)
    vals[p.decoded.numpy() != 0] = -np.inf
    for c in (1, 2, 3):
        dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window, c)
        ws = F.Workspace(dims)
        cap = F.plan_capacity(p.decoded, p.budget, c)
        kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
        F.focus_topk_select(dims, torch.from_numpy(vals).cuda(), p.decoded.cuda(),
                            p.budget.cuda(), kept, cu, ws)
        assert F.focus_read_device_status(ws) == 0
        okept, ocu, _ = orc.select_structured(vals.astype(np.float64), p.decoded, p.budget, c)
        np.testing.assert_array_equal(cu.cpu().numpy(), ocu)
        np.testing.assert_array_equal(kept[:int(ocu[-1])].cpu().numpy(), okept)


@pytest.mark.parametrize("cfg,wide", [(4, True), (2, False)], ids=["ragged_wide", "metric_literal"])
def test_structural_full_config_every_request(cfg, wide, orc, parity_report):
    """Both constraints on a full-size workload in the benchmark's launch configuration:
    every request's retained list is the closure of the GPU's top-k candidates, which
    match the oracle's selection (exactly where a margin decides it)."""
    p = synth.make_problem(cfg, wide_logits=wide)
    g = p.to("cuda")
    out = run_evict(g, constraints=3)
    cand = run_evict(g)
    assert out["status"] == 0 and cand["status"] == 0
    np.testing.assert_array_equal(out["delta"], cand["delta"])
    ref = orc.evict(p)
    assert_close_delta(out["delta"], ref["pooled"])
    rep = check_structured(out["kept"], out["cu_seqlens"], cand["kept"], cand["cu_seqlens"], ref,
                           p.decoded.numpy(), p.budget.numpy(), 3, orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))
    _report(parity_report, f"{synth.CONFIGS[cfg].name} ({'wide' if wide else 'literal'} logits), "
            "constraints 3", rep)


@pytest.mark.parametrize("case", ["sdar_r8_wide", "ragged_r10_ties", "tiny"])
def test_layer1_score_vs_oracle(case, orc):
    """Ranking by the layer-1 importance alone (the Figure 13 ablation): layer 0 is
    neither passed nor computed; the pooled score is MaxPool1D(I1)."""
    cfg, ov, wide = STRUCTURED_CASES[case]
    p = synth.make_problem(cfg, seed=400, wide_logits=wide, overrides=ov)
    ref = orc.evict(p, score=1)
    out = run_evict(p.to("cuda"), score=1)
    assert out["status"] == 0
    assert np.isnan(out["i0"]).all()  # left untouched
    assert_close_importance(out["i1"], ref["i1"], "I1")
    assert_close_delta(out["delta"], ref["pooled"])
    check_selection_all(out["kept"], out["cu_seqlens"], ref, p.decoded.numpy(),
                        p.budget.numpy(), orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))


def _row_lse(p, device="cpu"):
    """Layer-0 row log-sum-exps over each row's prefix and block keys (torch float64):
    the input an engine's layer-0 attention forward would hand over."""
    G = p.Hq // p.Hkv
    cu = p.cu_prefix.cpu().numpy()
    out = torch.zeros(p.R, p.B, p.Hq, dtype=torch.float64)
    for r in range(p.R):
        keys = torch.cat([p.k0_prefix[int(cu[r]):int(cu[r + 1])].cpu(), p.k0_block[r].cpu()], 0)
        for h in range(p.Hq):
            s = p.scale * p.q0[r, :, h].cpu().double() @ keys[:, h // G].double().T
            out[r, :, h] = torch.logsumexp(s, dim=-1)
    return out


@pytest.mark.parametrize("case", ["sdar_r8_wide", "ragged_r10_ties", "block128_r3", "tiny"])
def test_evict_with_lse0_vs_oracle(case, orc):
    """Layer 0 from the engine's row log-sum-exps: only Q0 and the block keys are read;
    the result matches the oracle's importance-from-LSE and, the LSE being the true one,
    the full computation."""
    import attention_delta_token_b200 as F
    cfg, ov, wide = STRUCTURED_CASES[case]
    p = synth.make_problem(cfg, seed=500, wide_logits=wide, overrides=ov)
    lse = _row_lse(p).float()
    g = p.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    ws = F.Workspace(dims)
    cap = F.plan_capacity(p.decoded, p.budget)
    kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.zeros(cap, p.H, dtype=torch.bfloat16, device="cuda")
    delta = torch.empty(p.R, p.B, device="cuda")
    i0 = torch.empty_like(delta)
    i1 = torch.empty_like(delta)
    F.focus_evict_with_lse0(dims, lse.cuda(), g.q0, g.k0_block, g.q1, g.k1_prefix, g.k1_block,
                            g.cu_prefix, g.hidden, g.decoded, g.budget, kept, cu, packed, ws,
                            delta_out=delta, i0_out=i0, i1_out=i1)
    assert F.focus_read_device_status(ws) == 0
    ref = orc.evict(p, lse0=lse.double().numpy())
    full = orc.evict(p)
    assert_close_importance(i0.cpu().numpy(), ref["i0"], "I0 from lse")
    assert_close_importance(i0.cpu().numpy(), full["i0"], "I0 vs full")
    assert_close_importance(i1.cpu().numpy(), ref["i1"], "I1")
    assert_close_delta(delta.cpu().numpy(), ref["pooled"])
    np.testing.assert_array_equal(cu.cpu().numpy(), ref["cu_seqlens"])
    check_selection_all(kept.cpu().numpy(), cu.cpu().numpy(), ref, p.decoded.numpy(),
                        p.budget.numpy(), orc)
    check_packed(packed.view(torch.int16).cpu().numpy().view(np.uint16), kept.cpu().numpy(),
                 cu.cpu().numpy(), hidden_bits(p))


@pytest.mark.parametrize("page_size", [8, 16, 64, 128, 256])
def test_evict_paged_vs_oracle(page_size, orc):
    """Prefix keys read in place from a paged pool (shuffled pages, junk after each
    prefix's end) give the oracle's results, for pages shorter and longer than a
    128-key tile."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(4, seed=600 + page_size, wide_logits=True,
                           overrides=dict(R=10, prefix=("loguniform", 700)))
    pg = synth.to_paged(p, page_size, seed=page_size)
    ref = orc.evict(p)
    paged_ref = orc.importance_paged(p.q0, pg.k0_pages, pg.page_table, pg.prefix_len,
                                     p.k0_block, Hq=p.Hq, Hkv=p.Hkv, scale=p.scale)
    np.testing.assert_allclose(paged_ref, ref["i0"], rtol=1e-12)
    g, gp = p.to("cuda"), pg.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    ws = F.Workspace(dims)
    cap = F.plan_capacity(p.decoded, p.budget)
    kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.zeros(cap, p.H, dtype=torch.bfloat16, device="cuda")
    delta = torch.empty(p.R, p.B, device="cuda")
    i0, i1 = torch.empty_like(delta), torch.empty_like(delta)
    F.focus_evict_paged(dims, g.q0, gp.k0_pages, g.k0_block, g.q1, gp.k1_pages, g.k1_block,
                        gp.page_table, gp.prefix_len, g.hidden, g.decoded, g.budget, kept, cu,
                        packed, ws, delta_out=delta, i0_out=i0, i1_out=i1)
    assert F.focus_read_device_status(ws) == 0
    assert_close_importance(i0.cpu().numpy(), ref["i0"], "I0")
    assert_close_importance(i1.cpu().numpy(), ref["i1"], "I1")
    assert_close_delta(delta.cpu().numpy(), ref["pooled"])
    np.testing.assert_array_equal(cu.cpu().numpy(), ref["cu_seqlens"])
    check_selection_all(kept.cpu().numpy(), cu.cpu().numpy(), ref, p.decoded.numpy(),
                        p.budget.numpy(), orc)
    check_packed(packed.view(torch.int16).cpu().numpy().view(np.uint16), kept.cpu().numpy(),
                 cu.cpu().numpy(), hidden_bits(p))


def test_evict_paged_matches_packed_bitwise():
    """With pages of >= 128 keys each tile is one box, so the paged call reproduces the
    packed call bit for bit; with 64-key pages too (same keys, same order)."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, seed=7, wide_logits=True, overrides=dict(R=12))
    want = run_evict(p.to("cuda"))
    for page_size in (64, 128, 512):
        pg = synth.to_paged(p, page_size, seed=1).to("cuda")
        g = p.to("cuda")
        dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
        ws = F.Workspace(dims)
        cap = F.plan_capacity(p.decoded, p.budget)
        kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
        packed = torch.zeros(cap, p.H, dtype=torch.bfloat16, device="cuda")
        i0 = torch.empty(p.R, p.B, device="cuda")
        i1 = torch.empty_like(i0)
        F.focus_evict_paged(dims, g.q0, pg.k0_pages, g.k0_block, g.q1, pg.k1_pages, g.k1_block,
                            pg.page_table, pg.prefix_len, g.hidden, g.decoded, g.budget, kept, cu,
                            packed, ws, i0_out=i0, i1_out=i1)
        assert F.focus_read_device_status(ws) == 0
        np.testing.assert_array_equal(i0.cpu().numpy(), want["i0"].astype(np.float32))
        np.testing.assert_array_equal(i1.cpu().numpy(), want["i1"].astype(np.float32))
        np.testing.assert_array_equal(kept.cpu().numpy(), want["kept"])


def _evict_dynamic(p, g, avg, constraints, **extra):
    """focus_evict_ex with the dynamic budget on the GPU problem `g`; returns numpy kept,
    cu_seqlens, budgets, pooled delta and packed rows.  `extra` passes further options
    (lse0, page pools) through to the call."""
    import attention_delta_token_b200 as F
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window, constraints)
    ws = F.Workspace(dims)
    cap = F.plan_capacity(p.decoded, None, constraints, dynamic=True)
    kept = torch.full((max(cap, 1),), -1, dtype=torch.int32, device="cuda")[:cap]
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.zeros(max(cap, 1), p.H, dtype=torch.bfloat16, device="cuda")[:cap]
    delta = torch.empty(p.R, p.B, device="cuda")
    kout = torch.full((p.R,), -1, dtype=torch.int32, device="cuda")
    args = dict(q0=g.q0, k0_prefix=g.k0_prefix, k0_block=g.k0_block, q1=g.q1,
                k1_prefix=g.k1_prefix, k1_block=g.k1_block, cu_prefix=g.cu_prefix)
    args.update(extra)
    F.focus_evict_ex(dims, **args, hidden=g.hidden, decoded=g.decoded,
                     decode_avg=torch.from_numpy(np.asarray(avg, np.float32)).cuda(),
                     budget_alpha=1.5, budget_out=kout, kept_idx=kept, cu_seqlens=cu,
                     packed=packed, ws=ws, delta_out=delta)
    status = F.focus_read_device_status(ws)
    cu_h = cu.cpu().numpy()
    n = int(cu_h[-1])
    return dict(status=status, kept=kept[:n].cpu().numpy(), cu_seqlens=cu_h,
                budget=kout.cpu().numpy(), delta=delta.cpu().numpy().astype(np.float64),
                packed=packed[:n].view(torch.int16).cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("case,constraints", [("sdar_r8_wide", 0), ("ragged_r10_ties", 0),
                                              ("block128_r3", 0), ("sdar_r8_wide", 3),
                                              ("ragged_r10_ties", 3)])
def test_dynamic_budget_vs_oracle(case, constraints, orc):
    """Dynamic budget (Eq. 4 as read): every request's K_r lies within the oracle's bounds
    (equal to the oracle's K_r wherever no masked pooled delta lies within 1e-2 of the
    mean + std threshold); the kept sets under the GPU's own K_r match the oracle's
    selection under the same K_r (with constraints: the closure of the candidates)."""
    cfg, ov, wide = STRUCTURED_CASES[case]
    p = synth.make_problem(cfg, seed=700, wide_logits=wide, overrides=ov)
    rng = np.random.default_rng(7)
    avg = rng.uniform(0.0, 4.0, size=p.R).astype(np.float32)
    ref = orc.evict(p, decode_avg=avg.astype(np.float64))
    g = p.to("cuda")
    out = _evict_dynamic(p, g, avg, constraints)
    assert out["status"] == 0
    assert_close_delta(out["delta"], ref["pooled"])
    dec = p.decoded.numpy()
    kg = out["budget"]
    check_dynamic_budget(kg, ref["pooled"], dec, avg)
    if constraints == 0:
        check_selection_all(out["kept"], out["cu_seqlens"], ref, dec, kg, orc)
    else:
        cand = _evict_dynamic(p, g, avg, 0)
        np.testing.assert_array_equal(cand["delta"], out["delta"])
        np.testing.assert_array_equal(cand["budget"], kg)
        check_structured(out["kept"], out["cu_seqlens"], cand["kept"], cand["cu_seqlens"], ref,
                         dec, kg, constraints, orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))


def test_head_sharded_two_way_matches_fused(orc):
    """Tensor-parallel head sharding, emulated on one GPU: two head shards' partial
    importance summed (the all-reduce), then delta/select/compaction, give the fused
    step's results within tolerance and the oracle's selection."""
    import attention_delta_token_b200 as F
    from attention_delta_token_b200 import parallel
    p = synth.make_problem(1, seed=800, wide_logits=True, overrides=dict(R=10))
    g = p.to("cuda")
    world = 2
    parts = []
    for rank in range(world):
        hq, hk = parallel.shard_heads(p.Hq, p.Hkv, rank, world)
        parts.append(parallel.partial_importance(
            p.R, p.B, p.Hq // world, p.Hkv // world, p.d,
            g.q0[:, :, hq].contiguous(), g.k0_prefix[:, hk].contiguous(),
            g.k0_block[:, :, hk].contiguous(), g.q1[:, :, hq].contiguous(),
            g.k1_prefix[:, hk].contiguous(), g.k1_block[:, :, hk].contiguous(), g.cu_prefix,
            p.scale))
    total = parts[0] + parts[1]  # what the all-reduce computes
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    cap = F.plan_capacity(p.decoded, p.budget)
    kept = torch.empty(cap, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.empty(cap, p.H, dtype=torch.bfloat16, device="cuda")
    delta = torch.empty(p.R, p.B, device="cuda")
    ws = parallel.finish_from_importance(dims, total, g.decoded, g.budget, g.hidden, kept, cu,
                                         packed, delta_out=delta)
    assert F.focus_read_device_status(ws) == 0
    fused = run_evict(g)
    assert_close_importance(total[0].cpu().numpy(), fused["i0"], "I0 sharded vs fused")
    assert_close_importance(total[1].cpu().numpy(), fused["i1"], "I1 sharded vs fused")
    ref = orc.evict(p)
    assert_close_delta(delta.cpu().numpy(), ref["pooled"])
    check_selection_all(kept.cpu().numpy(), cu.cpu().numpy(), ref, p.decoded.numpy(),
                        p.budget.numpy(), orc)
    check_packed(packed.view(torch.int16).cpu().numpy().view(np.uint16), kept.cpu().numpy(),
                 cu.cpu().numpy(), hidden_bits(p))


@pytest.mark.parametrize("constraints,score", [(0, 0), (3, 0), (0, 1), (3, 1)])
def test_split_halves_bitwise_equal_fused(constraints, score):
    """focus_partial_importance over all heads, then focus_evict_from_importance, give
    the fused step's importance, delta, kept set and packed rows bit for bit (the same
    column sums reduced in the same order); the importance also equals focus_attn_stats
    per layer."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(4, seed=810 + 2 * constraints + score, overrides=dict(R=12))
    g = p.to("cuda")
    fused = run_evict(g, constraints=constraints, score=score)
    assert fused["status"] == 0
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window, constraints,
                       score)
    ws = F.Workspace(dims, "cuda")
    imp = torch.full((2, p.R, p.B), float("nan"), device="cuda")
    l0 = (None, None, None) if score else (g.q0, g.k0_prefix, g.k0_block)
    F.focus_partial_importance(dims, *l0, g.q1, g.k1_prefix, g.k1_block, g.cu_prefix, imp, ws)
    cap = F.plan_capacity(p.decoded, p.budget, constraints)
    kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.zeros(cap, p.H, dtype=torch.bfloat16, device="cuda")
    delta = torch.empty(p.R, p.B, device="cuda")
    F.focus_evict_from_importance(dims, imp, g.hidden, g.decoded, g.budget, kept, cu, packed,
                                  ws, delta_out=delta)
    assert F.focus_read_device_status(ws) == 0
    np.testing.assert_array_equal(imp[1].cpu().numpy(), fused["i1"].astype(np.float32))
    if score:
        assert torch.isnan(imp[0]).all()  # layer 0 untouched
    else:
        np.testing.assert_array_equal(imp[0].cpu().numpy(), fused["i0"].astype(np.float32))
        one = torch.empty(p.R, p.B, device="cuda")
        for layer, (q, kp, kb) in enumerate(((g.q0, g.k0_prefix, g.k0_block),
                                             (g.q1, g.k1_prefix, g.k1_block))):
            F.focus_attn_stats(dims, q, kp, g.cu_prefix, kb, one, ws)
            assert torch.equal(one, imp[layer])
    np.testing.assert_array_equal(delta.cpu().numpy(), fused["delta"].astype(np.float32))
    cu_h = cu.cpu().numpy()
    np.testing.assert_array_equal(cu_h, fused["cu_seqlens"])
    n = int(cu_h[-1])
    np.testing.assert_array_equal(kept[:n].cpu().numpy(), fused["kept"][:n])
    np.testing.assert_array_equal(packed[:n].view(torch.int16).cpu().numpy().view(np.uint16),
                                  fused["packed"][:n])


EDGE_CASES = {
    # more than 1024 requests: the planner orders them with a bitonic sort
    "r1500_tiny_heads": (0, dict(R=1500, B=8, Hq=2, Hkv=1, d=64, H=64, prefix=("uniform", 0, 200),
                                 decoded=("uniform", 0.0, 0.5), lift=("frac", 0.2),
                                 budget=("ceil", 0.3))),
    # the last batch ordered by a rank count (1024), the last one sorted (4096; the compaction
    # no longer stages cu_seqlens in shared memory) and the first one kept in input order
    **{f"r{R}_tiny_heads": (0, dict(R=R, B=8, Hq=2, Hkv=1, d=64, H=64, prefix=("uniform", 0, 200),
                                    decoded=("uniform", 0.0, 0.5), lift=("frac", 0.2),
                                    budget=("ceil", 0.3)))
       for R in (1024, 4096, 4097)},
    # one very long prefix: 157 key tiles in one work item
    "long_prefix_20k": (1, dict(R=2, prefix=("uniform", 19000, 20000))),
    # multi-query attention: all 32 query heads read one kv head (4 tokens per row tile)
    "mqa_g32": (1, dict(R=3, Hq=32, Hkv=1, prefix=("uniform", 0, 400))),
    # d = 64 with 16 query heads per kv head
    "d64_g16": (1, dict(R=4, d=64, Hq=32, Hkv=2, prefix=("uniform", 0, 300))),
    # prefixes ending just before, at and just after a 128-key tile boundary
    "tile_edges_128": (1, dict(R=12, prefix=("uniform", 127, 129))),
    "tile_edges_256": (4, dict(R=12, prefix=("uniform", 255, 257))),
    # the largest group: 128 query heads on one kv head, one block token per row tile
    "g128_b4": (0, dict(R=3, B=4, Hq=128, Hkv=1, d=64, H=64, prefix=("uniform", 0, 300),
                        decoded=("uniform", 0.0, 0.5), lift=("frac", 0.25), budget=("ceil", 0.5))),
    # the largest block with 64 query heads per kv head: 64 row tiles per kv head
    "g64_b128": (3, dict(R=2, d=64, Hq=64, Hkv=1, H=256, prefix=("uniform", 100, 400))),
}


@pytest.mark.parametrize("case", sorted(EDGE_CASES))
def test_edge_shapes_vs_oracle(case, orc):
    cfg, ov = EDGE_CASES[case]
    p = synth.make_problem(cfg, seed=900 + sorted(EDGE_CASES).index(case), wide_logits=True,
                           overrides=ov)
    ref = orc.evict(p)
    out = run_evict(p.to("cuda"))
    assert out["status"] == 0
    assert_close_importance(out["i0"], ref["i0"], "I0")
    assert_close_importance(out["i1"], ref["i1"], "I1")
    assert_close_delta(out["delta"], ref["pooled"])
    np.testing.assert_array_equal(out["cu_seqlens"], ref["cu_seqlens"])
    check_selection_all(out["kept"], out["cu_seqlens"], ref, p.decoded.numpy(),
                        p.budget.numpy(), orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))


@pytest.mark.parametrize("constraints,score", [(0, 0), (3, 0), (0, 1)])
def test_peer_exchange_single_rank_bitwise_equal_fused(constraints, score):
    """The fused-exchange path with a group of one (the rank pushes to its own buffer and
    its selection waits for its own flag), over three consecutive steps so both slot
    parities are used, reproduces focus_evict bit for bit."""
    import attention_delta_token_b200 as F
    from attention_delta_token_b200 import parallel
    base = dict(R=9)
    dims = None
    ex = None
    for step, seed in enumerate((820, 821, 822)):
        p = synth.make_problem(4, seed=seed + 10 * constraints + 100 * score, overrides=base)
        g = p.to("cuda")
        fused = run_evict(g, constraints=constraints, score=score)
        assert fused["status"] == 0
        if dims is None:
            dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window,
                               constraints, score)
            ex = parallel.PeerExchange.local(dims, "cuda")
        cap = F.plan_capacity(p.decoded, p.budget, constraints)
        kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
        packed = torch.zeros(cap, p.H, dtype=torch.bfloat16, device="cuda")
        delta = torch.empty(p.R, p.B, device="cuda")
        l0 = (None, None, None) if score else (g.q0, g.k0_prefix, g.k0_block)
        ws = parallel.evict_head_sharded(dims, 0, 1, *l0, g.q1, g.k1_prefix, g.k1_block,
                                         g.cu_prefix, g.hidden, g.decoded, g.budget, kept, cu,
                                         packed, delta_out=delta, exchange=ex)
        assert F.focus_read_device_status(ws) == 0
        assert F.focus_read_device_status(ex.push_ws) == 0
        assert ex.epoch == step + 1
        np.testing.assert_array_equal(delta.cpu().numpy(), fused["delta"].astype(np.float32))
        cu_h = cu.cpu().numpy()
        np.testing.assert_array_equal(cu_h, fused["cu_seqlens"])
        n = int(cu_h[-1])
        np.testing.assert_array_equal(kept[:n].cpu().numpy(), fused["kept"][:n])
        np.testing.assert_array_equal(
            packed[:n].view(torch.int16).cpu().numpy().view(np.uint16), fused["packed"][:n])
    # the flags of both parities hold the last epoch that used them
    lay = F.focus_exchange_buffer_size(dims, 1)
    flags = ex.buffer[lay - 256:lay - 256 + 8].view(torch.int32).cpu().tolist()
    assert flags == [2, 3]


@pytest.mark.parametrize("world", [2, 3, 8])
def test_peer_exchange_protocol_emulated_ranks(world):
    """The push / flag / wait / rank-ordered sum of the exchange with `world` ranks
    emulated by block groups of one cooperative launch on one GPU: every rank ends with
    the same sums, equal (bitwise) to the float32 sum in rank order; three steps in a
    row use both slot parities."""
    import attention_delta_token_b200 as F
    R, B = 5, 32
    dims = F.make_dims(R, B, 4, 2, 64, 8)
    nbytes = F.focus_exchange_buffer_size(dims, world)
    bufs = [torch.zeros(nbytes, dtype=torch.uint8, device="cuda") for _ in range(world)]
    ptrs = torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device="cuda")
    gen = torch.Generator().manual_seed(world)
    for epoch in (1, 2, 3):
        scale = 10.0 ** torch.randint(-3, 3, (world, 1, 1, 1), generator=gen).float()
        parts = torch.randn(world, 2, R, B, generator=gen) * scale
        out = torch.full((world, 2, R, B), float("nan"), device="cuda")
        scratch = torch.zeros(1 + world, dtype=torch.int32, device="cuda")
        F.focus_selftest_exchange(parts.cuda(), ptrs, out, scratch, epoch)
        torch.cuda.synchronize()
        assert int(scratch[0]) == 0
        assert scratch[1:].eq(0).all()  # the last block of each rank reset its counter
        want = torch.zeros(2, R, B)
        for q in range(world):
            want = want + parts[q]
        got = out.cpu()
        for q in range(world):
            assert torch.equal(got[q], want), (epoch, q)


def test_peer_exchange_missing_rank_times_out():
    """A group of two in which rank 1 never pushes: rank 0's selection gives up after its
    bounded wait, reports FOCUS_ERR_TIMEOUT, and the context stays usable."""
    import time
    import attention_delta_token_b200 as F
    p = synth.make_problem(0, seed=830)
    g = p.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    nbytes = F.focus_exchange_buffer_size(dims, 2)
    bufs = [torch.zeros(nbytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    ptrs = torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device="cuda")
    sdims = F.make_dims(p.R, p.B, p.Hq // 2, p.Hkv // 2, p.d, 8, p.scale)
    push_ws = F.Workspace(sdims, "cuda")
    from attention_delta_token_b200 import parallel
    hq, hk = parallel.shard_heads(p.Hq, p.Hkv, 0, 2)
    F.focus_partial_importance_push(sdims, g.q0[:, :, hq].contiguous(),
                                    g.k0_prefix[:, hk].contiguous(),
                                    g.k0_block[:, :, hk].contiguous(), g.q1[:, :, hq].contiguous(),
                                    g.k1_prefix[:, hk].contiguous(),
                                    g.k1_block[:, :, hk].contiguous(), g.cu_prefix, ptrs, 0, 2, 1,
                                    push_ws)
    assert F.focus_read_device_status(push_ws) == 0
    ws = F.Workspace(dims, "cuda")
    cap = F.plan_capacity(p.decoded, p.budget)
    kept = torch.empty(cap, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.empty(cap, p.H, dtype=torch.bfloat16, device="cuda")
    t0 = time.time()
    F.focus_evict_from_exchange(dims, bufs[0], 2, 1, g.hidden, g.decoded, g.budget, kept, cu,
                                packed, ws)
    st = F.focus_read_device_status(ws, timeout_ms=20000)
    assert st == 7  # FOCUS_ERR_TIMEOUT
    assert 1.5 < time.time() - t0 < 15
    # rank 0's own slot arrived, rank 1's flag did not
    flags = bufs[0][nbytes - 256:nbytes - 256 + 16].view(torch.int32).cpu().tolist()
    assert flags == [0, 0, 1, 0]
    out = run_evict(g)  # the context is still usable
    assert out["status"] == 0


def test_peer_exchange_symmetric_memory_group_of_one():
    """PeerExchange.symmetric (torch symmetric memory, one NCCL rank on one GPU) drives the
    fused exchange end to end and matches focus_evict bit for bit; run in a child process
    under a time limit."""
    import socket
    import subprocess
    import sys
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0",
               WORLD_SIZE="1", LOCAL_RANK="0", NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, os.path.join(here, "_symm_exchange_child.py")],
                       capture_output=True, text=True, timeout=300, env=env, cwd=here)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout[-2000:] + r.stderr[-3000:]


@pytest.mark.parametrize("constraints", [0, 3])
def test_dynamic_budget_degenerate_blocks(constraints, orc):
    """Dynamic budget on degenerate blocks: a fully decoded block keeps nothing (K = 0), a
    single masked token is kept (K = 1, its sigma is 0), a fully masked block with a huge
    historical yield is capped at the masked count, a zero yield still keeps one token; the
    budgets, kept sets and packed rows equal the oracle's."""
    p = synth.make_problem(1, seed=850, wide_logits=True, overrides=dict(R=4))
    dec = p.decoded.numpy()
    dec[0] = 1
    dec[1] = 1
    dec[1, 7] = 0
    dec[2] = 0
    avg = np.array([3.0, 2.0, 1000.0, 0.0], np.float32)
    ref = orc.evict(p, decode_avg=avg.astype(np.float64))
    np.testing.assert_array_equal(ref["budget"][:3], [0, 1, p.B])
    g = p.to("cuda")
    out = _evict_dynamic(p, g, avg, constraints)
    assert out["status"] == 0
    kg = out["budget"]
    np.testing.assert_array_equal(kg[:3], ref["budget"][:3])
    check_dynamic_budget(kg, ref["pooled"], dec, avg)
    cu_h = out["cu_seqlens"]
    assert cu_h[1] == 0                       # the fully decoded block keeps nothing
    assert list(out["kept"][cu_h[1]:cu_h[2]]) == (
        [6, 7] if constraints & 1 else [7])   # the lone masked token (and its predecessor)
    assert cu_h[3] - cu_h[2] == p.B           # the fully masked block is kept whole
    check_packed(out["packed"], out["kept"], cu_h, hidden_bits(p))
    if constraints:
        cand = _evict_dynamic(p, g, avg, 0)
        check_structured(out["kept"], cu_h, cand["kept"], cand["cu_seqlens"], ref, dec, kg,
                         constraints, orc)
    else:
        check_selection_all(out["kept"], cu_h, ref, dec, kg, orc)


@pytest.mark.parametrize("window", [1, 5, 7])
def test_other_pool_windows_vs_oracle(window, orc):
    """MaxPool1D with windows other than the pages' k = 3 (the ABI takes any odd window):
    the fused step and the stand-alone delta call against the oracle."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, seed=860 + window, wide_logits=True,
                           overrides=dict(R=5, prefix=("uniform", 0, 500), pool_window=window))
    assert p.pool_window == window
    ref = orc.evict(p)
    g = p.to("cuda")
    _compare_full(p, run_evict(g), ref, orc)
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, window)
    i0 = torch.from_numpy(ref["i0"]).float().cuda()
    i1 = torch.from_numpy(ref["i1"]).float().cuda()
    delta = torch.empty(p.R, p.B, device="cuda")
    F.focus_importance_delta(dims, i0, i1, g.decoded, delta)
    _, want = orc.delta_pool_mask(i0.double().cpu().numpy(), i1.double().cpu().numpy(),
                                  p.decoded.numpy(), window=window)
    assert_close_delta(delta.cpu().numpy(), want)


def test_cuda_graph_replay_matches_direct_calls():
    """focus_evict captured into a CUDA graph (four kernels with programmatic dependent
    launch edges): replays on new inputs copied into the captured buffers give the same
    bits as direct calls on those inputs."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, seed=870, overrides=dict(R=8))
    g = p.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    ws = F.Workspace(dims, "cuda")
    # capacity for any decoded pattern of the same budgets: the replay's shape is fixed
    cap = int(p.budget.clamp(min=0).clamp(max=p.B).sum())
    kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.zeros(cap, p.H, dtype=torch.bfloat16, device="cuda")
    delta = torch.empty(p.R, p.B, device="cuda")

    def step():
        F.focus_evict(dims, g.q0, g.k0_prefix, g.k0_block, g.q1, g.k1_prefix, g.k1_block,
                      g.cu_prefix, g.hidden, g.decoded, g.budget, kept, cu, packed, ws,
                      delta_out=delta)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # the uncaptured first call
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for seed in (871, 872):
        # new values in the same buffers: the prefix layout (cu_prefix) and the budgets
        # stay, so the captured capacity still bounds every request's kept count
        q = synth.make_problem(1, seed=seed, overrides=dict(R=8))
        for name in ("q0", "k0_block", "q1", "k1_block", "hidden", "decoded"):
            getattr(g, name).copy_(getattr(q, name))
        gen = torch.Generator().manual_seed(seed)
        for name in ("k0_prefix", "k1_prefix"):
            t = getattr(g, name)
            t.copy_((torch.randn(t.shape, generator=gen) / p.d ** 0.5).to(torch.bfloat16))
        graph.replay()
        torch.cuda.synchronize()
        assert F.focus_read_device_status(ws) == 0
        got = [t.clone() for t in (kept, cu, packed.view(torch.int16), delta)]
        step()
        assert F.focus_read_device_status(ws) == 0
        want = [kept, cu, packed.view(torch.int16), delta]
        n = int(cu[-1])
        assert n <= cap
        assert torch.equal(got[1], want[1])
        assert torch.equal(got[0][:n], want[0][:n]) and torch.equal(got[2][:n], want[2][:n])
        assert torch.equal(got[3], want[3])


SPLIT_CASES = {
    # (config, overrides): batches of at most 148 (layer, request, kv head, row tile)
    # groups, so each group's prefix is split into chunks merged by the last one
    "r1_l13k": (1, dict(R=1, prefix=("uniform", 12000, 13000))),
    "r3_mixed": (1, dict(R=3, prefix=("uniform", 300, 6000))),
    "r2_b128_mt4": (3, dict(R=2, prefix=("uniform", 3000, 5000))),
    "r4_d64_g16": (1, dict(R=4, d=64, Hq=32, Hkv=2, prefix=("uniform", 2000, 9000))),
}


@pytest.mark.parametrize("case", sorted(SPLIT_CASES))
def test_split_prefix_vs_oracle_and_deterministic(case, orc):
    """Split prefixes (several CTAs per (layer, request, kv head, row tile), merged by
    the last chunk) against the oracle, bit-identical on a second run, and the
    stand-alone one-layer call splits the same way (bit-identical importance)."""
    import attention_delta_token_b200 as F
    cfg, ov = SPLIT_CASES[case]
    p = synth.make_problem(cfg, seed=880 + sorted(SPLIT_CASES).index(case), wide_logits=True,
                           overrides=ov)
    assert 2 * p.R * p.Hkv * -(-p.Hq // p.Hkv * p.B // 128) <= 148
    ref = orc.evict(p)
    g = p.to("cuda")
    a = run_evict(g)
    _compare_full(p, a, ref, orc)
    b = run_evict(g)
    for key in ("i0", "i1", "delta", "kept", "packed", "cu_seqlens"):
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    ws = F.Workspace(dims)
    i1 = torch.empty(p.R, p.B, device="cuda")
    F.focus_attn_stats(dims, g.q1, g.k1_prefix, g.cu_prefix, g.k1_block, i1, ws)
    assert F.focus_read_device_status(ws) == 0
    np.testing.assert_array_equal(i1.cpu().numpy(), a["i1"].astype(np.float32))


def test_split_prefix_paged_and_constrained(orc):
    """Split prefixes through the paged layout and with structural constraints."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, seed=890, wide_logits=True,
                           overrides=dict(R=2, prefix=("uniform", 4000, 7000)))
    ref = orc.evict(p)
    g = p.to("cuda")
    packed_out = run_evict(g)
    pg = synth.to_paged(p, 64, seed=890).to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    ws = F.Workspace(dims, "cuda")
    cap = F.plan_capacity(p.decoded, p.budget)
    kept = torch.empty(cap, dtype=torch.int32, device="cuda")
    cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
    packed = torch.empty(cap, p.H, dtype=torch.bfloat16, device="cuda")
    i0 = torch.empty(p.R, p.B, device="cuda")
    i1 = torch.empty(p.R, p.B, device="cuda")
    F.focus_evict_paged(dims, g.q0, pg.k0_pages, g.k0_block, g.q1, pg.k1_pages, g.k1_block,
                        pg.page_table, pg.prefix_len, g.hidden, g.decoded, g.budget, kept, cu,
                        packed, ws, i0_out=i0, i1_out=i1)
    assert F.focus_read_device_status(ws) == 0
    # the same chunks over the same keys: bit-identical to the packed layout
    np.testing.assert_array_equal(i0.cpu().numpy(), packed_out["i0"].astype(np.float32))
    np.testing.assert_array_equal(i1.cpu().numpy(), packed_out["i1"].astype(np.float32))
    out = run_evict(g, constraints=3)
    assert out["status"] == 0
    np.testing.assert_array_equal(out["delta"], packed_out["delta"])
    assert_close_delta(out["delta"], ref["pooled"])
    check_structured(out["kept"], out["cu_seqlens"], packed_out["kept"], packed_out["cu_seqlens"],
                     ref, p.decoded.numpy(), p.budget.numpy(), 3, orc)


def test_split_prefix_malformed_cu_prefix_reports():
    """A malformed prefix offset in a split batch: the request is computed with no
    prefix (its chunks carry no tiles), FOCUS_ERR_DEVICE_CHECK is reported, and no
    last chunk waits past its bound."""
    p = synth.make_problem(1, seed=895, overrides=dict(R=3, prefix=("uniform", 3000, 4000)))
    g = p.to("cuda")
    g.cu_prefix[2] = g.cu_prefix[3] + 5  # request 1 ends after request 2's end
    out = run_evict(g)
    assert out["status"] == 6  # FOCUS_ERR_DEVICE_CHECK, not a timeout


@pytest.mark.parametrize("case", ["sdar_r8_wide", "block128_r3"])
def test_all_options_together_vs_oracle(case, orc):
    """focus_evict_ex with every option at once: paged prefix keys (64-token pages), the
    layer-0 row log-sum-exps given, the dynamic budget and both structural constraints,
    against the oracle run with the same options: every request's budget within the
    oracle's bounds, every retained list the closure of candidates that match the
    oracle's selection under the GPU's budgets."""
    cfg, ov, wide = STRUCTURED_CASES[case]
    p = synth.make_problem(cfg, seed=910, wide_logits=wide, overrides=ov)
    lse = _row_lse(p).float()
    avg = np.random.default_rng(9).uniform(0.0, 4.0, size=p.R).astype(np.float32)
    ref = orc.evict(p, lse0=lse.double().numpy(), decode_avg=avg.astype(np.float64))
    g = p.to("cuda")
    pg = synth.to_paged(p, 64, seed=910).to("cuda")
    opts = dict(q0=g.q0, k0_prefix=None, k0_block=g.k0_block, lse0=lse.cuda(), q1=g.q1,
                k1_prefix=pg.k1_pages, k1_block=g.k1_block, cu_prefix=None,
                page_table=pg.page_table, prefix_len=pg.prefix_len)
    out = _evict_dynamic(p, g, avg, 3, **opts)
    cand = _evict_dynamic(p, g, avg, 0, **opts)
    assert out["status"] == 0 and cand["status"] == 0
    np.testing.assert_array_equal(out["delta"], cand["delta"])
    np.testing.assert_array_equal(out["budget"], cand["budget"])
    assert_close_delta(out["delta"], ref["pooled"])
    dec = p.decoded.numpy()
    kg = out["budget"]
    check_dynamic_budget(kg, ref["pooled"], dec, avg)
    check_structured(out["kept"], out["cu_seqlens"], cand["kept"], cand["cu_seqlens"], ref, dec,
                     kg, 3, orc)
    check_packed(out["packed"], out["kept"], out["cu_seqlens"], hidden_bits(p))


def test_paged_bad_entries_report():
    """A page index outside the pool (the copy falls back to page 0, in bounds) and a
    prefix length beyond the request's pages (computed with no prefix) are reported as
    FOCUS_ERR_DEVICE_CHECK; the call stays in bounds and later calls are unaffected."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, seed=920, overrides=dict(R=3, prefix=("uniform", 300, 600)))
    g = p.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    cap = F.plan_capacity(p.decoded, p.budget)

    def call(pg):
        ws = F.Workspace(dims)
        kept = torch.empty(cap, dtype=torch.int32, device="cuda")
        cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
        packed = torch.empty(cap, p.H, dtype=torch.bfloat16, device="cuda")
        F.focus_evict_paged(dims, g.q0, pg.k0_pages, g.k0_block, g.q1, pg.k1_pages, g.k1_block,
                            pg.page_table, pg.prefix_len, g.hidden, g.decoded, g.budget, kept, cu,
                            packed, ws)
        return F.focus_read_device_status(ws)

    pg = synth.to_paged(p, 64, seed=920).to("cuda")
    assert call(pg) == 0
    bad = synth.to_paged(p, 64, seed=920).to("cuda")
    bad.page_table[1, 0] = bad.k1_pages.shape[0] + 5     # past the pool
    assert call(bad) == 6
    bad = synth.to_paged(p, 64, seed=920).to("cuda")
    bad.page_table[2, 1] = -1
    assert call(bad) == 6
    bad = synth.to_paged(p, 64, seed=920).to("cuda")
    bad.prefix_len[0] = bad.page_table.shape[1] * 64 + 1  # longer than its pages
    assert call(bad) == 6
    assert call(pg) == 0


def test_split_prefix_with_lse0_vs_oracle(orc):
    """Split prefixes with layer 0's row log-sum-exps given: the layer-0 groups (block keys
    only) stay whole, the layer-1 groups are split; against the oracle's importance from
    the LSE, and bit-identical on a second run."""
    import attention_delta_token_b200 as F
    p = synth.make_problem(1, seed=930, wide_logits=True,
                           overrides=dict(R=2, prefix=("uniform", 8000, 9000)))
    assert 2 * p.R * p.Hkv <= 148  # a split batch
    lse = _row_lse(p).float()
    ref = orc.evict(p, lse0=lse.double().numpy())
    g = p.to("cuda")
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    cap = F.plan_capacity(p.decoded, p.budget)
    outs = []
    for _ in range(2):
        ws = F.Workspace(dims)
        kept = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
        packed = torch.zeros(cap, p.H, dtype=torch.bfloat16, device="cuda")
        i0 = torch.empty(p.R, p.B, device="cuda")
        i1 = torch.empty_like(i0)
        delta = torch.empty_like(i0)
        F.focus_evict_with_lse0(dims, lse.cuda(), g.q0, g.k0_block, g.q1, g.k1_prefix, g.k1_block,
                                g.cu_prefix, g.hidden, g.decoded, g.budget, kept, cu, packed, ws,
                                delta_out=delta, i0_out=i0, i1_out=i1)
        assert F.focus_read_device_status(ws) == 0
        outs.append([t.cpu() for t in (i0, i1, delta, kept, cu)])
    i0, i1, delta, kept, cu = outs[0]
    assert_close_importance(i0.numpy(), ref["i0"], "I0 from lse")
    assert_close_importance(i1.numpy(), ref["i1"], "I1 (split)")
    assert_close_delta(delta.numpy(), ref["pooled"])
    check_selection_all(kept.numpy(), cu.numpy(), ref, p.decoded.numpy(), p.budget.numpy(), orc)
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


def _guarded(n, dtype, fill, guard=256):
    """A device buffer of n elements with `guard` sentinel elements on each side; returns
    (whole, inner view).  Integer sentinels for integer dtypes, NaN bit patterns otherwise."""
    whole = torch.empty(n + 2 * guard, dtype=dtype, device="cuda")
    whole.view(torch.uint8).fill_(fill)
    return whole, whole[guard:guard + n]


def _guards_intact(whole, n, fill, guard=256):
    b = whole.view(torch.uint8)
    per = whole.element_size()
    return bool((b[:guard * per] == fill).all()) and bool((b[(guard + n) * per:] == fill).all())


@pytest.mark.parametrize("mode", ["plain", "constraints", "split", "paged", "static"])
def test_outputs_and_workspace_guard_zones(mode):
    """Canary zones before and after every output buffer and the workspace stay
    untouched: no kernel writes outside the ranges the ABI gives it."""
    import attention_delta_token_b200 as F
    ov = dict(R=3, prefix=("uniform", 4000, 6000)) if mode == "split" else \
        dict(R=20, prefix=("uniform", 100, 900))
    p = synth.make_problem(1, seed=940, overrides=ov)
    g = p.to("cuda")
    constraints = 3 if mode == "constraints" else 0
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window, constraints)
    cap = F.plan_capacity(p.decoded, p.budget, constraints)
    fill = 0xA5
    bufs = {
        "kept": (cap, torch.int32), "cu": (p.R + 1, torch.int32),
        "packed": (cap * p.H, torch.bfloat16), "delta": (p.R * p.B, torch.float32),
        "i0": (p.R * p.B, torch.float32), "i1": (p.R * p.B, torch.float32),
    }
    whole, inner = {}, {}
    for k, (n, dt) in bufs.items():
        whole[k], inner[k] = _guarded(n, dt, fill)
    ws_bytes = F.focus_workspace_size(dims)
    ws_whole, ws_inner = _guarded(ws_bytes, torch.uint8, fill, guard=4096)
    ws = F.Workspace.__new__(F.Workspace)
    ws.nbytes, ws.buf = ws_bytes, ws_inner
    assert ws_inner.data_ptr() % 256 == 0
    F.focus_clear_device_status(ws)
    packed = inner["packed"].view(cap, p.H)
    if mode == "paged":
        pg = synth.to_paged(p, 64, seed=940).to("cuda")
        F.focus_evict_paged(dims, g.q0, pg.k0_pages, g.k0_block, g.q1, pg.k1_pages, g.k1_block,
                            pg.page_table, pg.prefix_len, g.hidden, g.decoded, g.budget,
                            inner["kept"], inner["cu"], packed, ws,
                            delta_out=inner["delta"].view(p.R, p.B),
                            i0_out=inner["i0"].view(p.R, p.B), i1_out=inner["i1"].view(p.R, p.B))
    elif mode == "static":
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        F.focus_evict_static_scratch(dims, g.q0, g.k0_prefix, g.k0_block, g.q1, g.k1_prefix,
                                     g.k1_block, g.cu_prefix, g.hidden, g.decoded, g.budget,
                                     inner["kept"], inner["cu"], packed, device_status=st,
                                     delta_out=inner["delta"].view(p.R, p.B),
                                     i0_out=inner["i0"].view(p.R, p.B),
                                     i1_out=inner["i1"].view(p.R, p.B))
        torch.cuda.synchronize()
        assert int(st.item()) == 0
    else:
        F.focus_evict(dims, g.q0, g.k0_prefix, g.k0_block, g.q1, g.k1_prefix, g.k1_block,
                      g.cu_prefix, g.hidden, g.decoded, g.budget, inner["kept"], inner["cu"],
                      packed, ws, delta_out=inner["delta"].view(p.R, p.B),
                      i0_out=inner["i0"].view(p.R, p.B), i1_out=inner["i1"].view(p.R, p.B))
    if mode != "static":
        assert F.focus_read_device_status(ws) == 0
    torch.cuda.synchronize()
    for k, (n, _) in bufs.items():
        assert _guards_intact(whole[k], n, fill), k
    assert _guards_intact(ws_whole, ws_bytes, fill, guard=4096), "workspace"
