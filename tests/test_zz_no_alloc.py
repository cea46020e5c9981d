"""focus_evict_static_scratch: the fused step for callers that cannot allocate.

Some callers cannot hand the library a workspace: an engine that has committed
nearly all HBM to its KV cache and may not allocate while decoding, or a plug-in
that sees only the C ABI and not its host framework's memory pool.  For them the
library keeps the scratch in its own fixed device array.  These checks call that
entry point through the C ABI and compare it with focus_evict, which uses a
caller-allocated workspace, on two calls in a row (a larger problem, then a
smaller one, so a stale array would show), and check that repeated calls leave
the device's free memory untouched.

The file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import attention_delta_token_b200 as F
import synth
from focus_testutil import assert_close_delta, assert_close_importance, run_evict


def _outputs(p):
    """Output buffers of one static-scratch call, allocated by the test up front."""
    dev = p.q0.device
    cap = F.plan_capacity(p.decoded, p.budget)
    return dict(
        dims=F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window),
        kept=torch.full((max(cap, 1),), -1, dtype=torch.int32, device=dev)[:cap],
        cu=torch.full((p.R + 1,), -7, dtype=torch.int32, device=dev),
        packed=torch.zeros((max(cap, 1), p.H), dtype=torch.bfloat16, device=dev)[:cap],
        delta=torch.full((p.R, p.B), float("nan"), device=dev),
        i0=torch.full((p.R, p.B), float("nan"), device=dev),
        i1=torch.full((p.R, p.B), float("nan"), device=dev),
        status=torch.full((1,), -1, dtype=torch.int32, device=dev))


def _launch(p, o):
    F.focus_evict_static_scratch(o["dims"], p.q0, p.k0_prefix, p.k0_block, p.q1, p.k1_prefix,
                                 p.k1_block, p.cu_prefix, p.hidden, p.decoded, p.budget, o["kept"],
                                 o["cu"], o["packed"], device_status=o["status"],
                                 delta_out=o["delta"], i0_out=o["i0"], i1_out=o["i1"])


def _read(o):
    torch.cuda.synchronize()
    return dict(kept=o["kept"].cpu().numpy(), cu_seqlens=o["cu"].cpu().numpy(),
                packed=o["packed"].view(torch.int16).cpu().numpy().view(np.uint16),
                delta=o["delta"].cpu().numpy().astype(np.float64),
                i0=o["i0"].cpu().numpy().astype(np.float64),
                i1=o["i1"].cpu().numpy().astype(np.float64), status=int(o["status"].item()))


def _compare(got, want):
    assert got["status"] == 0 and want["status"] == 0
    assert_close_importance(got["i0"], want["i0"], "I0")
    assert_close_importance(got["i1"], want["i1"], "I1")
    assert_close_delta(got["delta"], want["delta"])
    np.testing.assert_array_equal(got["cu_seqlens"], want["cu_seqlens"])
    np.testing.assert_array_equal(got["kept"], want["kept"])
    np.testing.assert_array_equal(got["packed"], want["packed"])


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_twice():
    problems = [
        synth.make_problem(4, overrides=dict(R=48, prefix=("loguniform", 2000)), wide_logits=True),
        synth.make_problem(1, overrides=dict(R=6, prefix=("uniform", 0, 700))),
    ]
    gpu = [p.to("cuda") for p in problems]
    outs = [_outputs(g) for g in gpu]
    for g, o in zip(gpu, outs):  # two calls in a row, different shapes
        _launch(g, o)
        _compare(_read(o), run_evict(g))
    # The calls allocate nothing: with their buffers in place, repeated calls on new
    # inputs leave the device's free memory and torch's pool exactly where they were.
    torch.cuda.synchronize()
    before = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(),
              torch.cuda.memory_reserved())
    for g, o in zip(gpu, outs):
        for t in (g.q0, g.k1_block):
            t.neg_()  # new inputs, same buffers
        _launch(g, o)
    torch.cuda.synchronize()
    after = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(),
             torch.cuda.memory_reserved())
    assert after == before, (before, after)
    for g, o in zip(gpu, outs):  # and the results on the new inputs still match
        _compare(_read(o), run_evict(g))


def test_static_scratch_limit_at_the_sdar8b_shape():
    """The array holds the scratch of at most 3,840 requests at the SDAR-8B shape with
    B = 32 (the workspace grows by about 2.2 KB per request there); one more is refused
    before any CUDA call."""
    def dims(R):
        return F.make_dims(R=R, B=32, Hq=32, Hkv=8, head_dim=128, hidden=4096)
    assert F.focus_workspace_size(dims(3840)) <= F.STATIC_SCRATCH_BYTES
    assert F.focus_workspace_size(dims(3841)) > F.STATIC_SCRATCH_BYTES
    A = 0x100000
    st = F._lib.focus_evict_static_scratch(ctypes.byref(dims(3841)), A, A, A, A, A, A, A, 100, A,
                                           A, A, A, A, A, 16, None, None, None, None, None)
    assert st == 4  # FOCUS_ERR_WORKSPACE


def test_static_scratch_rejects_shapes_beyond_its_array():
    """Workspaces larger than the fixed array are refused before any CUDA call."""
    dims = F.make_dims(R=40000, B=128, Hq=32, Hkv=8, head_dim=128, hidden=4096)
    assert F.focus_workspace_size(dims) > F.STATIC_SCRATCH_BYTES
    A = 0x100000
    st = F._lib.focus_evict_static_scratch(ctypes.byref(dims), A, A, A, A, A, A, A, 100, A, A, A,
                                           A, A, A, 16, None, None, None, None, None)
    assert st == 4  # FOCUS_ERR_WORKSPACE
    bad = F.make_dims(R=4, B=200, Hq=32, Hkv=8, head_dim=128, hidden=4096)
    st = F._lib.focus_evict_static_scratch(ctypes.byref(bad), A, A, A, A, A, A, A, 100, A, A, A,
                                           A, A, A, 16, None, None, None, None, None)
    assert st == 2  # FOCUS_ERR_UNSUPPORTED_SHAPE, from the shared validation
