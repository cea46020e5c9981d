"""focus_evict_static_scratch: the fused step for callers that cannot allocate.

Some callers cannot hand the library a workspace: an engine that has committed
nearly all HBM to its KV cache and may not allocate while decoding, or a plug-in
that sees only the C ABI and not its host framework's memory pool.  For them the
library keeps the scratch in its own fixed device array.  These checks call that
entry point through the C ABI and compare it with focus_evict, which uses a
caller-allocated workspace, on two calls in a row (a larger problem, then a
smaller one, so a stale array would show).

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


def _static_scratch_run(p):
    dev = p.q0.device
    dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
    cap = F.plan_capacity(p.decoded, p.budget)
    kept = torch.full((max(cap, 1),), -1, dtype=torch.int32, device=dev)[:cap]
    cu = torch.full((p.R + 1,), -7, dtype=torch.int32, device=dev)
    packed = torch.zeros((max(cap, 1), p.H), dtype=torch.bfloat16, device=dev)[:cap]
    delta = torch.full((p.R, p.B), float("nan"), device=dev)
    i0, i1 = torch.full_like(delta, float("nan")), torch.full_like(delta, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    F.focus_evict_static_scratch(dims, p.q0, p.k0_prefix, p.k0_block, p.q1, p.k1_prefix,
                                 p.k1_block, p.cu_prefix, p.hidden, p.decoded, p.budget, kept, cu,
                                 packed, device_status=status, delta_out=delta, i0_out=i0,
                                 i1_out=i1)
    torch.cuda.synchronize()
    return dict(kept=kept.cpu().numpy(), cu_seqlens=cu.cpu().numpy(),
                packed=packed.view(torch.int16).cpu().numpy().view(np.uint16),
                delta=delta.cpu().numpy().astype(np.float64), i0=i0.cpu().numpy().astype(np.float64),
                i1=i1.cpu().numpy().astype(np.float64), status=int(status.item()))


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_twice():
    problems = [
        synth.make_problem(4, overrides=dict(R=48, prefix=("loguniform", 2000)), wide_logits=True),
        synth.make_problem(1, overrides=dict(R=6, prefix=("uniform", 0, 700))),
    ]
    for p in problems:  # two calls in a row, different shapes
        g = p.to("cuda")
        got = _static_scratch_run(g)
        want = run_evict(g)
        assert got["status"] == 0 and want["status"] == 0
        assert_close_importance(got["i0"], want["i0"], "I0")
        assert_close_importance(got["i1"], want["i1"], "I1")
        assert_close_delta(got["delta"], want["delta"])
        np.testing.assert_array_equal(got["cu_seqlens"], want["cu_seqlens"])
        np.testing.assert_array_equal(got["kept"], want["kept"])
        np.testing.assert_array_equal(got["packed"], want["packed"])


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
