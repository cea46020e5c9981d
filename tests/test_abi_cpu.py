"""The C-ABI library without a GPU: it loads, exports every entry point the header
declares, and its host-side validation rejects bad arguments before touching
CUDA.  No call here reaches a kernel launch."""
import ctypes
import math
import os
import re

import numpy as np
import pytest
import torch

import attention_delta_token_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "focus.h")
HEADER_DIR = os.path.dirname(HEADER)

OK, INVALID, UNSUPPORTED, CAPACITY, WORKSPACE, CUDA, DEVCHECK, TIMEOUT = range(8)
A = 0x100000  # a 256-byte-aligned fake device address (never dereferenced here)


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"FOCUS_API\s+[\w\s\*]*?\b(focus_\w+)\s*\(", src)


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    for want in ("focus_attn_stats", "focus_importance_delta", "focus_topk_select",
                 "focus_compact", "focus_evict", "focus_workspace_size",
                 "focus_read_device_status", "focus_clear_device_status"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(F.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    for code, name in F.STATUS.items():
        assert F.focus_status_string(code) == name
    assert F.focus_abi_version() == 5


def dims(**kw):
    base = dict(R=4, B=32, Hq=32, Hkv=8, head_dim=128, hidden=4096, softmax_scale=None,
                pool_window=3)
    base.update(kw)
    return F.make_dims(**base)


def _split_bytes(R, Hkv, MT):
    """Split-prefix regions: item_base (R+1 int32), chunk counters and chunk statistics
    ((chunk_max - 1) x 256 float2 per group), each rounded to 256; none for batches of
    more than 148 (layer, request, kv head, row tile) groups."""
    groups = 2 * R * Hkv * MT
    if groups > 148:
        return 0
    cm = min(16, -(-592 // groups))
    up = lambda x: -(-x // 256) * 256
    return up(4 * (R + 1)) + up(4 * groups) + up(8 * groups * (cm - 1) * 256)


def test_workspace_size():
    d = dims()
    n = F.focus_workspace_size(d)
    # status (256) + order (R int32, rounded to 256) + 2 layers x R x Hkv x MT x B fp32
    # + retained lists (R x B int32) + counts (R int32), each rounded to 256
    base = 256 + 256 + 2 * 4 * 8 * 1 * 32 * 4 + 512 + 256
    assert n == base + _split_bytes(4, 8, 1)
    assert _split_bytes(4, 8, 1) == 256 + 256 + 8 * 64 * 9 * 256    # 64 groups: 10 chunks
    assert _split_bytes(10, 8, 1) == 0                                # 160 groups: no split
    d3 = dims(B=128)  # G*B = 512 -> 4 row tiles
    assert F.focus_workspace_size(d3) == (256 + 256 + 2 * 4 * 8 * 4 * 128 * 4 + 2048 + 256 +
                                          _split_bytes(4, 8, 4))
    big = dims(R=256)  # 4096 groups: no split regions
    assert F.focus_workspace_size(big) == (256 + 1024 + 2 * 256 * 8 * 32 * 4 + 256 * 32 * 4 +
                                           1024)
    assert F._lib.focus_workspace_size(None) == 0
    assert F._lib.focus_workspace_size(ctypes.byref(dims(B=0))) == 0


BAD_DIMS = [
    (dict(R=0), INVALID), (dict(B=0), INVALID), (dict(Hq=0), INVALID),
    (dict(softmax_scale=-1.0), INVALID), (dict(softmax_scale=math.nan), INVALID),
    (dict(softmax_scale=math.inf), INVALID), (dict(pool_window=0), INVALID),
    (dict(constraints=4), INVALID), (dict(constraints=-1), INVALID),
    (dict(score=2), INVALID), (dict(score=-1), INVALID),
    (dict(B=129), UNSUPPORTED), (dict(head_dim=96), UNSUPPORTED), (dict(head_dim=256), UNSUPPORTED),
    (dict(Hq=30, Hkv=8), UNSUPPORTED), (dict(Hq=24, Hkv=8), UNSUPPORTED),
    (dict(Hq=256, Hkv=1), UNSUPPORTED), (dict(hidden=4092), UNSUPPORTED),
    (dict(pool_window=2), UNSUPPORTED),
    (dict(R=(1 << 30) // 32 + 1), UNSUPPORTED),                       # R * B > 2^30
    (dict(R=1 << 29, B=1, Hq=2, Hkv=2, head_dim=64), UNSUPPORTED),    # 2^31 work items
]


def evict_args(d, **over):
    ws = F.focus_workspace_size(dims()) if F._lib.focus_workspace_size(ctypes.byref(d)) == 0 \
        else F.focus_workspace_size(d)
    a = dict(q0=A, k0p=A, k0b=A, q1=A, k1p=A, k1b=A, cu=A, total=100, hidden=A, dec=A,
             budget=A, kept=A, cu_s=A, packed=A, cap=16, delta=None, i0=None, i1=None,
             ws=A, ws_bytes=ws, stream=None)
    a.update(over)
    return a


def call_evict(d, a):
    return F._lib.focus_evict(ctypes.byref(d), a["q0"], a["k0p"], a["k0b"], a["q1"], a["k1p"],
                              a["k1b"], a["cu"], a["total"], a["hidden"], a["dec"], a["budget"],
                              a["kept"], a["cu_s"], a["packed"], a["cap"], a["delta"], a["i0"],
                              a["i1"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("over,code", BAD_DIMS)
def test_bad_dims_rejected_everywhere(over, code):
    d = dims(**over)
    if "softmax_scale" in over:
        d.softmax_scale = over["softmax_scale"]
    assert call_evict(d, evict_args(d)) == code
    assert F._lib.focus_attn_stats(ctypes.byref(d), A, A, A, 100, A, A, A, 1 << 20, None) == code
    assert F._lib.focus_importance_delta(ctypes.byref(d), A, A, A, A, None, None) == code
    assert F._lib.focus_topk_select(ctypes.byref(d), A, A, A, A, A, 16, A, 1 << 20, None) == code
    assert F._lib.focus_compact(ctypes.byref(d), A, A, A, A, 16, A, 1 << 20, None) == code
    assert F._lib.focus_partial_importance(ctypes.byref(d), A, A, A, A, A, A, A, 100, A, A,
                                           1 << 20, None) == code
    assert F._lib.focus_evict_from_importance(ctypes.byref(d), A, A, A, A, A, A, A, 16, None, A,
                                              1 << 20, None) == code


BAD_PTRS = [
    (dict(q0=None), INVALID), (dict(q1=A + 8), INVALID), (dict(k0b=None), INVALID),
    (dict(k1p=None), INVALID), (dict(cu=None), INVALID), (dict(cu=A + 2), INVALID),
    (dict(hidden=A + 4), INVALID), (dict(dec=None), INVALID), (dict(budget=None), INVALID),
    (dict(kept=None), INVALID), (dict(packed=A + 8), INVALID), (dict(cu_s=None), INVALID),
    (dict(delta=A + 1), INVALID), (dict(i0=A + 2), INVALID), (dict(total=-1), INVALID),
    (dict(total=1 << 40), INVALID), (dict(cap=-1), INVALID),
    (dict(ws=None), WORKSPACE), (dict(ws=A + 16), WORKSPACE), (dict(ws_bytes=100), WORKSPACE),
]


@pytest.mark.parametrize("over,code", BAD_PTRS)
def test_bad_pointers_rejected(over, code):
    d = dims()
    assert call_evict(d, evict_args(d, **over)) == code


def test_other_entry_points_check_pointers():
    d = dims()
    ws = F.focus_workspace_size(d)
    L = F._lib
    assert L.focus_attn_stats(ctypes.byref(d), None, A, A, 100, A, A, A, ws, None) == INVALID
    assert L.focus_attn_stats(ctypes.byref(d), A, None, A, 100, A, A, A, ws, None) == INVALID
    assert L.focus_attn_stats(ctypes.byref(d), A, A, A, 100, A, A + 2, A, ws, None) == INVALID
    assert L.focus_attn_stats(ctypes.byref(d), A, A, A, 100, A, A, A, ws - 4, None) == WORKSPACE
    assert L.focus_importance_delta(ctypes.byref(d), A, None, A, A, None, None) == INVALID
    assert L.focus_importance_delta(ctypes.byref(d), A, A, A, A + 1, None, None) == INVALID
    assert L.focus_topk_select(ctypes.byref(d), A, A, None, A, A, 16, A, ws, None) == INVALID
    assert L.focus_topk_select(ctypes.byref(d), A, A, A, A, A, -3, A, ws, None) == INVALID
    assert L.focus_topk_select(ctypes.byref(d), A, A, A, A, A, 16, None, ws, None) == WORKSPACE
    assert L.focus_compact(ctypes.byref(d), A + 8, A, A, A, 16, A, ws, None) == INVALID
    assert L.focus_compact(ctypes.byref(d), A, A, A, A, 16, A, 8, None) == WORKSPACE
    assert L.focus_read_device_status(None, None, 10) == WORKSPACE
    assert L.focus_clear_device_status(None, 1024, None) == WORKSPACE


def test_lse0_entry_point_validation():
    d = dims()
    ws = F.focus_workspace_size(d)
    L = F._lib
    args = lambda lse, dd: (ctypes.byref(dd), lse, A, A, A, A, A, A, 100, A, A, A, A, A, A, 16,
                            None, None, None, A, ws, None)
    assert L.focus_evict_with_lse0(*args(None, d)) == INVALID         # lse0 required
    assert L.focus_evict_with_lse0(*args(A + 2, d)) == INVALID        # misaligned
    d1 = dims(score=1)
    assert L.focus_evict_with_lse0(*args(A, d1)) == INVALID           # I1-only ranking has no layer 0
    assert L.focus_evict_with_lse0(ctypes.byref(d), A, None, A, A, A, A, A, 100, A, A, A, A, A, A,
                                   16, None, None, None, A, ws, None) == INVALID  # q0 missing


def test_paged_entry_point_validation():
    d = dims()
    ws = F.focus_workspace_size(d)
    L = F._lib

    def call(page_table=A, max_pages=4, prefix_len=A, num_pages=8, page_size=64, pool=A):
        return L.focus_evict_paged(ctypes.byref(d), A, pool, A, A, pool, A, page_table, max_pages,
                                   prefix_len, num_pages, page_size, A, A, A, A, A, A, 16, None,
                                   None, None, A, ws, None)
    assert call(page_table=None) == INVALID
    assert call(prefix_len=A + 2) == INVALID
    assert call(max_pages=0) == INVALID
    assert call(num_pages=0) == INVALID
    assert call(page_size=48) == UNSUPPORTED     # not a power of two
    assert call(page_size=4) == UNSUPPORTED      # below 8
    assert call(pool=A + 8) == INVALID           # pools must be 16-byte aligned
    assert call(num_pages=1 << 30, page_size=1 << 12) == UNSUPPORTED


def test_plan_capacity_bounds_structured_counts():
    """With structural constraints plan_capacity is an upper bound of the retained rows."""
    import oracle
    import synth
    rng = np.random.default_rng(3)
    for cfg in range(5):
        p = synth.make_problem(cfg, overrides=dict(R=min(synth.CONFIGS[cfg].R, 12), d=64,
                                                   prefix=("fixed", 0)))
        pooled = rng.normal(size=(p.R, p.B))
        pooled[p.decoded.numpy() != 0] = -np.inf
        for c in (1, 2, 3):
            _, cu, _ = oracle.select_structured(pooled, p.decoded, p.budget, c)
            assert F.plan_capacity(p.decoded, p.budget, c) >= int(cu[-1])


def test_plan_capacity_matches_oracle_counts():
    import oracle
    import synth
    for cfg in range(5):
        p = synth.make_problem(cfg, overrides=dict(R=min(synth.CONFIGS[cfg].R, 12), d=64,
                                                   prefix=("fixed", 0)))
        _, cu, _ = oracle.select(np.zeros((p.R, p.B)), p.decoded, p.budget)
        assert F.plan_capacity(p.decoded, p.budget) == int(cu[-1])


def test_split_entry_points_validation():
    """focus_partial_importance / focus_evict_from_importance reject what focus_evict
    rejects (host checks only; nothing is launched)."""
    d = dims()
    ws = F.focus_workspace_size(d)
    L = F._lib

    def partial(dd=d, q0=A, k0p=A, q1=A, imp=A, w=ws):
        return L.focus_partial_importance(ctypes.byref(dd), q0, k0p, A, q1, A, A, A, 100, imp, A,
                                          w, None)

    def from_imp(dd=d, imp=A, hidden=A, budget=A, kept=A, packed=A, cap=16, delta=None, w=ws):
        return L.focus_evict_from_importance(ctypes.byref(dd), imp, hidden, A, budget, kept, A,
                                             packed, cap, delta, A, w, None)
    assert partial(q0=None) == INVALID             # layer 0 needed for the delta score
    assert partial(q1=A + 8) == INVALID
    assert partial(imp=None) == INVALID
    assert partial(imp=A + 2) == INVALID
    assert partial(w=ws - 4) == WORKSPACE
    assert partial(dd=dims(B=129)) == UNSUPPORTED
    assert from_imp(imp=None) == INVALID
    assert from_imp(hidden=A + 8) == INVALID
    assert from_imp(budget=None) == INVALID
    assert from_imp(kept=None) == INVALID
    assert from_imp(packed=A + 8) == INVALID
    assert from_imp(cap=-1) == INVALID
    assert from_imp(delta=A + 1) == INVALID
    assert from_imp(w=8) == WORKSPACE
    assert from_imp(dd=dims(pool_window=2)) == UNSUPPORTED


def test_exchange_entry_points_validation():
    """Host checks of the peer-exchange calls (nothing is launched)."""
    d = dims()
    ws = F.focus_workspace_size(d)
    L = F._lib
    for world in (1, 2, 8):
        slots = 2 * 2 * d.R * world * d.B * 4
        assert F.focus_exchange_buffer_size(d, world) == (slots + 255) // 256 * 256 + 256
    assert L.focus_exchange_buffer_size(ctypes.byref(d), 0) == 0
    assert L.focus_exchange_buffer_size(ctypes.byref(d), 9) == 0

    def push(ex):
        return L.focus_partial_importance_push(ctypes.byref(d), A, A, A, A, A, A, A, 100,
                                               None if ex is None else ctypes.byref(ex), A, ws,
                                               None)
    assert push(None) == INVALID
    assert push(F.FocusExchange(None, 0, 2, 1)) == INVALID       # no peer array
    assert push(F.FocusExchange(A + 4, 0, 2, 1)) == INVALID      # misaligned peer array
    assert push(F.FocusExchange(A, 2, 2, 1)) == INVALID          # rank >= world
    assert push(F.FocusExchange(A, -1, 2, 1)) == INVALID
    assert push(F.FocusExchange(A, 0, 9, 1)) == INVALID          # world > 8
    assert push(F.FocusExchange(A, 0, 2, 0)) == INVALID          # epoch 0
    assert L.focus_partial_importance_push(ctypes.byref(dims(B=0)), A, A, A, A, A, A, A, 100,
                                           ctypes.byref(F.FocusExchange(A, 0, 2, 1)), A, ws,
                                           None) == INVALID

    def from_ex(buf=A, world=2, epoch=1, w=ws):
        return L.focus_evict_from_exchange(ctypes.byref(d), buf, world, epoch, A, A, A, A, A, A,
                                           16, None, A, w, None)
    assert from_ex(buf=None) == INVALID
    assert from_ex(buf=A + 16) == INVALID                        # must be 256-byte aligned
    assert from_ex(world=0) == INVALID
    assert from_ex(epoch=0) == INVALID
    assert from_ex(w=8) == WORKSPACE

    def selftest(R=4, B=32, world=2, epoch=1, ptr=A):
        return L.focus_selftest_exchange(A, ptr, A, A, R, B, world, epoch, None)
    assert selftest(ptr=None) == INVALID
    assert selftest(B=129) == INVALID
    assert selftest(world=9) == INVALID
    assert selftest(epoch=0) == INVALID
    assert selftest(R=200, world=4) == INVALID                   # too many blocks to co-reside


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "focus.h"

int main(void) {
    focus_dims_t d;
    memset(&d, 0, sizeof d);
    d.R = 4; d.B = 32; d.Hq = 32; d.Hkv = 8; d.head_dim = 128; d.hidden = 4096;
    d.softmax_scale = 0.08838834764831845f; d.pool_window = 3;
    if (focus_abi_version() != FOCUS_ABI_VERSION) return 1;
    if (focus_workspace_size(&d) == 0 || focus_exchange_buffer_size(&d, 2) == 0) return 2;
    if (strcmp(focus_status_string(FOCUS_ERR_TIMEOUT), "FOCUS_ERR_TIMEOUT") != 0) return 3;
    /* host validation only: a NULL query is rejected before anything is launched */
    if (focus_evict(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, NULL, NULL, NULL,
                    NULL, NULL, 0, NULL, NULL, NULL, NULL, 0, NULL) != FOCUS_ERR_INVALID_ARGUMENT)
        return 4;
    printf("ok %zu\n", focus_workspace_size(&d));
    return 0;
}
"""


def test_c_program_links_and_calls_the_library(tmp_path):
    """The boundary is a plain C ABI: a C99 program that includes only focus.h compiles,
    links against libfocus.so and calls it (entry points that need no GPU)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_focus.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_focus"
    libdir = os.path.dirname(F.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", HEADER_DIR,
                    str(src), "-L", libdir, "-Wl,-rpath," + libdir, "-l:libfocus.so", "-o",
                    str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("ok ")
    assert int(r.stdout.split()[1]) == F.focus_workspace_size(dims())


def test_binding_rejects_bad_tensors_before_the_library():
    """The Python binding only marshals: it refuses host tensors, wrong dtypes and
    non-contiguous views (with the argument's name) before anything reaches the C ABI."""
    d = dims(R=1, B=32, Hq=4, Hkv=2, head_dim=64, hidden=256)
    cpu = torch.zeros(4, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="q0: must be a CUDA tensor"):
        F._ptr(cpu, torch.bfloat16, "q0")
    with pytest.raises(TypeError, match="expected a torch.Tensor"):
        F._ptr([1, 2], None, "q1")
    meta = torch.empty(8, 8, dtype=torch.float32, device="meta")
    with pytest.raises(ValueError):
        F._ptr(meta, torch.float32, "delta")  # not a CUDA tensor either
    assert F._ptr(None, torch.float32, "delta_out") is None
    with pytest.raises(ValueError, match="importance must be"):
        F.focus_partial_importance(d, None, None, None, None, None, None, None,
                                   torch.zeros(3, 1, 32), None)
    with pytest.raises(ValueError, match="importance must be"):
        F.focus_evict_from_importance(d, torch.zeros(2, 2, 32), None, None, None, None, None,
                                      None, None)
    with pytest.raises(ValueError, match="one address per rank"):
        F.focus_partial_importance_push(d, None, None, None, None, None, None, None,
                                        torch.zeros(3, dtype=torch.int64), 0, 2, 1, None)
    with pytest.raises(F.FocusError):
        F.focus_exchange_buffer_size(d, 9)


def test_plan_capacity_equals_the_oracle_row_count(orc):
    """focus_plan_capacity (host arithmetic behind the C ABI): without constraints it
    equals the oracle's cu_seqlens[R] for any delta; with constraints it bounds the
    oracle's retained count; with a dynamic budget it bounds every budget the oracle
    can choose.  Budgets include negative, zero and over-large values."""
    import synth
    rng = np.random.default_rng(11)
    for cfg, R in ((1, 40), (3, 9), (4, 70)):
        p = synth.make_problem(cfg, seed=40 + cfg, overrides=dict(R=R, prefix=("fixed", 0)))
        dec = p.decoded.numpy()
        bud = rng.integers(-3, p.B + 5, size=p.R).astype(np.int32)
        pooled = np.where(dec != 0, -np.inf, rng.normal(size=dec.shape))
        _, cu, _ = orc.select(pooled, dec, bud)
        d0 = dims(R=p.R, B=p.B)
        assert F.focus_plan_capacity(d0, p.decoded, torch.from_numpy(bud)) == int(cu[-1])
        assert F.plan_capacity(p.decoded, torch.from_numpy(bud)) == int(cu[-1])
        for c in (1, 2, 3):
            _, cu_s, _ = orc.select_structured(pooled, dec, bud, c)
            cap = F.focus_plan_capacity(dims(R=p.R, B=p.B, constraints=c), p.decoded,
                                        torch.from_numpy(bud))
            assert cap >= int(cu_s[-1])
        avg = rng.uniform(0, 40, size=p.R)
        k_dyn = orc.dynamic_budget(pooled, dec, avg)
        _, cu_d, _ = orc.select(pooled, dec, k_dyn)
        assert F.focus_plan_capacity(d0, p.decoded, None, dynamic=True) >= int(cu_d[-1])
        assert F.focus_plan_capacity(d0, p.decoded, None, dynamic=True) == int((dec == 0).sum())


def test_plan_capacity_rejects_bad_arguments():
    d0 = dims(R=2, B=8)
    out = ctypes.c_int64(-1)
    dec = np.zeros((2, 8), np.uint8)
    bud = np.ones(2, np.int32)
    P = lambda a: ctypes.c_void_p(a.ctypes.data)
    assert F._lib.focus_plan_capacity(ctypes.byref(d0), None, P(bud), 0, ctypes.byref(out)) == INVALID
    assert F._lib.focus_plan_capacity(ctypes.byref(d0), P(dec), None, 0, ctypes.byref(out)) == INVALID
    assert F._lib.focus_plan_capacity(ctypes.byref(d0), P(dec), None, 1, ctypes.byref(out)) == OK
    assert out.value == 16
    assert F._lib.focus_plan_capacity(ctypes.byref(d0), P(dec), P(bud), 0, None) == INVALID
    bad = dims(R=2, B=200)
    assert F._lib.focus_plan_capacity(ctypes.byref(bad), P(dec), P(bud), 0,
                                      ctypes.byref(out)) == UNSUPPORTED
