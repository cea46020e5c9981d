"""FOCUS importance-delta token eviction on B200 (sm_100a).

A thin Python binding over the C ABI of ``libfocus.so`` (declared in
``include/focus.h``).  Every function here only checks and marshals its
arguments (torch CUDA tensors -> raw device pointers, the current CUDA stream)
and calls the C entry point of the same name; all arithmetic of the eviction
step runs in the library's CUDA kernels.  There is no CPU fallback: if the
library is missing, importing this package raises.

Method: "FOCUS: DLLMs Know How to Tame Their Compute Bound" (pith.science review
page), "What carries the argument" and the Figure 5 caption.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "FocusError", "FocusDims", "make_dims", "focus_workspace_size", "Workspace",
    "focus_clear_device_status", "focus_read_device_status", "focus_attn_stats",
    "focus_importance_delta", "focus_topk_select", "focus_compact", "focus_evict",
    "focus_status_string", "focus_abi_version", "focus_set_trace_events", "plan_capacity",
    "focus_plan_capacity",
    "focus_evict_static_scratch", "STATIC_SCRATCH_BYTES", "focus_selftest_wait_timeout",
    "focus_partial_importance", "focus_evict_from_importance", "FocusExchange",
    "focus_exchange_buffer_size", "focus_partial_importance_push", "focus_evict_from_exchange",
    "focus_selftest_exchange", "LIB_PATH", "STATUS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfocus.so")

STATUS = {
    0: "FOCUS_OK", 1: "FOCUS_ERR_INVALID_ARGUMENT", 2: "FOCUS_ERR_UNSUPPORTED_SHAPE",
    3: "FOCUS_ERR_CAPACITY", 4: "FOCUS_ERR_WORKSPACE", 5: "FOCUS_ERR_CUDA",
    6: "FOCUS_ERR_DEVICE_CHECK", 7: "FOCUS_ERR_TIMEOUT",
}


class FocusError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS.get(self.status, self.status)}")


class FocusDims(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int32), ("B", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("pool_window", ctypes.c_int32),
                ("constraints", ctypes.c_int32), ("score", ctypes.c_int32)]


KEEP_PREDECESSOR = 1               # retain each candidate's immediate predecessor
KEEP_MASKED_BEFORE_RIGHTMOST = 2   # retain masked tokens left of the rightmost candidate
SCORE_DELTA = 0                    # rank by I1 - I0 (the method)
SCORE_LAYER1 = 1                   # rank by I1 alone (Figure 13 ablation; layer 0 skipped)


class FocusEvictArgs(ctypes.Structure):
    """Mirror of focus_evict_args_t (include/focus.h)."""
    _fields_ = [("q0", ctypes.c_void_p), ("k0_prefix", ctypes.c_void_p),
                ("k0_block", ctypes.c_void_p), ("lse0", ctypes.c_void_p),
                ("q1", ctypes.c_void_p), ("k1_prefix", ctypes.c_void_p),
                ("k1_block", ctypes.c_void_p), ("cu_prefix", ctypes.c_void_p),
                ("total_prefix", ctypes.c_int64), ("page_table", ctypes.c_void_p),
                ("prefix_len", ctypes.c_void_p), ("max_pages", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("hidden", ctypes.c_void_p), ("decoded", ctypes.c_void_p),
                ("budget", ctypes.c_void_p), ("decode_avg", ctypes.c_void_p),
                ("budget_alpha", ctypes.c_float), ("budget_out", ctypes.c_void_p),
                ("kept_idx", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p),
                ("packed", ctypes.c_void_p), ("capacity", ctypes.c_int64),
                ("delta_out", ctypes.c_void_p), ("i0_out", ctypes.c_void_p),
                ("i1_out", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("stream", ctypes.c_void_p)]


class FocusExchange(ctypes.Structure):
    """focus_exchange_t: peer_buffers is a DEVICE array of the ranks' buffer pointers."""
    _fields_ = [("peer_buffers", ctypes.c_void_p), ("rank", ctypes.c_int32),
                ("world", ctypes.c_int32), ("epoch", ctypes.c_uint32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with `python attention_delta_token_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    D = ctypes.POINTER(FocusDims)
    sig = {
        "focus_workspace_size": (sz, [D]),
        "focus_plan_capacity": (ctypes.c_int, [D, P, P, ctypes.c_int, ctypes.POINTER(i64)]),
        "focus_clear_device_status": (ctypes.c_int, [P, sz, P]),
        "focus_read_device_status": (ctypes.c_int, [P, P, ctypes.c_int]),
        "focus_attn_stats": (ctypes.c_int, [D, P, P, P, i64, P, P, P, sz, P]),
        "focus_importance_delta": (ctypes.c_int, [D, P, P, P, P, P, P]),
        "focus_topk_select": (ctypes.c_int, [D, P, P, P, P, P, i64, P, sz, P]),
        "focus_compact": (ctypes.c_int, [D, P, P, P, P, i64, P, sz, P]),
        "focus_evict": (ctypes.c_int, [D, P, P, P, P, P, P, P, i64, P, P, P, P, P, P, i64,
                                       P, P, P, P, sz, P]),
        "focus_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "focus_abi_version": (ctypes.c_int, []),
        "focus_set_trace_events": (None, [P, P]),
        "focus_evict_static_scratch": (ctypes.c_int, [D, P, P, P, P, P, P, P, i64, P, P, P, P, P,
                                                      P, i64, P, P, P, P, P]),
        "focus_selftest_wait_timeout": (ctypes.c_int, [P, ctypes.c_uint64, P, P]),
        "focus_evict_with_lse0": (ctypes.c_int, [D, P, P, P, P, P, P, P, i64, P, P, P, P, P, P,
                                                 i64, P, P, P, P, sz, P]),
        "focus_evict_ex": (ctypes.c_int, [D, ctypes.POINTER(FocusEvictArgs)]),
        "focus_partial_importance": (ctypes.c_int, [D, P, P, P, P, P, P, P, i64, P, P, sz, P]),
        "focus_evict_from_importance": (ctypes.c_int, [D, P, P, P, P, P, P, P, i64, P, P, sz, P]),
        "focus_exchange_buffer_size": (sz, [D, ctypes.c_int32]),
        "focus_partial_importance_push": (ctypes.c_int, [D, P, P, P, P, P, P, P, i64,
                                                         ctypes.POINTER(FocusExchange), P, sz, P]),
        "focus_evict_from_exchange": (ctypes.c_int, [D, P, ctypes.c_int32, ctypes.c_uint32, P, P,
                                                     P, P, P, P, i64, P, P, sz, P]),
        "focus_selftest_exchange": (ctypes.c_int, [P, P, P, P, ctypes.c_int32, ctypes.c_int32,
                                                   ctypes.c_int32, ctypes.c_uint32, P]),
        "focus_evict_paged": (ctypes.c_int, [D, P, P, P, P, P, P, P, ctypes.c_int32, P,
                                             ctypes.c_int32, ctypes.c_int32, P, P, P, P, P, P, i64,
                                             P, P, P, P, sz, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def make_dims(R, B, Hq, Hkv, head_dim, hidden, softmax_scale=None, pool_window=3,
              constraints=0, score=SCORE_DELTA) -> FocusDims:
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(head_dim)
    return FocusDims(int(R), int(B), int(Hq), int(Hkv), int(head_dim), int(hidden),
                     float(softmax_scale), int(pool_window), int(constraints), int(score))


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return ctypes.c_void_p(t.data_ptr()) if t.numel() else None


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ok(st: int, where: str):
    if st != 0:
        raise FocusError(st, where)


def focus_status_string(status: int) -> str:
    return _lib.focus_status_string(int(status)).decode()


def focus_abi_version() -> int:
    return int(_lib.focus_abi_version())


def focus_set_trace_events(start=None, stop=None):
    """Record the torch.cuda.Event pair `start`/`stop` around the attention-statistics
    kernel of every later focus_evict / focus_attn_stats call (None, None: off)."""
    if start is None or stop is None:
        _lib.focus_set_trace_events(None, None)
        return
    for e in (start, stop):
        if e.cuda_event == 0:  # torch creates the CUDA event lazily
            e.record()
    _lib.focus_set_trace_events(ctypes.c_void_p(start.cuda_event), ctypes.c_void_p(stop.cuda_event))


def focus_workspace_size(dims: FocusDims) -> int:
    n = int(_lib.focus_workspace_size(ctypes.byref(dims)))
    if n == 0:
        raise FocusError(2, "focus_workspace_size")
    return n


class Workspace:
    """Device scratch for one stream of calls (status word, request order, column sums)."""

    @staticmethod
    def size(dims: FocusDims) -> int:
        return focus_workspace_size(dims)

    def __init__(self, dims: FocusDims, device="cuda", stream=None):
        self.nbytes = focus_workspace_size(dims)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        focus_clear_device_status(self, stream)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


def focus_clear_device_status(ws: Workspace, stream=None):
    _ok(_lib.focus_clear_device_status(ws.ptr, ws.nbytes, _stream(stream)),
        "focus_clear_device_status")


def focus_read_device_status(ws: Workspace, stream=None, timeout_ms: int = 10000) -> int:
    """Synchronises with `stream` and returns the device status code (0 = FOCUS_OK)."""
    return int(_lib.focus_read_device_status(ws.ptr, _stream(stream), int(timeout_ms)))


def focus_attn_stats(dims, q, k_prefix, cu_prefix, k_block, importance, ws: Workspace,
                     stream=None):
    bf = torch.bfloat16
    _ok(_lib.focus_attn_stats(
        ctypes.byref(dims), _ptr(q, bf, "q"), _ptr(k_prefix, bf, "k_prefix"),
        _ptr(cu_prefix, torch.int32, "cu_prefix"), int(k_prefix.shape[0]),
        _ptr(k_block, bf, "k_block"), _ptr(importance, torch.float32, "importance"),
        ws.ptr, ws.nbytes, _stream(stream)), "focus_attn_stats")


def focus_importance_delta(dims, i0, i1, decoded, delta, raw_delta=None, stream=None):
    f32 = torch.float32
    _ok(_lib.focus_importance_delta(
        ctypes.byref(dims), _ptr(i0, f32, "i0"), _ptr(i1, f32, "i1"),
        _ptr(decoded, torch.uint8, "decoded"), _ptr(delta, f32, "delta"),
        _ptr(raw_delta, f32, "raw_delta"), _stream(stream)), "focus_importance_delta")


def focus_topk_select(dims, delta, decoded, budget, kept_idx, cu_seqlens, ws: Workspace,
                      stream=None):
    _ok(_lib.focus_topk_select(
        ctypes.byref(dims), _ptr(delta, torch.float32, "delta"),
        _ptr(decoded, torch.uint8, "decoded"), _ptr(budget, torch.int32, "budget"),
        _ptr(kept_idx, torch.int32, "kept_idx"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        int(kept_idx.numel()), ws.ptr, ws.nbytes, _stream(stream)), "focus_topk_select")


def focus_compact(dims, hidden, kept_idx, cu_seqlens, packed, ws: Workspace, stream=None):
    bf = torch.bfloat16
    _ok(_lib.focus_compact(
        ctypes.byref(dims), _ptr(hidden, bf, "hidden"), _ptr(kept_idx, torch.int32, "kept_idx"),
        _ptr(cu_seqlens, torch.int32, "cu_seqlens"), _ptr(packed, bf, "packed"),
        int(packed.shape[0]), ws.ptr, ws.nbytes, _stream(stream)), "focus_compact")


def focus_evict(dims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block, cu_prefix, hidden,
                decoded, budget, kept_idx, cu_seqlens, packed, ws: Workspace, delta_out=None,
                i0_out=None, i1_out=None, stream=None):
    bf, f32 = torch.bfloat16, torch.float32
    if k0_prefix is not None and k0_prefix.shape[0] != k1_prefix.shape[0]:
        raise ValueError("k0_prefix and k1_prefix must have the same number of rows")
    _ok(_lib.focus_evict(
        ctypes.byref(dims), _ptr(q0, bf, "q0"), _ptr(k0_prefix, bf, "k0_prefix"),
        _ptr(k0_block, bf, "k0_block"), _ptr(q1, bf, "q1"), _ptr(k1_prefix, bf, "k1_prefix"),
        _ptr(k1_block, bf, "k1_block"), _ptr(cu_prefix, torch.int32, "cu_prefix"),
        int(k1_prefix.shape[0]), _ptr(hidden, bf, "hidden"),
        _ptr(decoded, torch.uint8, "decoded"), _ptr(budget, torch.int32, "budget"),
        _ptr(kept_idx, torch.int32, "kept_idx"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        _ptr(packed, bf, "packed"), int(packed.shape[0]),
        _ptr(delta_out, f32, "delta_out"), _ptr(i0_out, f32, "i0_out"),
        _ptr(i1_out, f32, "i1_out"), ws.ptr, ws.nbytes, _stream(stream)), "focus_evict")


def focus_partial_importance(dims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block, cu_prefix,
                             importance, ws: Workspace, stream=None):
    """Both layers' importance over the heads in `dims` into importance [2, R, B] float32
    (I0, I1); the first half of focus_evict, for head-sharded (tensor-parallel) ranks."""
    bf = torch.bfloat16
    if importance.shape != (2, dims.R, dims.B):
        raise ValueError(f"importance must be [2, {dims.R}, {dims.B}]")
    _ok(_lib.focus_partial_importance(
        ctypes.byref(dims), _ptr(q0, bf, "q0"), _ptr(k0_prefix, bf, "k0_prefix"),
        _ptr(k0_block, bf, "k0_block"), _ptr(q1, bf, "q1"), _ptr(k1_prefix, bf, "k1_prefix"),
        _ptr(k1_block, bf, "k1_block"), _ptr(cu_prefix, torch.int32, "cu_prefix"),
        int(k1_prefix.shape[0]), _ptr(importance, torch.float32, "importance"), ws.ptr,
        ws.nbytes, _stream(stream)), "focus_partial_importance")


def focus_evict_from_importance(dims, importance, hidden, decoded, budget, kept_idx, cu_seqlens,
                                packed, ws: Workspace, delta_out=None, stream=None):
    """Delta, MaxPool1D, mask, top-K and compaction from importance [2, R, B] float32; the
    second half of focus_evict."""
    bf = torch.bfloat16
    if importance.shape != (2, dims.R, dims.B):
        raise ValueError(f"importance must be [2, {dims.R}, {dims.B}]")
    _ok(_lib.focus_evict_from_importance(
        ctypes.byref(dims), _ptr(importance, torch.float32, "importance"),
        _ptr(hidden, bf, "hidden"), _ptr(decoded, torch.uint8, "decoded"),
        _ptr(budget, torch.int32, "budget"), _ptr(kept_idx, torch.int32, "kept_idx"),
        _ptr(cu_seqlens, torch.int32, "cu_seqlens"), _ptr(packed, bf, "packed"),
        int(packed.shape[0]), _ptr(delta_out, torch.float32, "delta_out"), ws.ptr, ws.nbytes,
        _stream(stream)), "focus_evict_from_importance")


def focus_exchange_buffer_size(dims, world: int) -> int:
    n = int(_lib.focus_exchange_buffer_size(ctypes.byref(dims), int(world)))
    if n == 0:
        raise FocusError(1, "focus_exchange_buffer_size (invalid dims or world)")
    return n


def focus_partial_importance_push(dims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block,
                                  cu_prefix, peer_buffers, rank: int, world: int, epoch: int,
                                  ws: Workspace, stream=None):
    """focus_partial_importance whose [2, R, B] sums go to slot `rank` of every rank's exchange
    buffer; peer_buffers: int64 CUDA tensor [world] of the buffers' device addresses."""
    bf = torch.bfloat16
    if peer_buffers.numel() != world:
        raise ValueError("peer_buffers must hold one address per rank")
    ex = FocusExchange(_ptr(peer_buffers, torch.int64, "peer_buffers"), int(rank), int(world),
                       int(epoch))
    _ok(_lib.focus_partial_importance_push(
        ctypes.byref(dims), _ptr(q0, bf, "q0"), _ptr(k0_prefix, bf, "k0_prefix"),
        _ptr(k0_block, bf, "k0_block"), _ptr(q1, bf, "q1"), _ptr(k1_prefix, bf, "k1_prefix"),
        _ptr(k1_block, bf, "k1_block"), _ptr(cu_prefix, torch.int32, "cu_prefix"),
        int(k1_prefix.shape[0]), ctypes.byref(ex), ws.ptr, ws.nbytes, _stream(stream)),
        "focus_partial_importance_push")


def focus_evict_from_exchange(dims, exchange_buffer, world: int, epoch: int, hidden, decoded,
                              budget, kept_idx, cu_seqlens, packed, ws: Workspace,
                              delta_out=None, stream=None):
    """focus_evict_from_importance on the rank-ordered sum of this rank's exchange buffer
    (uint8 CUDA tensor of focus_exchange_buffer_size bytes) for `epoch`."""
    bf = torch.bfloat16
    _ok(_lib.focus_evict_from_exchange(
        ctypes.byref(dims), _ptr(exchange_buffer, torch.uint8, "exchange_buffer"), int(world),
        int(epoch), _ptr(hidden, bf, "hidden"), _ptr(decoded, torch.uint8, "decoded"),
        _ptr(budget, torch.int32, "budget"), _ptr(kept_idx, torch.int32, "kept_idx"),
        _ptr(cu_seqlens, torch.int32, "cu_seqlens"), _ptr(packed, bf, "packed"),
        int(packed.shape[0]), _ptr(delta_out, torch.float32, "delta_out"), ws.ptr, ws.nbytes,
        _stream(stream)), "focus_evict_from_exchange")


def focus_selftest_exchange(partials, buffer_ptrs, out, scratch, epoch: int, stream=None):
    """The exchange protocol with world = partials.shape[0] ranks emulated in one cooperative
    launch (see focus.h).  partials/out [world, 2, R, B] float32, buffer_ptrs int64 [world],
    scratch int32/uint32-sized zeroed [>= 1 + world] (scratch[0] = status bits)."""
    world, _, R, B = partials.shape
    _ok(_lib.focus_selftest_exchange(
        _ptr(partials, torch.float32, "partials"), _ptr(buffer_ptrs, torch.int64, "buffer_ptrs"),
        _ptr(out, torch.float32, "out"), _ptr(scratch, torch.int32, "scratch"), int(R), int(B),
        int(world), int(epoch), _stream(stream)), "focus_selftest_exchange")


def focus_evict_with_lse0(dims, lse0, q0, k0_block, q1, k1_prefix, k1_block, cu_prefix, hidden,
                          decoded, budget, kept_idx, cu_seqlens, packed, ws: Workspace,
                          delta_out=None, i0_out=None, i1_out=None, stream=None):
    """focus_evict with layer 0's row log-sum-exps given (lse0 [R, B, Hq] float32, natural
    log, over each row's prefix and block keys): layer 0 reads only Q0 and its block keys."""
    bf, f32 = torch.bfloat16, torch.float32
    _ok(_lib.focus_evict_with_lse0(
        ctypes.byref(dims), _ptr(lse0, f32, "lse0"), _ptr(q0, bf, "q0"),
        _ptr(k0_block, bf, "k0_block"), _ptr(q1, bf, "q1"), _ptr(k1_prefix, bf, "k1_prefix"),
        _ptr(k1_block, bf, "k1_block"), _ptr(cu_prefix, torch.int32, "cu_prefix"),
        int(k1_prefix.shape[0]), _ptr(hidden, bf, "hidden"),
        _ptr(decoded, torch.uint8, "decoded"), _ptr(budget, torch.int32, "budget"),
        _ptr(kept_idx, torch.int32, "kept_idx"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        _ptr(packed, bf, "packed"), int(packed.shape[0]),
        _ptr(delta_out, f32, "delta_out"), _ptr(i0_out, f32, "i0_out"),
        _ptr(i1_out, f32, "i1_out"), ws.ptr, ws.nbytes, _stream(stream)), "focus_evict_with_lse0")


def focus_evict_paged(dims, q0, k0_pages, k0_block, q1, k1_pages, k1_block, page_table,
                      prefix_len, hidden, decoded, budget, kept_idx, cu_seqlens, packed,
                      ws: Workspace, delta_out=None, i0_out=None, i1_out=None, stream=None):
    """focus_evict with the prefix keys in page pools k*_pages [num_pages, page_size, Hkv, d]
    addressed through page_table [R, max_pages] int32 and prefix_len [R] int32."""
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    if k0_pages.shape != k1_pages.shape:
        raise ValueError("both layers' page pools must have the same shape")
    _ok(_lib.focus_evict_paged(
        ctypes.byref(dims), _ptr(q0, bf, "q0"), _ptr(k0_pages, bf, "k0_pages"),
        _ptr(k0_block, bf, "k0_block"), _ptr(q1, bf, "q1"), _ptr(k1_pages, bf, "k1_pages"),
        _ptr(k1_block, bf, "k1_block"), _ptr(page_table, i32, "page_table"),
        int(page_table.shape[1]), _ptr(prefix_len, i32, "prefix_len"), int(k0_pages.shape[0]),
        int(k0_pages.shape[1]), _ptr(hidden, bf, "hidden"),
        _ptr(decoded, torch.uint8, "decoded"), _ptr(budget, i32, "budget"),
        _ptr(kept_idx, i32, "kept_idx"), _ptr(cu_seqlens, i32, "cu_seqlens"),
        _ptr(packed, bf, "packed"), int(packed.shape[0]),
        _ptr(delta_out, f32, "delta_out"), _ptr(i0_out, f32, "i0_out"),
        _ptr(i1_out, f32, "i1_out"), ws.ptr, ws.nbytes, _stream(stream)), "focus_evict_paged")


def focus_evict_ex(dims, *, q1, k1_prefix, k1_block, hidden, decoded, kept_idx, cu_seqlens,
                   packed, ws: Workspace, q0=None, k0_prefix=None, k0_block=None, lse0=None,
                   cu_prefix=None, page_table=None, prefix_len=None, budget=None,
                   decode_avg=None, budget_alpha=1.5, budget_out=None, delta_out=None,
                   i0_out=None, i1_out=None, stream=None):
    """The fused step with every option (focus_evict_ex).  Packed prefix: pass cu_prefix;
    paged prefix: pass page_table and prefix_len (k*_prefix are then page pools);
    lse0: layer-0 row log-sum-exps; decode_avg: dynamic budget (budget then unused)."""
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    a = FocusEvictArgs()
    a.q0, a.k0_prefix, a.k0_block = _ptr(q0, bf, "q0"), _ptr(k0_prefix, bf, "k0_prefix"), \
        _ptr(k0_block, bf, "k0_block")
    a.lse0 = _ptr(lse0, f32, "lse0")
    a.q1, a.k1_prefix, a.k1_block = _ptr(q1, bf, "q1"), _ptr(k1_prefix, bf, "k1_prefix"), \
        _ptr(k1_block, bf, "k1_block")
    if page_table is not None:
        a.page_table = _ptr(page_table, i32, "page_table")
        a.prefix_len = _ptr(prefix_len, i32, "prefix_len")
        a.max_pages = int(page_table.shape[1])
        a.num_pages, a.page_size = int(k1_prefix.shape[0]), int(k1_prefix.shape[1])
    else:
        a.cu_prefix = _ptr(cu_prefix, i32, "cu_prefix")
        a.total_prefix = int(k1_prefix.shape[0])
    a.hidden = _ptr(hidden, bf, "hidden")
    a.decoded = _ptr(decoded, torch.uint8, "decoded")
    a.budget = _ptr(budget, i32, "budget")
    a.decode_avg = _ptr(decode_avg, f32, "decode_avg")
    a.budget_alpha = float(budget_alpha)
    a.budget_out = _ptr(budget_out, i32, "budget_out")
    a.kept_idx = _ptr(kept_idx, i32, "kept_idx")
    a.cu_seqlens = _ptr(cu_seqlens, i32, "cu_seqlens")
    a.packed = _ptr(packed, bf, "packed")
    a.capacity = int(packed.shape[0])
    a.delta_out, a.i0_out, a.i1_out = _ptr(delta_out, f32, "delta_out"), \
        _ptr(i0_out, f32, "i0_out"), _ptr(i1_out, f32, "i1_out")
    a.workspace, a.workspace_bytes = ws.ptr, ws.nbytes
    a.stream = _stream(stream)
    _ok(_lib.focus_evict_ex(ctypes.byref(dims), ctypes.byref(a)), "focus_evict_ex")


STATIC_SCRATCH_BYTES = 8 << 20


def focus_evict_static_scratch(dims, q0, k0_prefix, k0_block, q1, k1_prefix, k1_block, cu_prefix,
                               hidden, decoded, budget, kept_idx, cu_seqlens, packed,
                               device_status=None, delta_out=None, i0_out=None, i1_out=None,
                               stream=None):
    """focus_evict without a workspace argument, for callers that cannot allocate:
    the scratch is the library's own fixed device array (STATIC_SCRATCH_BYTES).
    `device_status` (optional int32 CUDA tensor of one element) receives the raw
    device status bits (0 = fine)."""
    bf, f32 = torch.bfloat16, torch.float32
    if k0_prefix is not None and k0_prefix.shape[0] != k1_prefix.shape[0]:
        raise ValueError("k0_prefix and k1_prefix must have the same number of rows")
    _ok(_lib.focus_evict_static_scratch(
        ctypes.byref(dims), _ptr(q0, bf, "q0"), _ptr(k0_prefix, bf, "k0_prefix"),
        _ptr(k0_block, bf, "k0_block"), _ptr(q1, bf, "q1"), _ptr(k1_prefix, bf, "k1_prefix"),
        _ptr(k1_block, bf, "k1_block"), _ptr(cu_prefix, torch.int32, "cu_prefix"),
        int(k1_prefix.shape[0]), _ptr(hidden, bf, "hidden"),
        _ptr(decoded, torch.uint8, "decoded"), _ptr(budget, torch.int32, "budget"),
        _ptr(kept_idx, torch.int32, "kept_idx"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
        _ptr(packed, bf, "packed"), int(packed.shape[0]),
        _ptr(delta_out, f32, "delta_out"), _ptr(i0_out, f32, "i0_out"),
        _ptr(i1_out, f32, "i1_out"), _ptr(device_status, torch.int32, "device_status"),
        _stream(stream)), "focus_evict_static_scratch")


def focus_selftest_wait_timeout(status, elapsed_ns, limit_ns: int, stream=None):
    """Runs the bounded wait on a barrier that never completes (see include/focus.h).
    `status`: int32 CUDA tensor [1]; `elapsed_ns`: int64 CUDA tensor [1]."""
    _ok(_lib.focus_selftest_wait_timeout(_ptr(status, torch.int32, "status"), int(limit_ns),
                                         _ptr(elapsed_ns, torch.int64, "elapsed_ns"),
                                         _stream(stream)), "focus_selftest_wait_timeout")


def focus_plan_capacity(dims: FocusDims, decoded, budget=None, dynamic: bool = False) -> int:
    """Rows the packed batch needs (the C entry point of the same name): the kept count
    of every request from the scheduler's `decoded` [R, B] uint8 and `budget` [R] int32,
    exact without structural constraints, an upper bound with them (see focus.h).
    Tensors on any device; they are copied to host memory, which the call reads."""
    dec = decoded.detach().to("cpu", torch.uint8).contiguous()
    if tuple(dec.shape) != (dims.R, dims.B):
        raise ValueError(f"decoded must be [{dims.R}, {dims.B}]")
    bud = None
    if not dynamic:
        bud = budget.detach().to("cpu", torch.int32).contiguous()
        if tuple(bud.shape) != (dims.R,):
            raise ValueError(f"budget must be [{dims.R}]")
    out = ctypes.c_int64(-1)
    _ok(_lib.focus_plan_capacity(ctypes.byref(dims), ctypes.c_void_p(dec.data_ptr()),
                                 ctypes.c_void_p(bud.data_ptr()) if bud is not None else None,
                                 int(bool(dynamic)), ctypes.byref(out)), "focus_plan_capacity")
    return int(out.value)


def plan_capacity(decoded, budget, constraints: int = 0, dynamic: bool = False) -> int:
    """focus_plan_capacity for a batch described only by its arrays (the dims it needs
    are R, B and the constraint bits; the other fields are placeholders)."""
    R, B = int(decoded.shape[0]), int(decoded.shape[1])
    dims = make_dims(R, B, 1, 1, 64, 8, 1.0, 1, constraints)
    return focus_plan_capacity(dims, decoded, budget, dynamic)
