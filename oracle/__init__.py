"""float64 CPU oracle for FOCUS importance-delta token eviction.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
(``attention_delta_token_b200``) never imports it and shares no code with it.

The arithmetic lives in ``focus_oracle.c`` (plain C, float64, OpenMP over
requests).  This module only builds that file with gcc and marshals numpy
arrays into it.  bf16 tensors cross as their raw 16-bit patterns.

Method source: "FOCUS: DLLMs Know How to Tame Their Compute Bound" (pith.science
review page), "What carries the argument" (I_j, the importance delta of Eq. 3,
MaxPool1D, top-K under a budget); Referee Report, minor comment on Eq. (2)
(row softmax); Free-Parameter Ledger (MaxPool1D k = 3, Eq. 15); Figure 5 caption
(eviction after the layer-1 Q/K projections).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "focus_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libfocus_oracle.so")
_lock = threading.Lock()

OK, BAD_ARGUMENT, NO_MEMORY, CAPACITY = 0, 1, 2, 3


class OracleError(RuntimeError):
    pass


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile an oracle C source into a shared library (gcc, -fopenmp)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _u16(a) -> np.ndarray:
    """Raw bf16 bit patterns as a contiguous uint16 array (torch bf16 or numpy uint16)."""
    if hasattr(a, "detach"):  # torch tensor
        import torch
        a = a.detach().to("cpu").contiguous()
        assert a.dtype == torch.bfloat16, a.dtype
        return a.view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _arr(a, dtype) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a.size else ctypes.c_void_p(0)


def _check(st: int, what: str, allow_capacity: bool = False):
    if st == OK or (allow_capacity and st == CAPACITY):
        return st
    raise OracleError(f"{what}: oracle status {st}")


class Oracle:
    """The oracle's entry points, bound to one compiled library.

    ``Oracle()`` uses focus_oracle.c as committed; tests may bind a library
    built from a deliberately mutated copy to show that the pins catch it.
    """

    def __init__(self, lib_path: str | None = None):
        lib = ctypes.CDLL(lib_path or build())
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.focus_oracle_importance.argtypes = [i32, i32, i32, i32, i32, f64, P, P, P, P, P]
        lib.focus_oracle_delta.argtypes = [i32, i32, i32, P, P, P, P, P]
        lib.focus_oracle_select.argtypes = [i32, i32, P, P, P, P, P, i64]
        lib.focus_oracle_compact.argtypes = [i32, i32, i32, P, P, P, P, i64]
        lib.focus_oracle_select_structured.argtypes = [i32, i32, P, P, P, i32, P, P, i64]
        lib.focus_oracle_importance_lse.argtypes = [i32, i32, i32, i32, i32, f64, P, P, P, P]
        lib.focus_oracle_importance_paged.argtypes = [i32, i32, i32, i32, i32, f64, P, P, P, i32,
                                                      P, i32, i32, P, P]
        lib.focus_oracle_dynamic_budget.argtypes = [i32, i32, P, P, P, f64, P]
        lib.focus_oracle_num_threads.argtypes = []
        lib.focus_oracle_set_num_threads.argtypes = [i32]
        for fn in (lib.focus_oracle_importance, lib.focus_oracle_delta, lib.focus_oracle_select,
                   lib.focus_oracle_compact, lib.focus_oracle_num_threads,
                   lib.focus_oracle_select_structured, lib.focus_oracle_importance_lse,
                   lib.focus_oracle_importance_paged, lib.focus_oracle_dynamic_budget,
                   lib.focus_oracle_set_num_threads):
            fn.restype = ctypes.c_int
        self.lib = lib

    def num_threads(self) -> int:
        return int(self.lib.focus_oracle_num_threads())

    def set_num_threads(self, n: int) -> int:
        """Threads of the later calls (timing only: results do not depend on it)."""
        return int(self.lib.focus_oracle_set_num_threads(int(n)))

    def importance(self, q, k_prefix, cu_prefix, k_block, *, Hq: int, Hkv: int,
                   scale: float) -> np.ndarray:
        """I[r, j] (float64) of one layer.  q [R,B,Hq,d], k_prefix [sum L,Hkv,d], k_block [R,B,Hkv,d]."""
        qa, kp, kb = _u16(q), _u16(k_prefix), _u16(k_block)
        cu = _arr(cu_prefix, np.int32)
        R, B, hq, d = qa.shape
        assert hq == Hq and kb.shape == (R, B, Hkv, d) and cu.shape == (R + 1,)
        assert int(cu[0]) == 0 and (int(cu[-1]) == 0 or int(cu[-1]) <= kp.shape[0])
        if kp.size == 0:
            kp = np.zeros((1,), np.uint16)
        out = np.zeros((R, B), np.float64)
        st = self.lib.focus_oracle_importance(R, B, Hq, Hkv, d, float(scale), _p(qa), _p(kp),
                                              _p(cu), _p(kb), _p(out))
        _check(st, "importance")
        return out

    def importance_paged(self, q, k_pages, page_table, prefix_len, k_block, *, Hq: int, Hkv: int,
                         scale: float) -> np.ndarray:
        """I[r, j] with the prefix keys in a page pool k_pages [num_pages, page_size, Hkv, d]
        addressed through page_table [R, max_pages] and prefix_len [R]."""
        qa, kp, kb = _u16(q), _u16(k_pages), _u16(k_block)
        pt = _arr(page_table, np.int32)
        pl = _arr(prefix_len, np.int32)
        R, B, hq, d = qa.shape
        num_pages, page_size = kp.shape[0], kp.shape[1]
        assert hq == Hq and kb.shape == (R, B, Hkv, d) and pt.shape[0] == R and pl.shape == (R,)
        out = np.zeros((R, B), np.float64)
        st = self.lib.focus_oracle_importance_paged(R, B, Hq, Hkv, d, float(scale), _p(qa), _p(kp),
                                                    _p(pt), pt.shape[1], _p(pl), page_size,
                                                    num_pages, _p(kb), _p(out))
        _check(st, "importance_paged")
        return out

    def importance_lse(self, q, k_block, lse, *, Hq: int, Hkv: int, scale: float) -> np.ndarray:
        """I[r, j] from given row log-sum-exps lse [R, B, Hq]: only the block keys are read."""
        qa, kb = _u16(q), _u16(k_block)
        ls = _arr(lse, np.float64)
        R, B, hq, d = qa.shape
        assert hq == Hq and kb.shape == (R, B, Hkv, d) and ls.shape == (R, B, Hq)
        out = np.zeros((R, B), np.float64)
        st = self.lib.focus_oracle_importance_lse(R, B, Hq, Hkv, d, float(scale), _p(qa), _p(kb),
                                                  _p(ls), _p(out))
        _check(st, "importance_lse")
        return out

    def delta_pool_mask(self, i0, i1, decoded, *, window: int = 3):
        """(raw delta, pooled-and-masked delta), both float64 [R, B]."""
        a0, a1 = _arr(i0, np.float64), _arr(i1, np.float64)
        dec = _arr(decoded, np.uint8)
        R, B = a0.shape
        raw = np.empty((R, B), np.float64)
        pooled = np.empty((R, B), np.float64)
        st = self.lib.focus_oracle_delta(R, B, int(window), _p(a0), _p(a1), _p(dec), _p(raw),
                                         _p(pooled))
        _check(st, "delta")
        return raw, pooled

    def select(self, pooled, decoded, budget, *, capacity: int | None = None):
        """(kept positions [capacity] int32, cu_seqlens [R+1] int32, status).

        With ``capacity=None`` the buffer is sized to hold every row the
        oracle selects (B rows per request, an upper bound)."""
        pv = _arr(pooled, np.float64)
        dec = _arr(decoded, np.uint8)
        bud = _arr(budget, np.int32)
        R, B = pv.shape
        cap = R * B if capacity is None else int(capacity)
        kept = np.full((max(cap, 1),), -1, np.int32)
        cu = np.zeros((R + 1,), np.int32)
        st = self.lib.focus_oracle_select(R, B, _p(pv), _p(dec), _p(bud), _p(kept), _p(cu), cap)
        _check(st, "select", allow_capacity=True)
        n = min(cap, int(cu[-1]))
        return kept[:n], cu, st

    def select_structured(self, pooled, decoded, budget, constraints: int, *,
                          capacity: int | None = None):
        """Top-k candidates plus the structural constraints (bit 1: each candidate's
        predecessor; bit 2: masked tokens before the rightmost candidate).
        Returns (kept [n] int32, cu_seqlens [R+1] int32, status)."""
        pv = _arr(pooled, np.float64)
        dec = _arr(decoded, np.uint8)
        bud = _arr(budget, np.int32)
        R, B = pv.shape
        cap = R * B if capacity is None else int(capacity)
        kept = np.full((max(cap, 1),), -1, np.int32)
        cu = np.zeros((R + 1,), np.int32)
        st = self.lib.focus_oracle_select_structured(R, B, _p(pv), _p(dec), _p(bud),
                                                     int(constraints), _p(kept), _p(cu), cap)
        _check(st, "select_structured", allow_capacity=True)
        return kept[:min(cap, int(cu[-1]))], cu, st

    def dynamic_budget(self, pooled, decoded, decode_avg, alpha: float = 1.5) -> np.ndarray:
        """K_r from the historical yield and the masked-delta mean + std (see the C source)."""
        pv = _arr(pooled, np.float64)
        dec = _arr(decoded, np.uint8)
        avg = _arr(decode_avg, np.float64)
        R, B = pv.shape
        out = np.zeros((R,), np.int32)
        st = self.lib.focus_oracle_dynamic_budget(R, B, _p(pv), _p(dec), _p(avg), float(alpha),
                                                  _p(out))
        _check(st, "dynamic_budget")
        return out

    def compact(self, hidden, kept, cu_seqlens, *, capacity: int | None = None) -> np.ndarray:
        """packed [capacity, H] uint16 (bf16 bits) of the kept hidden rows."""
        hid = _u16(hidden)
        R, B, H = hid.shape
        k = _arr(kept, np.int32)
        cu = _arr(cu_seqlens, np.int32)
        if capacity is None:
            capacity = int(cu[-1])
        packed = np.zeros((max(capacity, 1), H), np.uint16)
        st = self.lib.focus_oracle_compact(R, B, H, _p(hid), _p(k), _p(cu), _p(packed),
                                           int(capacity))
        _check(st, "compact")
        return packed[:capacity]

    def evict(self, p, constraints: int = 0, score: int = 0, lse0=None, decode_avg=None,
              alpha: float = 1.5) -> dict:
        """The whole step on a problem object with the fields of ``synth.FocusProblem``.

        Returns float64 i0, i1, delta (raw), pooled (masked) [R, B]; int32 kept
        and cu_seqlens; uint16 packed [sum k, H].  With ``score=1`` (rank by the
        layer-1 importance alone) the layer-0 importance is taken as zero, so the
        pooled score is MaxPool1D(I1).  With ``lse0`` ([R, B, Hq] row log-sum-exps of
        layer 0) the layer-0 importance is taken from it (``importance_lse``).
        """
        if score:
            i0 = np.zeros((p.R, p.B), np.float64)
        elif lse0 is not None:
            i0 = self.importance_lse(p.q0, p.k0_block, lse0, Hq=p.Hq, Hkv=p.Hkv, scale=p.scale)
        else:
            i0 = self.importance(p.q0, p.k0_prefix, p.cu_prefix, p.k0_block, Hq=p.Hq,
                                 Hkv=p.Hkv, scale=p.scale)
        i1 = self.importance(p.q1, p.k1_prefix, p.cu_prefix, p.k1_block, Hq=p.Hq, Hkv=p.Hkv,
                             scale=p.scale)
        raw, pooled = self.delta_pool_mask(i0, i1, p.decoded, window=p.pool_window)
        budget = p.budget
        if decode_avg is not None:  # dynamic budget (Eq. 4 as read)
            budget = self.dynamic_budget(pooled, p.decoded, decode_avg, alpha)
        if constraints:
            kept, cu, st = self.select_structured(pooled, p.decoded, budget, constraints)
        else:
            kept, cu, st = self.select(pooled, p.decoded, budget)
        packed = self.compact(p.hidden, kept, cu)
        return dict(i0=i0, i1=i1, delta=raw, pooled=pooled, kept=kept, cu_seqlens=cu,
                    packed=packed, budget=np.asarray(_arr(budget, np.int32)))


_default = None


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle()
        return _default


def num_threads() -> int:
    return default().num_threads()


def set_num_threads(n: int) -> int:
    return default().set_num_threads(n)


def importance(*a, **k):
    return default().importance(*a, **k)


def delta_pool_mask(*a, **k):
    return default().delta_pool_mask(*a, **k)


def select(*a, **k):
    return default().select(*a, **k)


def compact(*a, **k):
    return default().compact(*a, **k)


def evict(p, constraints: int = 0, score: int = 0, lse0=None, decode_avg=None,
          alpha: float = 1.5) -> dict:
    return default().evict(p, constraints, score, lse0, decode_avg, alpha)


def dynamic_budget(*a, **k):
    return default().dynamic_budget(*a, **k)


def importance_lse(*a, **k):
    return default().importance_lse(*a, **k)


def importance_paged(*a, **k):
    return default().importance_paged(*a, **k)


def select_structured(*a, **k):
    return default().select_structured(*a, **k)
