"""CPU oracle for the AdaFuse adapter switch (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / ``--impl reference`` legs may import this package.  It is a
ctypes wrapper around ``adafuse_oracle.c`` (fp64, plain loops) and shares no
code with the CUDA library in ``weight_merge_b200``.

Sources, by page title and section:
  "AdaFuse: Accelerating Dynamic Adapter Inference via Token-Level Pre-Gating
  and Fused Kernel Optimization" -- shd-paper.top summary, English abstract;
  gist.science technical summary, section 2-ga (token-level pre-gating, top-2
  router in the first layer, decision applied to every layer) and section 2-na
  (fused adapter switching: un-merge the previous token's adapters, merge the
  current token's, all layers, in place).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, library routines (numpy matmul, torch bf16 rounding, stable
argsort) and hand-worked fixtures under ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "adafuse_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` with gcc + OpenMP."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
             "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        lib.orc_bf16_from_double.restype = ctypes.c_uint16
        lib.orc_bf16_from_double.argtypes = [dbl]
        lib.orc_bf16_to_double.restype = dbl
        lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_from_double_array.argtypes = [P, i64, P]
        lib.orc_pregate.argtypes = [P, i64, i64, P, i32, P, P, P]
        lib.orc_switch_rows.argtypes = [P, P, i64, i64, i64, P, P, i32, dbl,
                                        P, P, P, P, P, P]
        lib.orc_switch_rows_k.argtypes = [P, P, i64, i64, i64, P, P, i32, dbl, i32,
                                          P, P, P, P, P, P]
        lib.orc_pregate_topk.argtypes = [P, i64, i64, P, i32, i32, P, P, P]
        lib.orc_pregate_batch.argtypes = [P, i64, i64, P, i32, i32, P, P, P]
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().orc_num_threads()


def set_num_threads(n: int) -> None:
    _load().orc_set_num_threads(int(n))


def bf16_from_f64(x) -> np.ndarray:
    """Round fp64 values to bf16 bit patterns (uint16), nearest-even, one step."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().orc_bf16_from_double_array(_ptr(x), x.size, _ptr(out))
    return out


def bf16_to_f64(b) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp64 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def pregate(h: np.ndarray, Wr: np.ndarray, return_logits: bool = False):
    """Token-level top-2 pre-gating.

    h [T, d] fp32, Wr [d, E] fp32  ->  idx [T, 2] int32, gate [T, 2] fp32
    (and the fp64 logits [T, E] when ``return_logits``).
    """
    h = np.ascontiguousarray(h, dtype=np.float32)
    Wr = np.ascontiguousarray(Wr, dtype=np.float32)
    T, d = h.shape
    d2, E = Wr.shape
    assert d == d2
    idx = np.empty((T, 2), dtype=np.int32)
    gate = np.empty((T, 2), dtype=np.float32)
    z = np.empty((T, E), dtype=np.float64)
    _load().orc_pregate(_ptr(h), T, d, _ptr(Wr), E, _ptr(idx), _ptr(gate), _ptr(z))
    if return_logits:
        return idx, gate, z
    return idx, gate


def pregate_topk(h: np.ndarray, Wr: np.ndarray, k: int, return_logits: bool = False):
    """Token-level top-k pre-gating, k in [1, 4] (the pages' router is k = 2).

    h [T, d] fp32, Wr [d, E] fp32  ->  idx [T, k] int32, gate [T, k] fp32
    (slots past E: idx -1, gate 0), and the fp64 logits when ``return_logits``.
    """
    assert 1 <= k <= 4
    h = np.ascontiguousarray(h, dtype=np.float32)
    Wr = np.ascontiguousarray(Wr, dtype=np.float32)
    T, d = h.shape
    d2, E = Wr.shape
    assert d == d2
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k), dtype=np.float32)
    z = np.empty((T, E), dtype=np.float64)
    _load().orc_pregate_topk(_ptr(h), T, d, _ptr(Wr), E, k, _ptr(idx), _ptr(gate), _ptr(z))
    if return_logits:
        return idx, gate, z
    return idx, gate


def pregate_batch(h: np.ndarray, Wr: np.ndarray, k: int = 2, return_logits: bool = False):
    """One routing decision for a decode batch (a reading beyond the pages'
    per-token router, see adafuse_oracle.c): the top-k of the tokens' mean
    logits, gates = their softmax renormalised over the picks.

    h [T, d] fp32 (T >= 1), Wr [d, E] fp32  ->  idx [k] int32, gate [k] fp32
    (and the fp64 mean logits [E] when ``return_logits``).
    """
    assert 1 <= k <= 4
    h = np.ascontiguousarray(h, dtype=np.float32)
    Wr = np.ascontiguousarray(Wr, dtype=np.float32)
    T, d = h.shape
    d2, E = Wr.shape
    assert d == d2 and T >= 1
    idx = np.empty(k, dtype=np.int32)
    gate = np.empty(k, dtype=np.float32)
    zbar = np.empty(E, dtype=np.float64)
    _load().orc_pregate_batch(_ptr(h), T, d, _ptr(Wr), E, k, _ptr(idx), _ptr(gate), _ptr(zbar))
    if return_logits:
        return idx, gate, zbar
    return idx, gate


def _route_arrays(route, slots):
    if route is None:
        return None, None
    idx, gate = route
    return (np.ascontiguousarray(idx, dtype=np.int32).reshape(slots),
            np.ascontiguousarray(gate, dtype=np.float32).reshape(slots))


def _slots(prev, cur):
    for rt in (prev, cur):
        if rt is not None:
            return int(np.asarray(rt[0]).size)
    return 2


def switch_rows(W_rows, row_ids, out: int, A, B, s: float, prev, cur,
                exact: bool = False):
    """Switch chosen rows of one [out, in] bf16 weight.

    W_rows [n, in] uint16 (bf16 bits), row_ids [n] int64,
    A [E, r, in] uint16, B [E, out, r] uint16,
    prev / cur: (idx[k], gate[k]) or None, k in [1, 4] (2 for the top-2 router).
    Returns W_new [n, in] uint16, and W + dW in fp64 when ``exact``.
    """
    W_rows = np.ascontiguousarray(W_rows, dtype=np.uint16)
    n, inn = W_rows.shape
    row_ids = np.ascontiguousarray(row_ids, dtype=np.int64).reshape(n)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    E, r, in2 = A.shape
    assert in2 == inn and B.shape == (E, out, r)
    k = _slots(prev, cur)
    assert 1 <= k <= 4
    pi, pg = _route_arrays(prev, k)
    ci, cg = _route_arrays(cur, k)
    W_new = np.empty_like(W_rows)
    W_ex = np.empty((n, inn), dtype=np.float64) if exact else None
    if k == 2:
        _load().orc_switch_rows(_ptr(W_rows), _ptr(row_ids), n, out, inn, _ptr(A), _ptr(B),
                                r, float(s), _ptr(pi), _ptr(pg), _ptr(ci), _ptr(cg),
                                _ptr(W_new), _ptr(W_ex))
    else:
        _load().orc_switch_rows_k(_ptr(W_rows), _ptr(row_ids), n, out, inn, _ptr(A), _ptr(B),
                                  r, float(s), k, _ptr(pi), _ptr(pg), _ptr(ci), _ptr(cg),
                                  _ptr(W_new), _ptr(W_ex))
    if exact:
        return W_new, W_ex
    return W_new


def switch(W, A, B, s: float, prev, cur, exact: bool = False):
    """Switch a whole [out, in] weight (all rows)."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    return switch_rows(W, np.arange(W.shape[0], dtype=np.int64), W.shape[0], A, B, s,
                       prev, cur, exact=exact)
