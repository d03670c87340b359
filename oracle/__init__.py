"""CPU oracle for exact minimax FP16 group-scale selection (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA path.

* ``cq_oracle.c``   plain exhaustive fp64 solver over all 31,743 positive
                    finite binary16 scales (CliffQuant project page, "What
                    CliffQuant changes": the minimax objective, round-half-even
                    codes clipped to [-8, 7], lower bit pattern wins a tie).
* ``exact.py``      exact-integer brute force of the same definition for tiny
                    groups, used to pin the fp64 oracle.

The C library is built in-tree on first use (gcc, -O2 -ffp-contract=off).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cq_oracle.c")
_LIB = os.path.join(_HERE, "libcq_oracle.so")
_lib = None

QMIN, QMAX = -8, 7
FIRST_SCALE, LAST_SCALE = 0x0001, 0x7BFF


def build(force: bool = False) -> str:
    """Compile the oracle's C library in-tree; returns its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load(path: str):
    """Open a build of cq_oracle.c and declare its signatures."""
    L = ctypes.CDLL(path)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    f64p = ctypes.POINTER(ctypes.c_double)
    L.cqo_half_to_double.restype = ctypes.c_double
    L.cqo_half_to_double.argtypes = [ctypes.c_uint16]
    L.cqo_double_to_half_rne.restype = ctypes.c_uint16
    L.cqo_double_to_half_rne.argtypes = [ctypes.c_double]
    L.cqo_objective.restype = ctypes.c_double
    L.cqo_objective.argtypes = [u16p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_uint16,
                                ctypes.c_int, ctypes.c_int, ctypes.c_void_p, f64p]
    L.cqo_solve_batch.restype = ctypes.c_int
    L.cqo_solve_batch.argtypes = [u16p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                  ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    L.cqo_pack_codes.restype = None
    L.cqo_pack_codes.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    L.cqo_absmax_scale.restype = ctypes.c_uint16
    L.cqo_absmax_scale.argtypes = [u16p, ctypes.c_int, ctypes.c_int]
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load(_LIB)
    return _lib


def _set_lib(handle):
    """Swap the active library (the mutation tests use this); returns the old one."""
    global _lib
    old = _lib
    _lib = handle
    return old


def _ptr(a, ctype=None):
    return a.ctypes.data_as(ctypes.POINTER(ctype)) if ctype else ctypes.c_void_p(a.ctypes.data)


def half_to_double(bits: int) -> float:
    return lib().cqo_half_to_double(int(bits))


def double_to_half_rne(x: float) -> int:
    return int(lib().cqo_double_to_half_rne(float(x)))


def _diag_ptr_array(d: np.ndarray):
    arr = (ctypes.c_void_p * d.shape[0])()
    for e in range(d.shape[0]):
        arr[e] = d[e].ctypes.data
    return arr


def objective(w_bits, d, scale_bits: int, qmin: int = QMIN, qmax: int = QMAX):
    """(max_e objective, per-env objectives [E], codes int8 [n]) at one scale.
    w_bits: uint16 [n]; d: float32 [E, n]."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    d = np.ascontiguousarray(d, dtype=np.float32)
    E, n = d.shape
    assert w.shape == (n,)
    codes = np.zeros(n, dtype=np.int8)
    per = np.zeros(E, dtype=np.float64)
    ptrs = _diag_ptr_array(d)
    f = lib().cqo_objective(_ptr(w, ctypes.c_uint16), ctypes.cast(ptrs, ctypes.c_void_p), E, n,
                            int(scale_bits), qmin, qmax, _ptr(codes), _ptr(per, ctypes.c_double))
    return f, per, codes


def solve(W, D, K: int = 0, sel=None, qmin: int = QMIN, qmax: int = QMAX, threads: int | None = None):
    """Exhaustive solve.  W: uint16 [G, n].  D: float32 [E, K] per column (K > 0)
    or [E, G, n] per group (K == 0).  sel: optional group indices.

    Returns a dict of arrays indexed like ``sel`` (or all groups): best_bits,
    best_obj, runner_bits, runner_obj, codes (int8 [count, n])."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    D = np.ascontiguousarray(D, dtype=np.float32)
    G, n = W.shape
    E = D.shape[0]
    if K:
        assert D.shape == (E, K) and K % n == 0
    else:
        assert D.shape == (E, G, n)
    if sel is None:
        sel_arr = None
        count = G
    else:
        sel_arr = np.ascontiguousarray(sel, dtype=np.int64)
        count = len(sel_arr)
        assert count == 0 or (sel_arr.min() >= 0 and sel_arr.max() < G)
    out = dict(best_bits=np.zeros(count, np.uint16), best_obj=np.zeros(count, np.float64),
               runner_bits=np.zeros(count, np.uint16), runner_obj=np.zeros(count, np.float64),
               codes=np.zeros((count, n), np.int8))
    if count == 0:
        return out
    threads = threads or os.cpu_count() or 1
    st = lib().cqo_solve_batch(_ptr(W, ctypes.c_uint16), G, n, _ptr(D), E, K,
                               _ptr(sel_arr) if sel_arr is not None else None, count, qmin, qmax,
                               _ptr(out["best_bits"]), _ptr(out["best_obj"]), _ptr(out["runner_bits"]),
                               _ptr(out["runner_obj"]), _ptr(out["codes"]), int(threads))
    if st != 0:
        raise RuntimeError(f"oracle solve failed with status {st}")
    return out


def pack_codes(codes) -> np.ndarray:
    """(q + 8) nibbles, 8 per uint32, low nibble first.  codes: int8 [..., n]."""
    q = np.ascontiguousarray(codes, dtype=np.int8)
    n = q.shape[-1]
    flat = q.reshape(-1, n)
    out = np.zeros((flat.shape[0], n // 8), dtype=np.uint32)
    for r in range(flat.shape[0]):
        lib().cqo_pack_codes(_ptr(flat[r]), n, _ptr(out[r]))
    return out.reshape(q.shape[:-1] + (n // 8,))


def absmax_scale(w_bits, qmax: int = QMAX) -> int:
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    return int(lib().cqo_absmax_scale(_ptr(w, ctypes.c_uint16), w.shape[0], qmax))


def rel_gap(a: float, b: float) -> float:
    """|a - b| / max(|a|, |b|), 0/0 = 0."""
    m = max(abs(a), abs(b))
    return 0.0 if m == 0 else abs(a - b) / m
