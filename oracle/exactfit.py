"""Closed form of the exact-fit case, vectorised over groups (test infrastructure).

Only the tests may use this module.  It shares no code with the CUDA path.

CliffQuant project page, "What CliffQuant changes": the objective is
``max_e sum_i d_{e,i} (w_i - s q_i)^2`` with ``q_i = clip(rne(w_i / s), -8, 7)``
over the positive finite binary16 scales, and the lower bit pattern wins an
exact objective tie.  When every d is positive the objective is zero exactly
when every residual is zero, i.e. when ``w_i = s q_i`` with ``q_i`` in the code
range for every i.  Zero is the least possible value, so whenever such a scale
exists the answer is the LOWEST such scale, whatever the diagonals are.

Every finite binary16 value is an integer multiple of 2^-24: ``w_i = a_i 2^-24``
and ``s = v 2^-24`` with integers ``a_i`` (|a_i| < 2^40) and ``v``.  Then
``w_i = s q_i`` with ``qmin <= q_i <= qmax`` is the integer test

    v divides a_i  and  qmin <= a_i / v <= qmax.

So v divides ``g = gcd_i |a_i|`` and ``v >= L = max(ceil(P / qmax), ceil(N / -qmin))``
(P the largest positive a_i, N the largest |a_i| of a negative weight).  The
integers v that are binary16 values are those with at most 11 significant bits
up to 65504 * 2^24 = 2047 * 2^29: ``v = d 2^u`` with d odd, d < 2048.  The
lowest exact fit is therefore the least ``d 2^u >= L`` over the odd divisors
d < 2048 of g's odd part and 0 <= u <= (the power of two in g).

An all-zero group fits every scale; its answer is pattern 0x0001.
"""
from __future__ import annotations

import numpy as np

_MAX_UNITS = 2047 << 29  # 65504 in units of 2^-24


def _units_table() -> np.ndarray:
    """int64 [65536]: units of 2^-24 of every pattern; non-finite ones hold a
    marker outside the finite range."""
    b = np.arange(1 << 16, dtype=np.int64)
    ex = (b >> 10) & 0x1F
    man = b & 0x3FF
    mag = np.where(ex == 0, man, (1024 + man) << np.maximum(ex - 1, 0))
    mag = np.where(ex == 31, np.int64(1) << 60, mag)
    return np.where(b & 0x8000, -mag, mag)


_TABLE = _units_table()


def half_units(bits: np.ndarray) -> np.ndarray:
    """int64 a with value(bits) == a * 2^-24, for finite binary16 patterns (any shape)."""
    a = _TABLE[np.asarray(bits, dtype=np.uint16)]
    if np.any(np.abs(a) >= (np.int64(1) << 60)):
        raise ValueError("not finite")
    return a


def units_to_bits(v: np.ndarray) -> np.ndarray:
    """Binary16 pattern of each positive integer v (units of 2^-24) that is a
    binary16 value: v < 1024 is subnormal; otherwise v = m 2^k with
    1024 <= m < 2048 and the biased exponent is k + 1."""
    v = np.asarray(v, dtype=np.int64)
    out = np.zeros(v.shape, dtype=np.int64)
    sub = v < 1024
    out[sub] = v[sub]
    big = ~sub
    if np.any(big):
        vb = v[big]
        k = np.floor(np.log2(vb.astype(np.float64))).astype(np.int64) - 10
        # fix a log2 rounding near a power of two
        k = np.where((vb >> np.maximum(k, 0)) >= 2048, k + 1, k)
        k = np.where((vb >> np.maximum(k, 0)) < 1024, k - 1, k)
        m = vb >> k
        assert np.all((m << k) == vb) and np.all((m >= 1024) & (m < 2048))
        out[big] = ((k + 1) << 10) | (m - 1024)
    return out.astype(np.uint16)


def lowest_exact_fit(W_bits: np.ndarray, qmin: int = -8, qmax: int = 7) -> np.ndarray:
    """For each group (row of W_bits, uint16 [G, n]) the lowest binary16 scale
    pattern at which every weight is exactly s * q with q in [qmin, qmax], or 0
    when there is none.  All-zero groups give 0x0001.  The answer of the
    minimax selection equals it wherever it is nonzero and every d > 0."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    G = W.shape[0]
    out = np.zeros(G, dtype=np.uint16)
    g = np.zeros(G, dtype=np.int64)
    L = np.zeros(G, dtype=np.int64)
    for c0 in range(0, G, 1 << 14):  # chunks keep the int64 temporaries small
        a = half_units(W[c0:c0 + (1 << 14)])
        g[c0:c0 + len(a)] = np.gcd.reduce(np.abs(a), axis=1)
        pos = np.maximum(a, 0).max(axis=1)
        neg = np.maximum(-a, 0).max(axis=1)
        L[c0:c0 + len(a)] = np.maximum(-(-pos // qmax), -(-neg // (-qmin)))
    zero = g == 0
    out[zero] = 0x0001
    # v divides g, so v <= g: only groups with g >= L can fit
    cand = np.nonzero(~zero & (g >= L))[0]
    if len(cand) == 0:
        return out
    gc, Lc = g[cand], L[cand]
    t = np.zeros(len(cand), dtype=np.int64)  # power of two in g
    odd = gc.copy()
    while True:
        ev = (odd & 1) == 0
        if not np.any(ev):
            break
        odd = np.where(ev, odd >> 1, odd)
        t += ev
    best = np.full(len(cand), np.iinfo(np.int64).max, dtype=np.int64)
    # groups that share an odd part share its divisors: one small 2-D step each
    uo, inv = np.unique(odd, return_inverse=True)
    order = np.argsort(inv, kind="stable")
    starts = np.searchsorted(inv[order], np.arange(len(uo) + 1))
    for k, o in enumerate(uo.tolist()):
        idx = order[starts[k]:starts[k + 1]]
        dv = np.array([d for d in range(1, min(o, 2047) + 1, 2) if o % d == 0], dtype=np.int64)
        Lk = Lc[idx][:, None]
        # least u >= 0 with d 2^u >= L: u = ceil(log2(ceil(L / d))) = bitlen(ceil(L / d) - 1)
        y = np.maximum(-(-Lk // dv[None, :]) - 1, 0)
        u = np.frexp(y.astype(np.float64))[1].astype(np.int64)
        v = dv[None, :] << np.minimum(u, 40)
        ok = (u <= t[idx][:, None]) & (v <= _MAX_UNITS) & (v >= Lk)
        best[idx] = np.where(ok, v, np.iinfo(np.int64).max).min(axis=1)
    found = best != np.iinfo(np.int64).max
    out[cand[found]] = units_to_bits(best[found])
    return out
