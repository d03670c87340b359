"""Exact-integer brute force of minimax FP16 scale selection (test infrastructure).

Same definition as the fp64 oracle (CliffQuant project page, "What CliffQuant
changes"), evaluated without any rounding, for tiny groups:

* every finite binary16 value is an integer multiple of 2^-24: w_i = a_i 2^-24,
  s = c 2^-24 (the binary16 layout: 10 fraction bits, exponent bias 15);
* q_i = clip(round-half-even(a_i / c), qmin, qmax) by integer division with the
  remainder compared against c/2;
* each fp32 diagonal is an integer times a power of two, so after one common
  power-of-two factor every objective is the exact integer
  sum_i D_i (a_i - c q_i)^2, and max/argmin are exact;
* the lowest bit pattern wins an exact tie.

Used only to pin the fp64 oracle; it shares nothing with it.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

N_SCALES = 0x7BFF  # patterns 0x0001..0x7BFF


def half_units(bits: int) -> int:
    """Signed integer a with value(bits) == a * 2^-24 (finite patterns only)."""
    sign = -1 if bits & 0x8000 else 1
    ex = (bits >> 10) & 0x1F
    man = bits & 0x3FF
    if ex == 31:
        raise ValueError("not finite")
    a = man if ex == 0 else (1024 + man) << (ex - 1)
    return sign * a


def scale_units() -> np.ndarray:
    """int64 [31743]: c for patterns 0x0001..0x7BFF, ascending."""
    return np.array([half_units(b) for b in range(1, N_SCALES + 1)], dtype=np.int64)


_C = None


def _scales():
    global _C
    if _C is None:
        _C = scale_units()
    return _C


def _float_to_int_pow2(x: float):
    fr = Fraction(float(x))
    den = fr.denominator
    assert den & (den - 1) == 0
    return fr.numerator, den.bit_length() - 1  # x = num * 2^-k


def rne_div(a: int, c: np.ndarray) -> np.ndarray:
    """round-half-even(a / c) for integer a and a vector of positive c."""
    mag = abs(a)
    fl = mag // c
    rem = mag - fl * c
    twice = 2 * rem
    up = (twice > c) | ((twice == c) & (fl % 2 == 1))
    q = fl + up.astype(np.int64)
    return -q if a < 0 else q


def objectives(w_bits, d, qmin: int = -8, qmax: int = 7):
    """Exact objectives at every scale: (values as Python ints [31743],
    common factor as Fraction, codes int64 [31743, n]).  f_b = values[b-1] * factor."""
    w_bits = [int(x) for x in np.asarray(w_bits, dtype=np.uint16)]
    d = np.asarray(d, dtype=np.float32)
    E, n = d.shape
    a = [half_units(b) for b in w_bits]
    c = _scales()
    nums, ks = zip(*[_float_to_int_pow2(float(x)) for x in d.ravel()]) if d.size else ((), ())
    kmax = max(ks) if ks else 0
    Dint = np.array([nm << (kmax - k) for nm, k in zip(nums, ks)], dtype=object).reshape(E, n)
    codes = np.zeros((len(c), n), dtype=np.int64)
    res_sq = []
    for i in range(n):
        q = np.clip(rne_div(a[i], c), qmin, qmax)
        codes[:, i] = q
        r = (a[i] - c * q).astype(object)
        res_sq.append(r * r)
    f = None
    for e in range(E):
        acc = np.zeros(len(c), dtype=object)
        for i in range(n):
            acc = acc + Dint[e, i] * res_sq[i]
        f = acc if f is None else np.maximum(f, acc)
    factor = Fraction(1, 2 ** (48 + kmax))
    return f, factor, codes


def solve(w_bits, d, qmin: int = -8, qmax: int = 7):
    """Exact argmin.  Returns dict(best_bits, best (Fraction), runner_bits,
    runner (Fraction), codes int64 [n])."""
    f, factor, codes = objectives(w_bits, d, qmin, qmax)
    vals = list(f)
    best_i = min(range(len(vals)), key=lambda k: (vals[k], k))
    rest = [(vals[k], k) for k in range(len(vals)) if k != best_i]
    run_v, run_i = min(rest)
    return dict(best_bits=best_i + 1, best=vals[best_i] * factor, runner_bits=run_i + 1,
                runner=run_v * factor, codes=codes[best_i].copy())


def objective_at(w_bits, d, scale_bits: int, qmin: int = -8, qmax: int = 7):
    """Exact (max_e objective as Fraction, codes) at one scale."""
    f, factor, codes = objectives(w_bits, d, qmin, qmax)
    k = scale_bits - 1
    return f[k] * factor, codes[k].copy()
