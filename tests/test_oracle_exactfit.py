"""Pins of the vectorised exact-fit closed form (oracle/exactfit.py).

It is checked against a brute force over all 31,743 scales with the exact
integer test of oracle/exact.py, and against the fp64 oracle, on exact
multiples, single nonzero weights, all-zero groups, groups with no exact fit
and the ends of the binary16 range (CliffQuant project page, "What CliffQuant
changes": zero objective and the lower-pattern tie rule)."""
import numpy as np
import pytest

import oracle
from oracle import exact, exactfit


def f16bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def brute_lowest_fit(w_bits, qmin=-8, qmax=7):
    a = np.array([exact.half_units(int(b)) for b in w_bits], dtype=np.int64)
    c = exact.scale_units()
    ok = np.ones(len(c), bool)
    for ai in a:
        ok &= (ai % c == 0)
        ok &= (ai // c >= qmin) & (ai // c <= qmax)
    idx = np.nonzero(ok)[0]
    return int(idx[0]) + 1 if len(idx) else 0


def test_half_units_and_inverse_on_every_pattern():
    bits = np.array([b for b in range(1 << 16) if ((b >> 10) & 0x1F) != 31], dtype=np.uint16)
    a = exactfit.half_units(bits)
    ref = np.array([exact.half_units(int(b)) for b in bits], dtype=np.int64)
    assert np.array_equal(a, ref)
    posb = np.arange(1, 0x7C00, dtype=np.uint16)
    assert np.array_equal(exactfit.units_to_bits(exactfit.half_units(posb)), posb)


def _groups(rng):
    rows = []
    for t in range(10):
        s0 = np.ldexp(1.0 + int(rng.integers(0, 128)) / 128.0, int(rng.integers(-12, -3)))
        lo, hi = (-8, 8) if t % 2 == 0 else (-4, 4)
        rows.append(f16bits(rng.integers(lo, hi, 128) * s0))
    for v in (0.013, -0.027, 8 * 2.0 ** -10, -8 * 2.0 ** -10, 3 * 2.0 ** -24, -2.0 ** -24, 65504.0,
              -65504.0, 7 * 2.0 ** -3, -6 * 2.0 ** 5):
        w = np.zeros(128)
        w[int(rng.integers(0, 128))] = v
        rows.append(f16bits(w))
    rows.append(np.zeros(128, np.uint16))
    rows.append(np.full(128, 0x8000, np.uint16))
    rows.append(f16bits(rng.normal(0, 0.02, 128)))                # no fit
    rows.append(f16bits(rng.integers(-8, 8, 128) * 2.0 ** -24))   # subnormal multiples
    rows.append(f16bits(rng.integers(-1, 2, 128) * 32768.0))      # top of the range
    rows.append(f16bits(rng.integers(-8, 8, 128) * 3 * 2.0 ** -20))  # odd step 3
    w = f16bits(rng.integers(-8, 8, 128) * 2.0 ** -9)
    w[0] = f16bits([9 * 2.0 ** -9])[0]                             # 9 s0 does not fit at s0
    rows.append(w)
    return np.stack(rows)


def test_lowest_exact_fit_matches_bruteforce():
    rng = np.random.default_rng(31)
    W = _groups(rng)
    got = exactfit.lowest_exact_fit(W)
    for g in range(W.shape[0]):
        want = brute_lowest_fit(W[g])
        if np.all((W[g] & 0x7FFF) == 0):
            want = 1
        assert int(got[g]) == want, g
    assert got[-5] == 0                       # gaussian: no exact fit
    assert np.all(got[:20] > 0)


@pytest.mark.parametrize("qmin,qmax", [(-4, 3), (-16, 15), (-1, 1)])
def test_lowest_exact_fit_other_ranges(qmin, qmax):
    rng = np.random.default_rng(32 + qmax)
    W = _groups(rng)[:14]
    got = exactfit.lowest_exact_fit(W, qmin, qmax)
    for g in range(W.shape[0]):
        assert int(got[g]) == brute_lowest_fit(W[g], qmin, qmax), g


def test_lowest_exact_fit_is_the_oracle_answer():
    rng = np.random.default_rng(33)
    W = _groups(rng)
    fit = exactfit.lowest_exact_fit(W)
    sel = np.nonzero(fit)[0]
    D = rng.lognormal(0, 2.5, (8, W.shape[0], 128)).astype(np.float32)
    o = oracle.solve(W, D, sel=sel)
    assert np.array_equal(o["best_bits"], fit[sel])
    assert np.all(o["best_obj"] == 0.0)
