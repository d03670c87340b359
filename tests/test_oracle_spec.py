"""Pins of the oracle for quantiser specs other than (qmin, qmax, n) =
(-8, 7, 128) (CliffQuant project page, "Use the solver": the solver takes a
QuantizerSpec(qmin, qmax)), against the exact-integer brute force and closed
forms.  Group sizes other than 128 use the same definition over n weights."""
import numpy as np
import pytest

import oracle
from oracle import exact

SPECS = [(-4, 3), (-2, 1), (-1, 1), (-16, 15), (-128, 127), (-8, 8)]
NEAR_TIE = 1e-12


def f16bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def solve1(w_bits, d, **kw):
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    d = np.asarray(d, dtype=np.float32)
    r = oracle.solve(w_bits[None, :], d[:, None, :], **kw)
    return {k: v[0] for k, v in r.items()}


def _check_against_exact(w, d, qmin, qmax):
    x = exact.solve(w, d, qmin, qmax)
    o = solve1(w, d, qmin=qmin, qmax=qmax)
    xb, xr = float(x["best"]), float(x["runner"])
    assert oracle.rel_gap(o["best_obj"], xb) <= 1e-13 or (xb == 0 and o["best_obj"] == 0)
    gap = oracle.rel_gap(xb, xr) if x["best"] != x["runner"] else 0.0
    if x["best"] == 0 or gap > NEAR_TIE:
        assert o["best_bits"] == x["best_bits"]
        assert np.array_equal(o["codes"][: len(w)], x["codes"])
        assert int(o["codes"].min()) >= qmin and int(o["codes"].max()) <= qmax
    else:
        fo, _ = exact.objective_at(w, d, int(o["best_bits"]), qmin, qmax)
        assert oracle.rel_gap(float(fo), xb) <= NEAR_TIE


@pytest.mark.parametrize("spec", SPECS)
def test_spec_matches_exact_bruteforce(spec):
    qmin, qmax = spec
    rng = np.random.default_rng(abs(qmin) * 100 + qmax)
    for n, E, sigma in ((3, 1, 0.3), (5, 2, 0.02), (8, 3, 7.0), (6, 2, 1e-4)):
        w = f16bits(rng.normal(0, sigma, n))
        d = rng.lognormal(0, 1.5, (E, n)).astype(np.float32)
        _check_against_exact(w, d, qmin, qmax)


@pytest.mark.parametrize("n", [16, 64, 256])
def test_group_sizes_match_exact_bruteforce(n):
    rng = np.random.default_rng(n)
    w = f16bits(rng.normal(0, 0.02, n) * np.where(rng.random(n) < 0.05, 8, 1))
    d = rng.lognormal(0, 1.5, (2, n)).astype(np.float32)
    _check_against_exact(w, d, -8, 7)
    if n == 16:
        _check_against_exact(w, d, -4, 3)


def _single_nonzero_expected(wb, qmin, qmax):
    """Least |w|/m (m = 1..|qmin| for w < 0, 1..qmax for w > 0) that is a
    binary16 value, by integer divisibility on the 2^-24 grid."""
    a = exact.half_units(int(wb))
    K = -qmin if a < 0 else qmax
    units = {int(c): b for b, c in enumerate(exact.scale_units(), start=1)}
    for m in range(K, 0, -1):
        if abs(a) % m == 0 and abs(a) // m in units:
            return units[abs(a) // m]
    raise AssertionError


@pytest.mark.parametrize("spec,n", [((-4, 3), 64), ((-2, 1), 32), ((-128, 127), 256), ((-16, 15), 128)])
def test_single_nonzero_closed_form(spec, n):
    qmin, qmax = spec
    rng = np.random.default_rng(n + qmax)
    for v in list(rng.normal(0, 0.02, 6)) + [12 * 2.0 ** -10, -12 * 2.0 ** -10, 65504.0, -2.0 ** -24]:
        wb = f16bits([v])[0]
        w = np.zeros(n, np.uint16)
        w[int(rng.integers(0, n))] = wb
        d = rng.lognormal(0, 1, (2, n)).astype(np.float32)
        o = solve1(w, d, qmin=qmin, qmax=qmax)
        assert o["best_obj"] == 0.0
        assert o["best_bits"] == _single_nonzero_expected(wb, qmin, qmax), (spec, v)


@pytest.mark.parametrize("spec", SPECS)
def test_absmax_bound_and_more_levels_never_worse(spec):
    qmin, qmax = spec
    rng = np.random.default_rng(7)
    W = f16bits(rng.normal(0, 0.02, (4, 64)))
    D = rng.lognormal(0, 1.5, (3, 4, 64)).astype(np.float32)
    r = oracle.solve(W, D, qmin=qmin, qmax=qmax)
    wide = oracle.solve(W, D, qmin=qmin - 1, qmax=qmax + 1)
    for g in range(4):
        ab = oracle.absmax_scale(W[g], qmax)
        if ab:
            assert r["best_obj"][g] <= oracle.objective(W[g], D[:, g, :], ab, qmin, qmax)[0]
        # a wider code range contains every code vector of the narrower one at each scale
        assert wide["best_obj"][g] <= r["best_obj"][g]
