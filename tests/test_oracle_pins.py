"""Pins of the fp64 CPU oracle to things other than itself.

Each check follows the CliffQuant project page ("What CliffQuant changes"):
minimise max_e sum_i d_{e,i} (w_i - s q_i(s))^2 over the 31,743 positive finite
binary16 scales, q = clip(round-half-even(w/s), -8, 7), lower bit pattern wins
an exact tie.  The pins are: the exact-integer brute force on tiny groups, the
page's own solver example (golden), closed forms (all-zero, single nonzero,
exact fit), library conversions (numpy float16), and invariants of the
definition.  Relative gaps use |a-b|/max(|a|,|b|).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact

HERE = os.path.dirname(os.path.abspath(__file__))
NEAR_TIE = 1e-12


def f16bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def rel(a, b):
    return oracle.rel_gap(float(a), float(b))


def solve1(w_bits, d, **kw):
    """Oracle on one group: w_bits [n], d [E, n]."""
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    d = np.asarray(d, dtype=np.float32)
    r = oracle.solve(w_bits[None, :], d[:, None, :], **kw)
    return {k: v[0] for k, v in r.items()}


# --------------------------------------------------------------- conversions

def test_scale_domain_is_31743_ordered_patterns():
    # The page's exhaustive reference enumerates 31,743 positive finite FP16 values.
    bits = np.arange(0x0001, 0x7C00, dtype=np.uint16)
    assert len(bits) == 31743
    ref = bits.view(np.float16).astype(np.float64)
    mine = np.array([oracle.half_to_double(int(b)) for b in bits])
    assert np.array_equal(ref, mine)                    # library decode
    assert np.all(np.diff(mine) > 0)                    # bit order == value order
    assert np.all(np.isfinite(mine)) and mine[0] == 2.0 ** -24 and mine[-1] == 65504.0
    units = exact.scale_units()                          # integer decode agrees
    assert np.array_equal(units.astype(np.float64) * 2.0 ** -24, mine)


def test_double_to_half_rne_matches_numpy():
    rng = np.random.default_rng(5)
    xs = np.concatenate([rng.lognormal(-6, 4, 4000), 2.0 ** rng.uniform(-26, 16, 2000)])
    # exact midpoints between neighbouring halves (ties)
    b = rng.integers(1, 0x7BFE, 500).astype(np.uint16)
    lo = b.view(np.float16).astype(np.float64)
    hi = (b + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    xs = np.concatenate([xs, (lo + hi) / 2, [65504.0, 65519.0, 65520.0, 2.0 ** -25, 3 * 2.0 ** -26]])
    xs = xs[xs < 65520]
    ref = xs.astype(np.float16).view(np.uint16)
    mine = np.array([oracle.double_to_half_rne(x) for x in xs], dtype=np.uint16)
    assert np.array_equal(ref, mine)


def test_pack_codes_layout():
    q = np.tile(np.arange(-8, 8, dtype=np.int8), 8)  # nibbles 0..15 twice per 16 codes
    words = oracle.pack_codes(q)
    assert words.shape == (16,)
    assert list(words[:2]) == [0x76543210, 0xFEDCBA98]
    assert np.all(words[0::2] == 0x76543210) and np.all(words[1::2] == 0xFEDCBA98)
    assert list(oracle.pack_codes(np.zeros(128, np.int8))) == [0x88888888] * 16


# ------------------------------------------------------- exact brute force

def _tiny_cases():
    rng = np.random.default_rng(11)
    cases = []
    for t, (n, E, sigma) in enumerate([(1, 1, 0.3), (2, 1, 0.02), (3, 2, 1.0), (4, 2, 7.0), (5, 3, 0.05),
                                       (6, 2, 1e-5), (7, 3, 0.02), (8, 2, 120.0), (8, 3, 0.5),
                                       (4, 1, 2e-7), (6, 3, 3000.0), (8, 1, 0.02)]):
        w = f16bits(rng.normal(0, sigma, n))
        d = rng.lognormal(0, 1.5, (E, n)).astype(np.float32)
        if t % 4 == 3:
            d[rng.integers(0, E), rng.integers(0, n)] = 0.0
        cases.append((w, d))
    return cases


@pytest.mark.parametrize("case", range(12))
def test_oracle_matches_exact_bruteforce(case):
    w, d = _tiny_cases()[case]
    x = exact.solve(w, d)
    o = solve1(w, d)
    xb, xr = float(x["best"]), float(x["runner"])
    # fp64 objective agrees with the exact value far inside the 1e-12 rule
    assert rel(o["best_obj"], xb) <= 1e-13 or (xb == 0 and o["best_obj"] == 0)
    assert rel(o["runner_obj"], xr) <= 1e-13 or (xr == 0 and o["runner_obj"] == 0)
    exact_gap = oracle.rel_gap(xb, xr) if x["best"] != x["runner"] else 0.0
    if x["best"] == 0 or exact_gap > NEAR_TIE:
        assert o["best_bits"] == x["best_bits"]
        assert o["runner_bits"] == x["runner_bits"]
        assert np.array_equal(o["codes"][: len(w)], x["codes"])
    else:
        fo, _ = exact.objective_at(w, d, int(o["best_bits"]))
        assert rel(fo, x["best"]) <= NEAR_TIE


def test_pages_solver_example_golden():
    with open(os.path.join(HERE, "golden", "p2_example.json")) as f:
        g = json.load(f)
    w = f16bits(g["weights"])
    assert [int(x) for x in w] == g["w_bits"]
    d = np.array(g["environment_diagonals"], dtype=np.float32)
    o = solve1(w, d)
    assert o["best_bits"] == g["best_bits"]
    assert o["runner_bits"] == g["runner_up_bits"]
    assert rel(o["best_obj"], Fraction(g["best_objective_fraction"])) <= 1e-15
    assert list(o["codes"][:4]) == g["codes"]
    # exact brute force recomputed here agrees with the stored values
    x = exact.solve(w, d)
    assert x["best_bits"] == g["best_bits"] and str(x["best"]) == g["best_objective_fraction"]


def test_objective_at_rounding_ties_and_clip():
    """Scales where w/s is an exact half-integer (round-half-even decides) and
    where codes clip at -8 / +7, against the exact integer evaluation."""
    rng = np.random.default_rng(3)
    s = np.float16(2.0 ** -6)
    halves = np.array([0.5, 1.5, 2.5, 3.5, 6.5, 7.5, 8.5, -0.5, -1.5, -2.5, -7.5, -8.5, 9.0, -11.0, 0.0, -0.0])
    w = f16bits(halves * float(s))
    d = rng.lognormal(0, 1, (2, len(w))).astype(np.float32)
    sb = int(np.array(s).view(np.uint16))
    f, per, codes = oracle.objective(w, d, sb)
    expect = np.array([0, 2, 2, 4, 6, 7, 7, 0, -2, -2, -8, -8, 7, -8, 0, 0])
    assert list(codes) == list(expect)
    fx, cx = exact.objective_at(w, d, sb)
    assert list(cx) == list(expect)
    assert rel(f, fx) <= 1e-15


# -------------------------------------------------------------- closed forms

def test_all_zero_group():
    for w in (np.zeros(128, np.uint16), np.full(128, 0x8000, np.uint16)):  # +0 and -0
        d = np.random.default_rng(1).lognormal(0, 1, (4, 128)).astype(np.float32)
        o = solve1(w, d)
        assert o["best_bits"] == 0x0001 and o["best_obj"] == 0.0 and o["runner_obj"] == 0.0
        assert list(oracle.pack_codes(o["codes"])) == [0x88888888] * 16


def _single_nonzero_expected(wb):
    """Least |w|/m (m = 1..8 for w < 0, 1..7 for w > 0) that is a binary16
    value, found by integer divisibility on the 2^-24 grid."""
    a = exact.half_units(int(wb))
    K = 8 if a < 0 else 7
    units = {int(c): b for b, c in enumerate(exact.scale_units(), start=1)}
    for m in range(K, 0, -1):
        if abs(a) % m == 0 and abs(a) // m in units:
            return units[abs(a) // m]
    raise AssertionError


def test_single_nonzero_closed_form():
    rng = np.random.default_rng(4)
    vals = list(rng.normal(0, 0.02, 10)) + [8 * 2.0 ** -10, -8 * 2.0 ** -10, 3 * 2.0 ** -24, -2.0 ** -24,
                                           65504.0, -65504.0, 7 * 2.0 ** -3, -6 * 2.0 ** 5]
    for v in vals:
        wb = f16bits([v])[0]
        w = np.zeros(128, np.uint16)
        pos = int(rng.integers(0, 128))
        w[pos] = wb
        d = rng.lognormal(0, 1, (3, 128)).astype(np.float32)
        o = solve1(w, d)
        assert o["best_obj"] == 0.0
        assert o["best_bits"] == _single_nonzero_expected(wb), v
    # the clip asymmetry: -8*2^-10 reaches q=-8 at 2^-10, +8*2^-10 needs q=4 at 2^-9
    assert _single_nonzero_expected(f16bits([-8 * 2.0 ** -10])[0]) == 0x1400
    assert _single_nonzero_expected(f16bits([8 * 2.0 ** -10])[0]) == 0x1800


def test_exact_fit_lowest_zero_scale():
    """w_i = m_i * s0: the answer is the smallest scale c (in 2^-24 units)
    dividing every a_i with a_i / c in [-8, 7] (integer test)."""
    rng = np.random.default_rng(6)
    c_all = exact.scale_units()
    for t in range(6):
        s0 = np.ldexp(1.0 + int(rng.integers(0, 128)) / 128.0, int(rng.integers(-12, -3)))
        lo, hi = (-8, 8) if t % 2 == 0 else (-4, 4)
        m = rng.integers(lo, hi, 128)
        w = f16bits(m * s0)
        a = np.array([exact.half_units(int(b)) for b in w])
        ok = np.ones(len(c_all), bool)
        for ai in a:
            ok &= (ai % c_all == 0) & (ai // c_all >= -8) & (ai // c_all <= 7)
        expect = int(np.nonzero(ok)[0][0]) + 1
        d = rng.lognormal(0, 2.5, (8, 128)).astype(np.float32)
        o = solve1(w, d)
        assert o["best_obj"] == 0.0
        assert o["best_bits"] == expect
        if t % 2 == 1 and np.any(m != 0):
            # codes in U{-4..3} also fit exactly at s0/2, which must win
            assert oracle.half_to_double(expect) <= s0 / 2


# --------------------------------------------------------------- invariants

def make_groups128():
    rng = np.random.default_rng(21)
    W = f16bits(rng.normal(0, 0.02, (6, 128)) * np.where(rng.random((6, 128)) < 0.02, 10, 1))
    D = rng.lognormal(0, 1.5, (4, 6, 128)).astype(np.float32)
    D /= D.mean(axis=2, keepdims=True)
    return W, D.astype(np.float32)


@pytest.fixture(scope="module")
def groups128():
    return make_groups128()


def test_env_duplicate_permute_pow2_invariance(groups128):
    W, D = groups128
    base = oracle.solve(W, D)
    dup = oracle.solve(W, np.concatenate([D, D[1:2]], axis=0))
    perm = oracle.solve(W, D[[2, 0, 3, 1]])
    p2 = oracle.solve(W, (D * 8.0).astype(np.float32))
    for r in (dup, perm):
        assert np.array_equal(r["best_bits"], base["best_bits"])
        assert np.array_equal(r["best_obj"], base["best_obj"])
    assert np.array_equal(p2["best_bits"], base["best_bits"])
    assert np.array_equal(p2["best_obj"], base["best_obj"] * 8.0)


def test_common_constant_scaling(groups128):
    W, D = groups128
    base = oracle.solve(W, D)
    sc = oracle.solve(W, (D.astype(np.float64) * 1.37).astype(np.float32))
    for k in range(len(W)):
        # fp32 rounding of d*c perturbs each term by <= 2^-24 relative
        if oracle.rel_gap(base["best_obj"][k], base["runner_obj"][k]) > 1e-6:
            assert sc["best_bits"][k] == base["best_bits"][k]


def test_bounds_absmax_single_env_and_added_env(groups128):
    W, D = groups128
    base = oracle.solve(W, D)
    for k in range(len(W)):
        ab = oracle.absmax_scale(W[k])
        if ab:
            f_ab, _, _ = oracle.objective(W[k], D[:, k, :], ab)
            assert base["best_obj"][k] <= f_ab
    singles = [oracle.solve(W, D[e:e + 1]) for e in range(D.shape[0])]
    lower = np.max([s["best_obj"] for s in singles], axis=0)
    assert np.all(base["best_obj"] >= lower)
    three = oracle.solve(W, D[:3])
    assert np.all(base["best_obj"] >= three["best_obj"])


def test_weight_permutation(groups128):
    W, D = groups128
    rng = np.random.default_rng(2)
    perm = rng.permutation(128)
    base = oracle.solve(W, D)
    pr = oracle.solve(W[:, perm], D[:, :, perm])
    for k in range(len(W)):
        if oracle.rel_gap(base["best_obj"][k], base["runner_obj"][k]) > NEAR_TIE:
            assert pr["best_bits"][k] == base["best_bits"][k]
            assert np.array_equal(pr["codes"][k], base["codes"][k][perm])
        assert rel(pr["best_obj"][k], base["best_obj"][k]) <= NEAR_TIE


def test_per_column_and_per_group_layouts_agree():
    rng = np.random.default_rng(8)
    K, R, E = 384, 2, 3
    W = f16bits(rng.normal(0, 0.02, (R, K))).reshape(-1, 128)
    Dc = rng.lognormal(0, 1, (E, K)).astype(np.float32)
    gpr = K // 128
    Dg = np.stack([Dc[:, (g % gpr) * 128:(g % gpr) * 128 + 128] for g in range(W.shape[0])], axis=1)
    a = oracle.solve(W, Dc, K=K)
    b = oracle.solve(W, Dg)
    for k in a:
        assert np.array_equal(a[k], b[k])
    sel = np.array([4, 1])
    c = oracle.solve(W, Dc, K=K, sel=sel)
    assert np.array_equal(c["best_bits"], a["best_bits"][sel])


@pytest.mark.parametrize("seed", [0, 1])
def test_full_group_against_exact(seed):
    """One realistic 128-weight, E=4 group against the exact integer brute force."""
    rng = np.random.default_rng(100 + seed)
    w = f16bits(rng.normal(0, 0.02, 128) * np.where(rng.random(128) < 0.05, 8, 1))
    d = rng.lognormal(0, 1.5, (4, 128)).astype(np.float32)
    x = exact.solve(w, d)
    o = solve1(w, d)
    assert rel(o["best_obj"], x["best"]) <= 1e-13
    if oracle.rel_gap(float(x["best"]), float(x["runner"])) > NEAR_TIE:
        assert o["best_bits"] == x["best_bits"]
        assert np.array_equal(o["codes"], x["codes"])
