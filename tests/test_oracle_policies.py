"""Pins for the oracle's comparison policies and reconstruction proxy
(oracle/policies.py), against values fixed by the definitions and by exact
arithmetic, not by the module itself.

CliffQuant project page, "Held-out reconstruction proxy": the policies are
CliffQuant (exact minimax), Pooled-WMSE (environments averaged first) and
AbsMax (fp16(max|w|/7)); the proxy is the module-macro worst-environment
weighted MSE.  Each ``check_*`` takes the policies module so that the mutant
test can run the same checks against a copy with one planted mistake.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact
from oracle import policies as P

F32_MANT = 24


def f16bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def fraction_to_f32(x: Fraction) -> np.float32:
    """Round an exact rational to the nearest fp32, ties to even (normal and
    subnormal range), by integer arithmetic."""
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** max(e - (F32_MANT - 1), -149)
    m = a / ulp
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return np.float32(sign * float(fl * ulp))


# ----------------------------------------------------------------- pooling

def check_pool_identities(P):
    rng = np.random.default_rng(11)
    x = rng.lognormal(0, 3, (1, 300)).astype(np.float32)
    assert np.array_equal(P.pool_diagonals(x), x)
    for E in (2, 3, 5, 6, 7, 8):  # the mean of E equal values is that value
        assert np.array_equal(P.pool_diagonals(np.repeat(x, E, axis=0)), x)


def check_pool_exact(P):
    rng = np.random.default_rng(12)
    for E in (2, 4, 8):  # fp64 sum exact (spread < 2^25) and /E exact: one rounding
        D = (2.0 ** rng.uniform(-12, 12, (E, 200)) * rng.uniform(1, 2, (E, 200))).astype(np.float32)
        got = P.pool_diagonals(D)[0]
        exp = [fraction_to_f32(sum(Fraction(float(v)) for v in D[:, i]) / E) for i in range(D.shape[1])]
        assert np.array_equal(got, np.array(exp, dtype=np.float32)), E
    for E in (3, 5, 6, 7):  # integer sums below 2^24: fp32 operands, so fp64 then fp32 is one rounding
        D = rng.integers(0, 1 << 21, (E, 200)).astype(np.float32)
        got = P.pool_diagonals(D)[0]
        exp = [fraction_to_f32(Fraction(int(D[:, i].astype(np.int64).sum()), E)) for i in range(D.shape[1])]
        assert np.array_equal(got, np.array(exp, dtype=np.float32)), E
    # an fp32 running sum would lose both 2^-24 terms: (1 + 2^-23) / 4 = 2^-2 + 2^-25 exactly
    D = np.array([[1.0], [2.0 ** -24], [2.0 ** -24], [0.0]], dtype=np.float32)
    assert P.pool_diagonals(D)[0, 0] == np.float32(0.25 + 2.0 ** -25)
    assert P.pool_diagonals(D[:, None, :]).shape == (1, 1, 1)


# ------------------------------------------------------------------ AbsMax

def check_absmax_worked_example(P):
    w = np.zeros(128)
    w[:6] = [-7.0, 2.5, 3.5, 0.5, -1.5, 6.75]
    s, c = P.absmax_policy(f16bits(w)[None])
    assert int(s[0]) == 0x3C00  # 7 / 7 = 1.0
    q = np.zeros(128, np.int8)
    q[:6] = [-7, 2, 4, 0, -2, 7]  # round half to even: 2.5 -> 2, 3.5 -> 4, 0.5 -> 0, -1.5 -> -2
    assert np.array_equal(c[0], oracle.pack_codes(q))


def check_absmax_degenerate(P):
    z = np.zeros((1, 128), dtype=np.uint16)
    s, c = P.absmax_policy(z)
    assert int(s[0]) == 0x0001 and np.all(c == 0x88888888)
    tiny = z.copy()
    tiny[0, 5] = 0x0001  # 2^-24 / 7 rounds to zero: raised to the smallest scale
    s, c = P.absmax_policy(tiny)
    assert int(s[0]) == 0x0001
    assert (int(c[0, 0]) >> 20) & 0xF == 9  # w = s: code 1 at index 5
    for bad in (0x7C00, 0xFC00, 0x7E00):
        g = f16bits(np.linspace(-1, 1, 128))[None].copy()
        g[0, 3] = bad
        s, c = P.absmax_policy(g)
        assert int(s[0]) == 0x0001 and np.all(c == 0x88888888)


def check_absmax_random(P):
    rng = np.random.default_rng(13)
    W = f16bits(rng.normal(0, 0.02, (40, 128)) * np.where(rng.random((40, 128)) < 0.03, 20, 1))
    s, c = P.absmax_policy(W)
    vals = W.view(np.float16).astype(np.float64)
    amax = np.abs(vals).max(axis=1)
    assert np.array_equal(s, (amax / 7.0).astype(np.float16).view(np.uint16))  # numpy's own RNE
    for g in range(40):
        q = oracle.objective(W[g], np.ones((1, 128), np.float32), int(s[g]))[2]
        assert np.array_equal(c[g], oracle.pack_codes(q))
        k = int(np.argmax(np.abs(vals[g])))
        assert abs(int(q[k])) == 7  # s is within 2^-11 of amax/7, so amax/s rounds to 7


# --------------------------------------------------------------- objective

def check_objectives_exact(P):
    rng = np.random.default_rng(14)
    W = f16bits(rng.normal(0, 0.03, (2, 128)))
    D = rng.lognormal(0, 1, (2, 2, 128)).astype(np.float32)
    scales = np.array([0x2300, 0x2A10], dtype=np.uint16)
    got = P.group_objectives(W, D, 0, scales)
    assert got.shape == (2, 2)
    for g in range(2):
        for e in range(2):
            f, _ = exact.objective_at(W[g], D[e:e + 1, g, :], int(scales[g]))
            assert abs(got[g, e] - float(f)) <= 2.0 ** -45 * float(f)


def check_objective_layouts(P):
    rng = np.random.default_rng(15)
    K, rows, E = 384, 2, 3
    W = f16bits(rng.normal(0, 0.02, (rows, K))).reshape(-1, 128)
    G = W.shape[0]
    Dc = rng.lognormal(0, 1, (E, K)).astype(np.float32)
    Dg = np.stack([Dc[:, (g % (K // 128)) * 128:(g % (K // 128)) * 128 + 128] for g in range(G)], axis=1)
    scales = f16bits(np.abs(rng.normal(0, 0.004, G)) + 1e-4)
    assert np.array_equal(P.group_objectives(W, Dc, K, scales), P.group_objectives(W, Dg, 0, scales))
    # group 4 is row 1, column block 1: its diagonal starts at column 128
    assert np.array_equal(P.group_diagonal(Dc, K, 4, G), Dc[:, 128:256])


# ------------------------------------------------------------------- proxy

def check_proxy_worked_example(P):
    per_env = np.array([[1.0, 4.0], [3.0, 0.0], [8.0, 2.0]])
    env, worst, macro = P.reconstruction_proxy(per_env, [0, 2, 3], scale=1.0)
    assert np.array_equal(env, [[2.0, 2.0], [8.0, 2.0]])
    assert np.array_equal(worst, [2.0, 8.0])
    assert macro == 5.0  # the mean of per-group maxima would give (3.5 + 8) / 2 = 5.75
    env, worst, macro = P.reconstruction_proxy(per_env, [0, 2, 3])
    assert macro == 5.0 / 128  # per-weight mean by default
    env, worst, macro = P.reconstruction_proxy(per_env, [0, 0, 3], scale=1.0)
    assert np.isnan(worst[0]) and worst[1] == 4.0 and np.isnan(macro)


# ---------------------------------------------------------- pooled policy

def check_pooled_policy(P):
    from test_oracle_pins import make_groups128
    W, D = make_groups128()
    cq = oracle.solve(W, D)["best_bits"]
    pooled = P.pooled_policy(W, D)
    assert np.array_equal(P.pooled_policy(W, D[:1]), oracle.solve(W, D[:1])["best_bits"])
    assert np.array_equal(P.pooled_policy(W, np.repeat(D[:1], 3, axis=0)), oracle.solve(W, D[:1])["best_bits"])
    absm, _ = P.absmax_policy(W)
    Dp = P.pool_diagonals(D)
    for g in range(W.shape[0]):
        f = [oracle.objective(W[g], D[:, g, :], int(s))[0] for s in (cq[g], pooled[g], absm[g])]
        assert f[0] <= f[1] and f[0] <= f[2]  # minimax is the minimum of the worst environment
        fp = [oracle.objective(W[g], Dp[:, g, :], int(s))[0] for s in (cq[g], pooled[g])]
        assert fp[1] <= fp[0]  # pooled is the minimum of the pooled objective
    assert not np.array_equal(cq, pooled)  # the two policies do differ on these groups


CHECKS = (check_pool_identities, check_pool_exact, check_absmax_worked_example, check_absmax_degenerate,
          check_absmax_random, check_objectives_exact, check_objective_layouts, check_proxy_worked_example,
          check_pooled_policy)


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_policies_pin(check):
    check(P)


def test_fraction_to_f32_matches_numpy_on_doubles():
    rng = np.random.default_rng(16)
    xs = np.concatenate([rng.lognormal(0, 20, 3000), 2.0 ** rng.uniform(-150, -120, 500)])
    for x in xs:
        assert fraction_to_f32(Fraction(float(x))) == np.float32(x)
