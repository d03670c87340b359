"""Pins for the oracle's diagonal estimation (oracle/diagonals.py): closed
forms, invariants and exact small cases, not the module itself.  Each
``check_*`` takes the module so that the mutant test can reuse it."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import diagonals as OD
from minimax_scale_search_b200 import synth


def check_decode(D):
    x = np.array([1.0, -2.5, 3.0e-39, 6.0e4, 1.0 / 3.0], dtype=np.float32)  # includes an fp32 subnormal
    bf = synth.to_bf16_bits(x)
    assert np.array_equal(D.decode(bf, D.BF16), (bf.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    assert D.decode(np.array([0x3F80], np.uint16), D.BF16)[0] == 1.0
    assert D.decode(np.array([0xC020], np.uint16), D.BF16)[0] == -2.5
    assert D.decode(np.array([0x3C00, 0x0001], np.uint16), D.FP16).tolist() == [1.0, 2.0 ** -24]
    assert D.decode(x, D.FP32).tolist() == x.astype(np.float64).tolist()


def check_worked_example(D):
    # env 0: rows (1, 2), (3, 0) -> m = (5, 2); env 1: row (2, 2) -> m = (4, 4)
    X = np.array([[1.0, 2.0], [3.0, 0.0], [2.0, 2.0]], dtype=np.float32)
    m, d = D.estimate(X, D.FP32, [0, 2, 3])
    assert m.tolist() == [[5.0, 2.0], [4.0, 4.0]]
    assert d.tolist() == [[np.float32(5.0 / 3.5), np.float32(2.0 / 3.5)], [1.0, 1.0]]


def check_constant_and_invariants(D):
    X, off = synth.make_activations([40, 25, 33], 64, dtype=2, seed=3)
    m, d = D.estimate(X, D.FP32, off)
    assert d.shape == (3, 64) and m.shape == (3, 64)
    # each environment is normalised to mean 1 (within fp32 rounding of each entry)
    assert np.all(np.abs(d.astype(np.float64).mean(axis=1) - 1.0) < 1e-6)
    # a power-of-two rescale of X scales m by its square and leaves d unchanged
    m2, d2 = D.estimate(X * np.float32(4.0), D.FP32, off)
    assert np.array_equal(m2, 16.0 * m) and np.array_equal(d2, d)
    # duplicating every row of an environment leaves m and d unchanged
    a, b = off[1], off[2]
    Xdup = np.concatenate([X[:b], X[a:b], X[b:]])
    off_dup = np.array([0, off[1], off[2] + (b - a), off[3] + (b - a)])
    md, dd = D.estimate(Xdup, D.FP32, off_dup)
    assert np.array_equal(md, m) and np.array_equal(dd, d)
    # environments are separate: dropping env 2 does not change env 0 and 1
    m3, d3 = D.estimate(X[:off[2]], D.FP32, off[:3])
    assert np.array_equal(m3, m[:2]) and np.array_equal(d3, d[:2])
    # constant columns: m = c^2, and d = 1 when every column has the same c
    Xc = np.full((7, 16), 3.0, dtype=np.float32)
    mc, dc = D.estimate(Xc, D.FP32, [0, 7])
    assert np.all(mc == 9.0) and np.all(dc == 1.0)


def check_exact_small(D):
    X, off = synth.make_activations([5, 9], 16, dtype=0, seed=4)
    m, d = D.estimate(X, D.BF16, off)
    x = (X.astype(np.uint32) << 16).view(np.float32)
    for e in range(2):
        a, b = off[e], off[e + 1]
        for k in (0, 7, 15):
            exact = sum(Fraction(float(v)) ** 2 for v in x[a:b, k]) / (b - a)
            assert m[e, k] == float(exact)  # correctly rounded mean of exact squares


def check_degenerate(D):
    X = np.zeros((4, 8), dtype=np.float32)
    m, d = D.estimate(X, D.FP32, [0, 0, 4])
    assert np.all(np.isnan(m[0])) and np.all(np.isnan(d[0]))  # no tokens
    assert np.all(m[1] == 0.0) and np.all(np.isnan(d[1]))     # only zeros


CHECKS = (check_decode, check_worked_example, check_constant_and_invariants, check_exact_small, check_degenerate)


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_diagonals_pin(check):
    check(OD)


def test_to_bf16_bits_rounds_to_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -20, -1.5], dtype=np.float32)
    assert synth.to_bf16_bits(x).tolist() == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xBFC0]
