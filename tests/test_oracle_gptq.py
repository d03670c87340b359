"""Pins for the oracle's GPTQ v1 export and dequantisation (oracle/gptq.py),
against worked words of the public v1 layout and the round trip to s * q.
Each ``check_*`` takes the module so that the mutant test can reuse it."""
import numpy as np
import pytest

import oracle
from oracle import gptq as Q


def _f16bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def _small_layer(R=16, K=256, seed=41):
    rng = np.random.default_rng(seed)
    q = rng.integers(-8, 8, (R * K // 128, 128)).astype(np.int8)
    scales = _f16bits(np.abs(rng.normal(0, 0.004, R * K // 128)) + 1e-4)
    codes = np.stack([oracle.pack_codes(q[g]) for g in range(q.shape[0])])
    return q, scales, codes, R, K


def check_worked_words(Q):
    R, K = 8, 128
    q = np.zeros((R, 128), dtype=np.int8)
    q[0, :8] = np.arange(-8, 0)      # u = 0..7 on inputs 0..7 of output 0
    q[3, 8:16] = np.arange(0, 8)     # u = 8..15 on inputs 8..15 of output 3
    codes = np.stack([oracle.pack_codes(q[r]) for r in range(R)])
    scales = _f16bits(np.arange(1, R + 1) * 0.25)
    qweight, qzeros, gscales, g_idx = Q.export_v1(scales, codes, R, K)
    assert qweight.shape == (16, 8) and qweight.dtype == np.int32
    w = qweight.view(np.uint32)
    assert w[0, 0] == 0x76543210
    assert w[1, 3] == 0xFEDCBA98
    assert w[0, 1] == 0x88888888  # q = 0 -> u = 8 everywhere else
    assert qzeros.shape == (1, 1) and qzeros.view(np.uint32)[0, 0] == 0x77777777
    assert gscales.shape == (1, 8) and np.array_equal(gscales[0], scales)
    assert np.array_equal(g_idx, np.zeros(128, np.int32))


def check_layout_two_groups_per_row(Q):
    q, scales, codes, R, K = _small_layer()
    qweight, qzeros, gscales, g_idx = Q.export_v1(scales, codes, R, K)
    assert qweight.shape == (K // 8, R) and qzeros.shape == (K // 128, R // 8)
    assert gscales.shape == (K // 128, R) and np.array_equal(g_idx, np.arange(K) // 128)
    # group (r, c) is the selection's group r * (K/128) + c
    for r, c in ((0, 1), (5, 0), (15, 1)):
        g = r * (K // 128) + c
        assert gscales[c, r] == scales[g]
        for i in (0, 7, 8, 127):
            word = qweight.view(np.uint32)[(c * 128 + i) // 8, r]
            assert (word >> (4 * (i % 8))) & 0xF == q[g, i] + 8


def check_round_trip(Q):
    q, scales, codes, R, K = _small_layer(seed=42)
    deq = Q.dequantize_v1(*Q.export_v1(scales, codes, R, K))
    s = scales.view(np.float16).astype(np.float64).reshape(R, K // 128)
    expect = (s[:, :, None] * q.reshape(R, K // 128, 128)).reshape(R, K)
    assert np.array_equal(deq, expect)


def check_unpack(Q):
    q, _, codes, _, _ = _small_layer(seed=43)
    assert np.array_equal(Q.unpack_group_codes(codes).astype(np.int16) - 8, q)


CHECKS = (check_worked_words, check_layout_two_groups_per_row, check_round_trip, check_unpack)


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_gptq_pin(check):
    check(Q)


def test_export_rejects_bad_shapes():
    with pytest.raises(ValueError):
        Q.export_v1(np.zeros(1, np.uint16), np.zeros((1, 16), np.uint32), 4, 128)  # R not a multiple of 8
