"""GPU parity of the diagonal estimation (csrc/cq_diag.cu) against the
oracle's correctly rounded version (oracle/diagonals.py).

Tolerance, from the kernel's summation order: each of the 64 row slots of an
(environment, column) sums about N/64 exact squares sequentially in fp64, then
8 warp and 8 CTA partials are added in order, then one division: at most
N/64 + 17 roundings of non-negative terms, so the relative error of a mean is
below (N/64 + 17) * 2^-53.  D is m / mean(m) rounded once to fp32 on both sides
from fp64 values that agree to ~1e-14, so the two may differ by one fp32 ulp."""
import numpy as np
import pytest

from oracle import diagonals as OD
from minimax_scale_search_b200 import synth

pytestmark = pytest.mark.gpu


def _run(X, offsets, dtype):
    import torch
    from minimax_scale_search_b200 import cq
    Xt = torch.from_numpy(X.view(np.int16) if X.dtype == np.uint16 else X).cuda()
    means, D = cq.estimate_diagonals(Xt, offsets, dtype=dtype)
    return means.cpu().numpy(), D.cpu().numpy()


def _compare(X, offsets, dtype):
    m_gpu, d_gpu = _run(X, offsets, dtype)
    m_or, d_or = OD.estimate(X, dtype, offsets)
    n_max = int(np.max(np.diff(offsets))) if len(offsets) > 1 else 0
    tol = (n_max / 64 + 17) * 2.0 ** -53
    nan = np.isnan(m_or)
    assert np.array_equal(np.isnan(m_gpu), nan)
    rel = np.abs(m_gpu[~nan] - m_or[~nan]) / np.maximum(m_or[~nan], np.finfo(np.float64).tiny)
    assert np.all((rel <= tol) | (m_or[~nan] == m_gpu[~nan])), rel.max()
    dnan = np.isnan(d_or)
    assert np.array_equal(np.isnan(d_gpu), dnan)
    ulp = np.spacing(np.abs(d_or[~dnan]))
    assert np.all(np.abs(d_gpu[~dnan].astype(np.float64) - d_or[~dnan]) <= ulp)
    return m_gpu, d_gpu


@pytest.mark.parametrize("dtype", [OD.BF16, OD.FP16, OD.FP32])
@pytest.mark.parametrize("tokens,K", [([1], 8), ([63, 64, 65], 264), ([0, 300, 1], 512), ([257] * 8, 136),
                                       ([1000, 1500, 777, 2048], 1024)])
def test_diagonals_match_oracle(tokens, K, dtype):
    X, off = synth.make_activations(tokens, K, dtype=dtype, seed=len(tokens) * 100 + K)
    _compare(X, off, dtype)


def test_diagonals_large_bf16_and_deterministic():
    X, off = synth.make_activations([4096, 3000, 5000, 4096], 4096, dtype=OD.BF16, seed=9)
    m1, d1 = _compare(X, off, OD.BF16)
    m2, d2 = _run(X, off, OD.BF16)
    assert np.array_equal(m1.view(np.uint64), m2.view(np.uint64)) and np.array_equal(d1.view(np.uint32), d2.view(np.uint32))
    assert np.all(np.abs(d1.astype(np.float64).mean(axis=1) - 1.0) < 1e-5)


def test_zero_activations_and_empty_environment_give_nan():
    X = np.zeros((50, 256), dtype=np.float32)
    m, d = _run(X, np.array([0, 0, 50]), OD.FP32)
    assert np.all(np.isnan(m[0])) and np.all(np.isnan(d[0]))
    assert np.all(m[1] == 0.0) and np.all(np.isnan(d[1]))
