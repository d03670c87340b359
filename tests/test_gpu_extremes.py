"""Both GPU selection paths at the ends of the input range, against the oracle.

Every finite fp32 d >= 0 and every finite binary16 weight is a valid input.
The fp32 screens of both kernels rest on relative rounding bounds, which hold
only while no fp32 value overflows or falls below the normal range.  These
cases put the per-environment sums sum d w^2 far above FLT_MAX (d up to
FLT_MAX, weights up to 65504) and the terms d r^2 below 2^-126 (subnormal and
tiny d), alone and mixed across environments and weights, so a kernel must
route such groups to its fp64 path to stay exact.  CQ_EXTREME_SEEDS ("N" or
"A:B") widens the seed range for a longer campaign."""
import numpy as np
import pytest

import oracle
from parity import check_against_oracle, oracle_threads, run_gpu, seed_range

pytestmark = pytest.mark.gpu

FLT_MAX = float(np.finfo(np.float32).max)


def f16bits(x):
    return np.clip(np.asarray(x, dtype=np.float64), -65504, 65504).astype(np.float16).view(np.uint16)


def extreme_inputs(seed, G=48, E=4):
    """[G,128] weights and [E,G,128] diagonals in six classes of G/6 groups."""
    rng = np.random.default_rng(seed)
    W = np.empty((G, 128), dtype=np.uint16)
    D = np.empty((E, G, 128), dtype=np.float64)
    k = G // 6
    for c in range(6):
        sl = slice(c * k, (c + 1) * k if c < 5 else G)
        n = W[sl].shape[0]
        w = rng.normal(0, 0.02, (n, 128)) * 10.0 ** rng.uniform(-2, 5.5, (n, 1))
        d = rng.lognormal(0, 1.0, (E, n, 128))
        if c == 0:    # huge d on every environment: sum d w^2 far above FLT_MAX
            d *= 2.0 ** rng.uniform(100, 126, (E, n, 1))
        elif c == 1:  # tiny and subnormal d: terms d r^2 below 2^-126
            d *= 2.0 ** rng.uniform(-148, -90, (E, n, 1))
        elif c == 2:  # one environment each: huge, tiny, ordinary, zero
            d[0] *= 2.0 ** 120
            d[1] *= 2.0 ** -140
            if E > 3:
                d[3] = 0.0
        elif c == 3:  # tiny d on a random half of the weights only
            d *= np.where(rng.random((E, n, 128)) < 0.5, 2.0 ** -130, 1.0)
        elif c == 4:  # extreme weights: +-65504 beside 2^-24 multiples, ordinary d
            w = np.where(rng.random((n, 128)) < 0.1, np.sign(w) * 65504.0,
                         rng.integers(-40, 40, (n, 128)) * 2.0 ** -24)
        else:         # d at FLT_MAX exactly on some weights
            d = np.where(rng.random((E, n, 128)) < 0.05, FLT_MAX, d)
        W[sl] = f16bits(w)
        D[:, sl, :] = np.minimum(d, FLT_MAX)
    return W, D.astype(np.float32)


@pytest.mark.parametrize("seed", seed_range("CQ_EXTREME_SEEDS", 2))
def test_fast_path_extremes(seed):
    W, D = extreme_inputs(4100 + seed)
    assert np.all(np.isfinite(D)) and np.all(D >= 0)
    gpu = run_gpu(W, D)
    check_against_oracle(W, D, gpu, where=f"extremes seed {seed}")


@pytest.mark.parametrize("seed", seed_range("CQ_EXTREME_SEEDS", 2))
def test_general_kernel_extremes_w4_spec(seed):
    """The general kernel at (-8, 7, 128) on the same extreme inputs, bit-exact."""
    import torch
    from minimax_scale_search_b200 import cq
    W, D = extreme_inputs(4100 + seed)
    r = cq.select_scales_spec(torch.from_numpy(W.view(np.int16)).cuda(), torch.from_numpy(D).cuda(),
                              want_objective=True, want_flags=True, general_kernel=True)
    torch.cuda.synchronize()
    o = oracle.solve(W, D, threads=oracle_threads())
    s = r.scales.cpu().numpy().view(np.uint16)
    bad = np.nonzero(s != o["best_bits"])[0]
    assert bad.size == 0, (seed, bad[:8])
    assert np.array_equal(r.codes.cpu().numpy(), o["codes"])


@pytest.mark.parametrize("qmin,qmax,n", [(-8, 7, 128), (-4, 3, 128), (-8, 7, 64)])
def test_general_path_extremes(qmin, qmax, n):
    import torch
    from minimax_scale_search_b200 import cq
    W, D = extreme_inputs(4200 + n + qmax)
    if n != 128:
        W = W.reshape(-1, n)
        D = D.reshape(D.shape[0], -1, n)
    r = cq.select_scales_spec(torch.from_numpy(W.view(np.int16)).cuda(), torch.from_numpy(D).cuda(),
                              qmin=qmin, qmax=qmax, group_size=n, want_objective=True, want_flags=True)
    torch.cuda.synchronize()
    o = oracle.solve(W, D, qmin=qmin, qmax=qmax, threads=oracle_threads())
    s = r.scales.cpu().numpy().view(np.uint16)
    bad = np.nonzero(s != o["best_bits"])[0]
    assert bad.size == 0, (bad[:8], s[bad[:8]], o["best_bits"][bad[:8]])
    assert np.array_equal(r.codes.cpu().numpy(), o["codes"][:, :n])
    live = r.flags.cpu().numpy() == 0
    assert np.array_equal(r.objective.cpu().numpy()[live].view(np.uint64), o["best_obj"][live].view(np.uint64))
