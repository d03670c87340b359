"""Seeded random small cases for both GPU selection paths against the oracle:
random E (1..8), diagonal layout (per column or per group), group counts that
are not multiples of the CTA's warps, weight scales from 1e-6 to 1e3, sparse,
heavy-tailed and exact-multiple weight patterns, lognormal and zero-heavy
diagonals.  The W4/G128 path follows the selection's parity rule; the
general-spec path (random code ranges and group sizes) is bit-exact.
CQ_FUZZ_FAST_SEEDS and CQ_FUZZ_GENERAL_SEEDS ("N" or "A:B") widen the seed
ranges for a longer campaign."""
import numpy as np
import pytest

import oracle
from parity import check_against_oracle, groups_and_diag, oracle_threads, run_gpu, seed_range

pytestmark = pytest.mark.gpu


def f16bits(x):
    return np.clip(np.asarray(x, dtype=np.float64), -65504, 65504).astype(np.float16).view(np.uint16)


def random_weights(rng, G, n):
    kind = rng.integers(0, 4)
    scale = 10.0 ** rng.uniform(-6, 3)
    if kind == 0:
        w = rng.normal(0, scale, (G, n))
    elif kind == 1:
        w = scale * rng.standard_t(2, (G, n))
    elif kind == 2:
        w = rng.normal(0, scale, (G, n)) * (rng.random((G, n)) < 0.1)
    else:
        step = np.ldexp(1.0 + rng.integers(0, 128) / 128.0, int(rng.integers(-20, 0)))
        w = rng.integers(-8, 8, (G, n)) * step
    return f16bits(w)


def random_diagonals(rng, E, shape):
    d = rng.lognormal(0, rng.uniform(0.3, 2.5), (E,) + shape)
    if rng.random() < 0.3:
        d *= rng.random((E,) + shape) < 0.5  # many zero diagonals
    return d.astype(np.float32)


@pytest.mark.parametrize("seed", seed_range("CQ_FUZZ_FAST_SEEDS", 12))
def test_fast_path_fuzz(seed):
    rng = np.random.default_rng(1000 + seed)
    E = int(rng.integers(1, 9))
    if rng.random() < 0.5:
        gpr = int(rng.integers(1, 5))
        rows = int(rng.integers(1, 12))
        K = 128 * gpr
        W = random_weights(rng, rows * gpr, 128).reshape(rows, K)
        D = random_diagonals(rng, E, (K,))
        gpu = run_gpu(W, D, K)
        Wg, Dg = groups_and_diag(W, D, K)
    else:
        G = int(rng.integers(1, 45))
        W = random_weights(rng, G, 128)
        D = random_diagonals(rng, E, (G, 128))
        gpu = run_gpu(W, D)
        Wg, Dg = W, D
    check_against_oracle(Wg, Dg, gpu, where=f"fuzz seed {seed} E={E}")


@pytest.mark.parametrize("seed", seed_range("CQ_FUZZ_GENERAL_SEEDS", 10))
def test_general_path_fuzz(seed):
    import torch
    from minimax_scale_search_b200 import cq
    rng = np.random.default_rng(2000 + seed)
    E = int(rng.integers(1, 9))
    qmax = int(rng.choice([1, 2, 3, 7, 15, 31, 127]))
    qmin = -qmax - int(rng.integers(0, 2))
    n = int(rng.choice([8, 16, 33, 64, 128, 200]))
    G = int(rng.integers(1, 30))
    W = random_weights(rng, G, n)
    D = random_diagonals(rng, E, (G, n))
    r = cq.select_scales_spec(torch.from_numpy(W.view(np.int16)).cuda(), torch.from_numpy(D).cuda(),
                              qmin=qmin, qmax=qmax, group_size=n, want_objective=True, want_flags=True)
    torch.cuda.synchronize()
    o = oracle.solve(W, D, qmin=qmin, qmax=qmax, threads=oracle_threads())
    s = r.scales.cpu().numpy().view(np.uint16)
    assert np.array_equal(s, o["best_bits"]), (seed, qmin, qmax, n, E)
    assert np.array_equal(r.codes.cpu().numpy(), o["codes"][:, :n])
    live = r.flags.cpu().numpy() == 0
    assert np.array_equal(r.objective.cpu().numpy()[live].view(np.uint64), o["best_obj"][live].view(np.uint64))
