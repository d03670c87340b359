"""GPU parity of the general-spec path (csrc/cq_spec.cu) against the oracle.

Every value the kernel compares is the definition's own fp64 objective, the
same arithmetic in the same order as the oracle, and the minimum is taken by
(objective, pattern) like the oracle's ascending strict-< scan.  So scales,
codes and objectives must agree bit for bit in every group, near ties
included: a stronger bar than the main kernel's near-tie rule."""
import numpy as np
import pytest

import oracle
from minimax_scale_search_b200 import synth
from parity import oracle_threads

pytestmark = pytest.mark.gpu


def _run(W, D, qmin, qmax, n, K=None):
    import torch
    from minimax_scale_search_b200 import cq
    Wt = torch.from_numpy(np.ascontiguousarray(W).view(np.int16)).cuda()
    Dt = torch.from_numpy(np.ascontiguousarray(D, dtype=np.float32)).cuda()
    r = cq.select_scales_spec(Wt, Dt, K, qmin=qmin, qmax=qmax, group_size=n, want_objective=True,
                              want_flags=True)
    torch.cuda.synchronize()
    return (r.scales.cpu().numpy().view(np.uint16), r.codes.cpu().numpy(), r.objective.cpu().numpy(),
            r.flags.cpu().numpy())


def _check(W, D, qmin, qmax, n, K=0, where=""):
    """W [G, n] (or [R, K] when K > 0); D per group [E, G, n] or per column [E, K]."""
    s, c, f, fl = _run(W, D, qmin, qmax, n, K or None)
    Wg = np.ascontiguousarray(W).reshape(-1, n)
    o = oracle.solve(Wg, D, K=K, qmin=qmin, qmax=qmax, threads=oracle_threads())
    bad = np.nonzero(s != o["best_bits"])[0]
    assert bad.size == 0, (where, bad[:5], s[bad[:5]], o["best_bits"][bad[:5]])
    assert np.array_equal(c, o["codes"][:, :n]), where
    live = fl == 0
    assert np.array_equal(f[live].view(np.uint64), o["best_obj"][live].view(np.uint64)), where
    return s, c, f, fl


def _groups(G, n, sigma=0.02, seed=0, outliers=0.03):
    rng = np.random.default_rng(seed)
    w = rng.normal(0, sigma, (G, n)) * np.where(rng.random((G, n)) < outliers, 8.0, 1.0)
    return w.astype(np.float16).view(np.uint16)


def _diag(E, G, n, seed=1, sigma=1.5):
    rng = np.random.default_rng(seed)
    d = rng.lognormal(0, sigma, (E, G, n))
    return (d / d.mean(axis=2, keepdims=True)).astype(np.float32)


@pytest.mark.parametrize("spec", [(-4, 3), (-2, 1), (-1, 1), (-16, 15), (-128, 127), (-8, 8)])
def test_other_code_ranges(spec):
    qmin, qmax = spec
    W = _groups(96, 128, seed=abs(qmin) + qmax)
    D = _diag(4, 96, 128, seed=qmax)
    _check(W, D, qmin, qmax, 128, where=f"spec {spec}")


@pytest.mark.parametrize("n,E", [(1, 2), (32, 1), (64, 4), (100, 3), (256, 8), (1024, 2), (1024, 8)])
def test_other_group_sizes(n, E):
    G = max(8, 4096 // n)
    W = _groups(G, n, seed=n)
    D = _diag(E, G, n, seed=n + 1)
    _check(W, D, -8, 7, n, where=f"n={n}")
    if n in (64, 256):
        _check(W, D, -4, 3, n, where=f"n={n} W3")


def test_default_spec_matches_oracle_including_near_ties():
    """(-8, 7, 128) through the general path on the stress workload's exact
    multiples, zero and single-nonzero groups (many exact ties) and gaussian
    groups, per-column diagonals with E = 8."""
    cls = synth.stress_classes()
    pick = np.sort(np.concatenate([np.nonzero(cls == c)[0][:40] for c in range(5)]))
    Wg, Dg = synth.group_rows(4, pick)
    s, _, _, fl = _check(Wg, Dg, -8, 7, 128, where="stress")
    assert np.any(fl == 1)  # the all-zero class is flagged trivial


def test_per_column_layout_and_edge_groups():
    wl = synth.workload(1)
    W = synth.make_weights(1)
    D = synth.make_diagonals(1)
    _check(W, D, -4, 3, 128, K=wl.cols, where="per-column W3")
    _check(W, D, -8, 7, 64, K=wl.cols, where="per-column n=64")
    # non-finite and zero groups: scale 0x0001, zero codes, flagged
    Wb = _groups(6, 64, seed=3)
    Wb[1, 5] = 0x7C00
    Wb[2, :] = 0
    Wb[3, 0] = 0xFE00
    s, c, f, fl = _run(Wb, _diag(2, 6, 64), -4, 3, 64)
    assert list(fl[:4]) == [0, 8, 1, 8]
    assert np.all(s[1:4] == 1) and np.all(c[1:4] == 0) and np.all(f[1:4] == 0)


def _run_kernel(W, D, qmin, qmax, n, K, general):
    import torch
    from minimax_scale_search_b200 import cq
    Wt = torch.from_numpy(np.ascontiguousarray(W).view(np.int16)).cuda()
    Dt = torch.from_numpy(np.ascontiguousarray(D, dtype=np.float32)).cuda()
    r = cq.select_scales_spec(Wt, Dt, K, qmin=qmin, qmax=qmax, group_size=n, want_objective=True,
                              want_flags=True, general_kernel=general)
    torch.cuda.synchronize()
    return (r.scales.cpu().numpy().view(np.uint16), r.codes.cpu().numpy(), r.objective.cpu().numpy(),
            r.flags.cpu().numpy())


@pytest.mark.parametrize("n,spec", [(n, sp) for n in (128, 64)
                                     for sp in ((-8, 7), (-4, 3), (-2, 1), (-1, 1), (-8, 8), (-5, 4))] +
                         [(128, sp) for sp in ((-16, 15), (-16, 16), (-12, 11), (-9, 8))])
def test_w4_search_and_general_kernel_same_bytes(spec, n):
    """Group size 128 or 64 with |qmin| = qmax or qmax + 1 runs the W4
    kernel's search; the general kernel is the other implementation of the
    same definition.  On the first 2,048 sweep rows (262,144 groups of 128,
    524,288 of 64) every scale, code, objective and flag is the same, and a
    sample meets the oracle."""
    qmin, qmax = spec
    wl = synth.workload(3)
    W = synth.make_weights(3, 0, 2048)
    D = synth.make_diagonals(3)
    a = _run_kernel(W, D, qmin, qmax, n, wl.cols, general=False)
    b = _run_kernel(W, D, qmin, qmax, n, wl.cols, general=True)
    for x, y, name in zip(a, b, ("scales", "codes", "objective", "flags")):
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), (spec, n, name)
    G = W.size // n
    sel = np.sort(np.random.default_rng(29 + n).choice(G, 600, replace=False))
    gpr = wl.cols // n
    Wg = W.reshape(-1, n)[sel]
    Dg = np.ascontiguousarray(D.reshape(4, gpr, n)[:, sel % gpr, :])
    o = oracle.solve(Wg, Dg, qmin=qmin, qmax=qmax, threads=oracle_threads())
    assert np.array_equal(a[0][sel], o["best_bits"]), (spec, n)
    assert np.array_equal(a[1][sel], o["codes"][:, :n]), (spec, n)
    assert np.array_equal(a[2][sel].view(np.uint64), o["best_obj"].view(np.uint64)), (spec, n)


@pytest.mark.parametrize("E", [1, 2, 3, 5, 8])
def test_w4_search_each_environment_count(E):
    for n in (128, 64):
        W = _groups(160, n, seed=200 + E)
        D = _diag(E, 160, n, seed=300 + E, sigma=2.0)
        specs = ((-4, 3), (-2, 1), (-8, 8), (-8, 7)) + (((-16, 15), (-16, 16)) if n == 128 else ())
        for qmin, qmax in specs:
            _check(W, D, qmin, qmax, n, where=f"E={E} n={n} spec ({qmin}, {qmax})")


def test_w4_search_sixteen_layers_stress():
    """Code ranges of 16 layers at group size 128 (their own merge network) on
    the tie/stress workload's classes, with E = 8."""
    cls = synth.stress_classes()
    pick = np.sort(np.concatenate([np.nonzero(cls == c)[0][:40] for c in range(5)]))
    Wg, Dg = synth.group_rows(4, pick)
    _check(Wg, Dg, -16, 15, 128, where="stress (-16, 15)")
    _check(Wg, Dg, -12, 11, 128, where="stress (-12, 11)")


def test_w4_search_group64_stress_and_edges():
    """Group size 64 on the tie/stress workload's classes (exact multiples,
    zero and single-nonzero halves of groups) and on edge groups."""
    cls = synth.stress_classes()
    pick = np.sort(np.concatenate([np.nonzero(cls == c)[0][:40] for c in range(5)]))
    Wg, Dg = synth.group_rows(4, pick)
    W64 = np.ascontiguousarray(Wg.reshape(-1, 64))
    D64 = np.ascontiguousarray(Dg.reshape(Dg.shape[0], -1, 64))
    _check(W64, D64, -8, 7, 64, where="stress n=64")
    Wb = _groups(6, 64, seed=3)
    Wb[1, 5] = 0x7C00
    Wb[2, :] = 0
    Wb[3, 0] = 0xFE00
    s, c, f, fl = _run(Wb, _diag(2, 6, 64), -8, 7, 64)
    assert list(fl[:4]) == [0, 8, 1, 8]
    assert np.all(s[1:4] == 1) and np.all(c[1:4] == 0) and np.all(f[1:4] == 0)
