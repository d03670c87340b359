"""Seeded input generators: shapes, determinism under chunking, recipe stats."""
import numpy as np

from minimax_scale_search_b200 import synth


def test_shapes_and_group_counts():
    assert synth.workload(1).groups == 256
    assert synth.workload(2).groups == 24576
    assert synth.workload(3).groups == 3883008
    assert synth.workload(3).rows * synth.workload(3).cols == 497025024
    assert synth.workload(4).groups == 1048576
    assert synth.workload(5).groups == 14680064
    W, D = synth.make_inputs(1)
    assert W.shape == (64, 512) and W.dtype == np.uint16
    assert D.shape == (4, 512) and D.dtype == np.float32


def test_chunking_does_not_change_values():
    full = synth.make_weights(2, 0, 700)
    parts = np.concatenate([synth.make_weights(2, 0, 100), synth.make_weights(2, 100, 613),
                            synth.make_weights(2, 613, 700)])
    assert np.array_equal(full, parts)
    assert np.array_equal(synth.make_weights(2, 0, 700, threads=1), full)


def test_diagonals_mean_one_per_env():
    for idx in (1, 2, 4):
        D = synth.make_diagonals(idx)
        assert np.all(D > 0)
        assert np.allclose(D.astype(np.float64).mean(axis=1), 1.0, rtol=1e-6)


def test_group_rows_matches_full_matrix():
    W, D = synth.make_inputs(2)
    gs = synth.sample_groups(2, 50, seed=3)
    Wg, Dg = synth.group_rows(2, gs)
    Wf = W.reshape(-1, 128)
    assert np.array_equal(Wg, Wf[gs])
    gpr = 1024 // 128
    for k, g in enumerate(gs):
        c = (g % gpr) * 128
        assert np.array_equal(Dg[:, k, :], D[:, c:c + 128])


def test_stress_classes_recipe():
    cls = synth.stress_classes()
    frac = np.bincount(cls, minlength=5) / len(cls)
    assert np.allclose(frac, [0.65, 0.125, 0.125, 0.05, 0.05], atol=1e-4)
    W = synth.make_weights(4, 0, 16).reshape(-1, 128)
    c = cls[: W.shape[0]]
    assert np.all(W[c == 3] & 0x7FFF == 0)
    assert np.all(((W[c == 4] & 0x7FFF) != 0).sum(axis=1) <= 1)
    vals = W.view(np.float16).astype(np.float64)
    steps = np.array([np.ldexp(1.0 + j / 128.0, p) for p in range(-12, -3) for j in range(128)])
    for g in np.nonzero((c == 1) | (c == 2))[0]:
        m = vals[g][None, :] / steps[:, None]
        ok = np.all((m == np.round(m)) & (m >= -8) & (m <= 7), axis=1)
        assert ok.any()
