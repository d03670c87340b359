"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Rule: scale bit patterns and packed codes identical wherever the oracle's best
and runner-up objectives differ by more than 1e-12 relative or the best is 0;
elsewhere the oracle's objective at the GPU's scale is within 1e-12 of the
oracle minimum.  Full-size workloads are compared on seeded samples plus every
group the kernel flagged (near-tie or exhaustive fallback), and checked on all
groups for code consistency and the AbsMax bound."""
import ctypes

import numpy as np
import pytest

import oracle
import parity as P
from oracle import exactfit
from minimax_scale_search_b200 import synth

pytestmark = pytest.mark.gpu

SAMPLE = 10_000  # seeded groups per full-size workload, besides every flagged group


def f16bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def absmax_bound_ok(Wg, Dg, scales, obj):
    w = np.abs(Wg.view(np.float16).astype(np.float64))
    sab = (w.max(axis=1) / 7.0).astype(np.float16)
    ok = sab.view(np.uint16) > 0
    f_ab = P.objective_np(Wg[ok], Dg[:, ok], sab.view(np.uint16)[ok])
    return np.all(obj[ok] <= f_ab * (1 + 1e-12))


def test_tiny_workload_every_group():
    W, D = synth.make_inputs(1)
    gpu = P.run_gpu(W, D)
    Wg, Dg = P.groups_and_diag(W, D, W.shape[1])
    P.check_against_oracle(Wg, Dg, gpu, where="tiny")
    P.record(synth.workload(1).name, groups=Wg.shape[0], oracle=Wg.shape[0])
    assert np.array_equal(P.recompute_codes(Wg, gpu["scales"]), gpu["codes"])
    assert gpu["counters"]["nonfinite"] == 0
    assert absmax_bound_ok(Wg, Dg, gpu["scales"], gpu["obj"])


def test_projection_workload_every_group():
    """All 24,576 groups of the projection workload meet the oracle."""
    W, D = synth.make_inputs(2)
    gpu = P.run_gpu(W, D)
    gpu2 = P.run_gpu(W, D)
    assert np.array_equal(gpu["scales"], gpu2["scales"]) and np.array_equal(gpu["codes"], gpu2["codes"])
    Wg, Dg = P.groups_and_diag(W, D, W.shape[1])
    P.check_against_oracle(Wg, Dg, gpu, where="projection")
    assert np.array_equal(P.recompute_codes(Wg, gpu["scales"]), gpu["codes"])
    assert absmax_bound_ok(Wg, Dg, gpu["scales"], gpu["obj"])
    s = gpu["scales"]
    assert s.min() >= 0x0001 and s.max() <= 0x7BFF
    flagged = int(np.count_nonzero(gpu["flags"] & (0x02 | 0x04)))
    P.record(synth.workload(2).name, groups=Wg.shape[0], flagged=flagged, oracle=Wg.shape[0])


def _check_full_matrix(idx, matrix, W, D, gpu, n_sample, where):
    """North-star rule on one full-size matrix: every group's codes are the
    codes of its scale; every group with an exact fit (zero objective) has the
    lowest such scale bit for bit (closed form, all groups); the oracle checks a
    seeded sample of n_sample groups plus every group the kernel flagged
    (near-tie or exhaustive fallback) that the closed form does not settle."""
    Wg = W.reshape(-1, 128)
    G = Wg.shape[0]
    for g0 in range(0, G, 1 << 18):
        g1 = min(G, g0 + (1 << 18))
        assert np.array_equal(P.recompute_codes(Wg[g0:g1], gpu["scales"][g0:g1]), gpu["codes"][g0:g1]), where
    s = gpu["scales"]
    assert s.min() >= 0x0001 and s.max() <= 0x7BFF
    assert np.all(D > 0)  # the closed form needs every diagonal positive
    fit = exactfit.lowest_exact_fit(Wg)
    has_fit = fit > 0
    assert np.array_equal(s[has_fit], fit[has_fit]), where
    assert np.all(gpu["obj"][has_fit] == 0.0), where
    flagged = np.nonzero(gpu["flags"] & (0x02 | 0x04))[0]
    sample = synth.sample_groups(idx, n_sample, seed=13, matrix=matrix)
    sel = np.union1d(sample, flagged[~has_fit[flagged]])
    E = D.shape[0]
    gpr = D.shape[1] // 128
    Dsel = np.ascontiguousarray(D.reshape(E, gpr, 128)[:, sel % gpr, :])
    sub = {k: v[sel] for k, v in gpu.items() if k != "counters"}
    P.check_against_oracle(Wg[sel], Dsel, sub, where=where)
    return dict(groups=G, sample=len(sample), flagged=len(flagged), exact_fit=int(has_fit.sum()),
                flagged_by_closed_form=int(has_fit[flagged].sum()), oracle=len(sel))


@pytest.mark.parametrize("idx", [3, 4])
def test_full_size_workload_north_star_rule(idx):
    wl = synth.workload(idx)
    W, D = synth.make_inputs(idx, matrix=0)
    gpu = P.run_gpu(W, D)
    assert W.size // 128 == wl.groups_per_matrix
    c = _check_full_matrix(idx, 0, W, D, gpu, SAMPLE, wl.name)
    if idx == 4:
        cls = synth.stress_classes()
        assert np.all(gpu["scales"][cls == 3] == 1)
        assert np.all(gpu["codes"][cls == 3] == 0x88888888)
        assert gpu["counters"]["trivial"] >= int((cls == 3).sum())
        # every exact-multiple, all-zero and single-nonzero group is settled
        # bit for bit by the closed form
        fit = exactfit.lowest_exact_fit(W.reshape(-1, 128))
        assert np.all(fit[cls != 0] > 0)
    P.record(wl.name, **c)


def test_large_workload_all_matrices_north_star_rule():
    """All 32 matrices run one by one; the 10,000-group sample is spread over
    them (313 or 312 per matrix) and every flagged group of every matrix meets
    the oracle."""
    wl = synth.workload(5)
    per = [SAMPLE // wl.n_matrices + (1 if m < SAMPLE % wl.n_matrices else 0) for m in range(wl.n_matrices)]
    tot = {}
    for m in range(wl.n_matrices):
        W, D = synth.make_inputs(5, matrix=m)
        gpu = P.run_gpu(W, D)
        c = _check_full_matrix(5, m, W, D, gpu, per[m], f"{wl.name} matrix {m}")
        for k, v in c.items():
            tot[k] = tot.get(k, 0) + v
    assert tot["groups"] == wl.groups and tot["sample"] == SAMPLE
    P.record(wl.name, **tot)


@pytest.mark.parametrize("E", [1, 2, 3, 4, 5, 6, 7, 8])
def test_each_environment_count_per_group_layout(E):
    rng = np.random.default_rng(40 + E)
    G = 37  # ragged: not a multiple of the warps per CTA
    W = f16bits(rng.normal(0, 0.02, (G, 128)) * np.where(rng.random((G, 128)) < 0.02, 9, 1))
    D = rng.lognormal(0, 1.5, (E, G, 128)).astype(np.float32)
    gpu = P.run_gpu(W, D)
    P.check_against_oracle(W, D, gpu, where=f"E={E}")


def _edge_groups(rng):
    rows = []
    rows.append(f16bits(rng.normal(0, 1e-6, 128)))                   # subnormal weights
    rows.append(f16bits(np.clip(rng.normal(0, 3000, 128), -65504, 65504)))  # near the top of fp16
    big = np.zeros(128)
    big[5] = 65504.0
    big[9] = -65504.0
    rows.append(f16bits(big))
    one = np.zeros(128)
    one[77] = -8 * 2.0 ** -10
    rows.append(f16bits(one))                                        # single nonzero, q=-8 fits
    one = np.zeros(128)
    one[3] = 8 * 2.0 ** -10
    rows.append(f16bits(one))                                        # single nonzero, positive
    s0 = np.ldexp(1 + 37 / 128, -7)
    rows.append(f16bits(rng.integers(-8, 8, 128) * s0))              # exact fit
    rows.append(f16bits(rng.integers(-4, 4, 128) * s0))              # exact fit at s0 and s0/2
    rows.append(np.zeros(128, np.uint16))                            # all zero
    rows.append(np.full(128, 0x8000, np.uint16))                     # all -0
    halves = rng.integers(0, 16, 128) + 0.5
    rows.append(f16bits(halves * 2.0 ** -9 * rng.choice([-1, 1], 128)))  # RNE ties at s=2^-9
    rows.append(f16bits(rng.normal(0, 0.02, 128)))
    return np.stack(rows)


def test_edge_cases():
    rng = np.random.default_rng(77)
    W = _edge_groups(rng)
    G = W.shape[0]
    E = 3
    D = rng.lognormal(0, 1, (E, G, 128)).astype(np.float32)
    D[0, -1, :64] = 0.0          # zero diagonal columns
    D[1, -2, :] = 0.0            # a whole environment zero in one group
    gpu = P.run_gpu(W, D)
    P.check_against_oracle(W, D, gpu, where="edges")
    assert gpu["scales"][7] == 1 and gpu["scales"][8] == 1
    assert np.all(gpu["codes"][7] == 0x88888888)
    assert gpu["flags"][7] & 0x01 and gpu["flags"][8] & 0x01


def test_nonfinite_inputs_are_flagged_not_trapped():
    import torch
    from minimax_scale_search_b200 import cq
    rng = np.random.default_rng(5)
    W = f16bits(rng.normal(0, 0.02, (6, 128)))
    D = rng.lognormal(0, 1, (2, 6, 128)).astype(np.float32)
    W[0, 3] = 0x7C00            # +inf
    W[1, 0] = 0xFE00            # NaN
    D[0, 2, 5] = -1.0           # negative diagonal
    D[1, 3, 9] = np.nan
    D[0, 4, 0] = np.inf
    gpu = P.run_gpu(W, D)
    for g in range(5):
        assert gpu["flags"][g] & 0x08
        assert gpu["scales"][g] == 1 and np.all(gpu["codes"][g] == 0x88888888)
    assert not (gpu["flags"][5] & 0x08)
    assert gpu["counters"]["nonfinite"] == 5
    P.check_against_oracle(W, D, gpu, sel=[5], where="finite neighbour")
    # the counters call reports the condition as a status
    Wt = torch.from_numpy(W.view(np.int16)).cuda()
    Dt = torch.from_numpy(D).cuda()
    res = cq.select_scales(Wt, Dt)
    host = np.zeros(8, np.uint32)
    st = cq.lib.cq_read_counters(ctypes.c_void_p(res.workspace.data_ptr()), ctypes.c_void_p(host.ctypes.data),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == cq.CQ_ERR_NONFINITE and host[2] == 5
    assert cq.get_status(res.workspace) == cq.CQ_ERR_NONFINITE
    # a finite call on the same workspace resets the status
    res2 = cq.select_scales(Wt[5:6].contiguous(), Dt[:, 5:6].contiguous(), workspace=res.workspace)
    assert cq.get_status(res2.workspace) == cq.CQ_OK


def test_exhaustive_path_matches_oracle_bit_for_bit():
    """The fallback evaluates every scale in the oracle's own order, so even
    near-ties resolve identically."""
    rng = np.random.default_rng(9)
    G = 24
    W = f16bits(rng.normal(0, 0.02, (G, 128)))
    W[3] = f16bits(rng.integers(-4, 4, 128) * 2.0 ** -8)
    D = rng.lognormal(0, 2.5, (4, G, 128)).astype(np.float32)
    gpu = P.run_gpu(W, D, force_exhaustive=True)
    o = oracle.solve(W, D, threads=P.oracle_threads())
    assert np.array_equal(gpu["scales"], o["best_bits"])
    assert np.array_equal(gpu["obj"], o["best_obj"])
    assert np.all(gpu["flags"] & 0x02)
    assert gpu["counters"]["fallback"] == G


def test_small_finalist_cap_still_exact():
    W, D = synth.make_inputs(1)
    gpu = P.run_gpu(W, D, finalist_cap=1)
    Wg, Dg = P.groups_and_diag(W, D, W.shape[1])
    P.check_against_oracle(Wg, Dg, gpu, where="cap=1")


def test_entry_points_agree_and_empty_input():
    import torch
    from minimax_scale_search_b200 import cq
    W, D = synth.make_inputs(1)
    ex = P.run_gpu(W, D)
    Wt = torch.from_numpy(W.view(np.int16)).cuda()
    Dt = torch.from_numpy(D).cuda()
    s, c = cq.select_scales_plain(Wt, Dt)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint16), ex["scales"])
    assert np.array_equal(c.cpu().numpy().view(np.uint32), ex["codes"])
    hs, hc = cq.select_scales_host(W, D)
    assert np.array_equal(hs, ex["scales"]) and np.array_equal(hc, ex["codes"])
    # per-group layout through the host entry point
    Wg, Dg = P.groups_and_diag(W, D, W.shape[1])
    hs2, hc2 = cq.select_scales_host(Wg, Dg)
    assert np.array_equal(hs2, ex["scales"]) and np.array_equal(hc2, ex["codes"])
    # empty input is a no-op
    e = cq.select_scales(torch.zeros((0, 128), dtype=torch.int16, device="cuda"),
                         torch.ones((4, 0, 128), dtype=torch.float32, device="cuda"))
    assert e.scales.numel() == 0


def test_host_entry_point_chunks_large_input():
    """Many more groups than one host-path chunk (2^16), so the copy/compute
    pipeline runs over 20 chunks and reuses each of its six slots."""
    from minimax_scale_search_b200 import cq
    rows = 10240  # 1.31M groups over 16384-wide rows
    W = synth.make_weights(3, 0, rows)
    D = synth.make_diagonals(3)
    hs, hc = cq.select_scales_host(W, D)
    ex = P.run_gpu(W, D)
    assert np.array_equal(hs, ex["scales"]) and np.array_equal(hc, ex["codes"])


def test_host_entry_point_ragged_chunks():
    """Chunks rounded down to whole rows (3 groups per row: 65,535-group
    chunks) with a ragged last chunk, and the per-group diagonal layout over
    several chunks, against the device entry point."""
    import torch
    from minimax_scale_search_b200 import cq
    rng = np.random.default_rng(77)
    rows, K, E = 50_001, 384, 3
    W = np.clip(rng.normal(0, 0.02, (rows, K)), -1, 1).astype(np.float16).view(np.uint16)
    D = rng.lognormal(0, 1.0, (E, K)).astype(np.float32)
    hs, hc = cq.select_scales_host(W, D)
    ex = P.run_gpu(W, D, K)
    assert np.array_equal(hs, ex["scales"]) and np.array_equal(hc, ex["codes"])
    G = 140_000  # two full 2^16 chunks and a ragged 8,928-group one
    Wg = np.ascontiguousarray(W.reshape(-1, 128)[:G])
    Dg = rng.lognormal(0, 1.0, (E, G, 128)).astype(np.float32)
    hs2, hc2 = cq.select_scales_host(Wg, Dg)
    r = cq.select_scales(torch.from_numpy(Wg.view(np.int16)).cuda(), torch.from_numpy(Dg).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(hs2, r.scales.cpu().numpy().view(np.uint16))
    assert np.array_equal(hc2, r.codes.cpu().numpy().view(np.uint32))


# ---- the pairwise environment-intersection solver (cq_opts.intersections) ----

@pytest.mark.parametrize("idx", [1, 2])
def test_intersection_solver_every_group(idx):
    """Surviving runs searched by the environment-intersection solver: every
    group of the tiny and projection workloads against the oracle."""
    W, D = synth.make_inputs(idx)
    gpu = P.run_gpu(W, D, intersections=True)
    Wg, Dg = P.groups_and_diag(W, D, W.shape[1])
    P.check_against_oracle(Wg, Dg, gpu, where=f"intersections {synth.workload(idx).name}")
    assert np.array_equal(P.recompute_codes(Wg, gpu["scales"]), gpu["codes"])


@pytest.mark.parametrize("E", [1, 2, 3, 4, 5, 6, 7, 8])
def test_intersection_solver_each_environment_count(E):
    rng = np.random.default_rng(140 + E)
    G = 301
    W = f16bits(rng.normal(0, 0.02, (G, 128)) * np.where(rng.random((G, 128)) < 0.02, 9, 1))
    D = rng.lognormal(0, 2.0, (E, G, 128)).astype(np.float32)
    gpu = P.run_gpu(W, D, intersections=True)
    P.check_against_oracle(W, D, gpu, where=f"intersections E={E}")


@pytest.mark.parametrize("idx,rows", [(3, 8192), (4, 8192)])
def test_intersection_solver_same_output_as_default(idx, rows):
    """Both run searches certify the unique grid minimiser of every run, so
    the outputs (scales, codes, objectives, flags) are the same bytes; a
    sample of the groups also meets the oracle."""
    W = synth.make_weights(idx, 0, rows)
    D = synth.make_diagonals(idx)
    a = P.run_gpu(W, D)
    b = P.run_gpu(W, D, intersections=True)
    for k in ("scales", "codes", "obj", "flags"):
        assert np.array_equal(a[k], b[k]), k
    assert a["counters"] == b["counters"]
    Wg = W.reshape(-1, 128)
    sel = synth.sample_groups(idx, 1000, seed=19)
    sel = sel[sel < Wg.shape[0]]
    E = D.shape[0]
    Dsel = np.ascontiguousarray(D.reshape(E, -1, 128)[:, sel % (D.shape[1] // 128), :])
    P.check_against_oracle(Wg[sel], Dsel, {k: v[sel] for k, v in b.items() if k != "counters"},
                           where=f"intersections {synth.workload(idx).name}")
