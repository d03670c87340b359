"""The benchmark's accounting helpers, on hand-computed cases (CPU).

The roofline fraction the benchmark reports rests on these: the counted FLOP
convention (per non-trivial group, (T + 1) runs of FLOP_run(E) fp32 flops with
T = qmax #(w > 0) + |qmin| #(w < 0), plus 2 n E 5 fp64 rescoring flops), the
peaks from unit counts and the clock, and the whole-job rate."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def f16bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def test_flop_run_values():
    # 4E + E + 12 E(E-1)/2 + (E^2 + 4)(5E - 1)
    assert bench.flop_run(1) == 4 + 1 + 0 + 5 * 4
    assert bench.flop_run(4) == 472
    assert bench.flop_run(8) == 3028


def test_counted_flops_hand_example():
    W = np.zeros((3, 128), dtype=np.uint16)
    W[0, 5] = f16bits([0.5])[0]          # one positive weight: T = 7
    W[0, 9] = f16bits([-0.25])[0]        # one negative weight: T += 8
    W[1, :] = f16bits(np.full(128, 0.1))  # 128 positive: T = 896
    W[2, 7] = 0x8000                      # -0 only: a trivial group, not counted
    f32, f64 = bench.counted_flops(W, 4)
    assert f32 == (15 + 1) * 472 + (896 + 1) * 472
    assert f64 == 2 * 2 * 128 * 4 * 5
    # a general spec counts its own transitions and group size
    f32s, f64s = bench.counted_flops(W[:2, :64], 4, qmin=-4, qmax=3)
    assert f32s == (3 + 4 + 1) * 472 + (3 * 64 + 1) * 472
    assert f64s == 2 * 2 * 64 * 4 * 5


def test_peaks_and_job_rate():
    p32, p64, mhz, _ = bench.peaks()
    assert abs(p32 - 148 * 128 * 2 * mhz * 1e6 / 1e12) < 1e-9
    assert abs(p64 - p32 / 2) < 1e-9
    # whole-job rate: all ranks' units over the slowest rank's time
    assert bench.job_rate(8000, 0.5) == 16000.0  # the job's groups over the slowest rank's seconds


def test_objective_roofline_picks_the_binding_bound():
    p32, p64, mhz, _ = bench.peaks()
    ops_peak = 148 * 64 * mhz * 1e6 / 1e12  # fp64 operations per second, T
    G, E = 3_883_008, 4
    # 10 fp64 operations per weight at E = 4, 298 bytes per group
    r = bench.objective_roofline(G, E, 0.774, 6525.0)
    assert r["fp64_ops"] == G * 128 * 10 and r["bytes_per_group"] == 298
    assert r["bound"] == "alu"  # 0.267 ms of fp64 issue against 0.177 ms of HBM
    assert abs(r["peak"] - ops_peak) < 1e-9
    assert abs(r["frac"] - G * 1280 / 0.774e-3 / (ops_peak * 1e12)) < 1e-12
    assert abs(r["hbm_frac"] - G * 298 / 0.774e-3 / 6525e9) < 1e-12
    # with a slow memory the bytes bind instead
    r2 = bench.objective_roofline(G, E, 0.774, 1000.0)
    assert r2["bound"] == "hbm" and abs(r2["frac"] - G * 298 / 0.774e-3 / 1000e9) < 1e-12


def test_traffic_records_parse_and_match_their_summaries():
    """The committed ncu records the benchmark reads: well formed, positive,
    and the main kernel's hash is the one its profile summary cites."""
    prof = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles")
    kv = dict(t.split("=", 1) for t in open(os.path.join(prof, "select_kernel_traffic.txt")).read().split())
    assert int(kv["groups"]) > 0 and int(kv["dram_bytes"]) > 0
    assert len(kv["kernel_sha"]) == 16
    assert kv["kernel_sha"] in open(os.path.join(prof, kv["capture"])).read()
    # bytes per group near the algorithmic 322 (some output still in L2): a sanity range
    assert 250 <= int(kv["dram_bytes"]) / int(kv["groups"]) <= 340
    names = set()
    for ln in open(os.path.join(prof, "secondary_kernels_traffic.txt")).read().splitlines():
        rec = dict(t.split("=", 1) for t in ln.split() if "=" in t)
        assert {"kernel", "src", "sha", "units", "dram_bytes"} <= set(rec), ln
        assert int(rec["units"]) > 0 and int(rec["dram_bytes"]) > 0
        assert os.path.exists(os.path.join(os.path.dirname(prof), "minimax_scale_search_b200", "csrc", rec["src"]))
        names.add(rec["kernel"])
    assert {"absmax_kernel", "objective_kernel<4,", "spec_kernel<4>"} <= names


def test_spec_routing_matches_the_header():
    """bench.py labels a spec line with the kernel cq_select_scales_spec picks:
    the W4 search for qmin = -qmax or -qmax - 1, up to 16 layers at group size
    128 and 8 at 64, else the general kernel."""
    w4 = [(-8, 7, 128), (-4, 3, 128), (-1, 1, 128), (-16, 15, 128), (-16, 16, 128), (-8, 7, 64), (-8, 8, 64)]
    general = [(-17, 16, 128), (-16, 15, 64), (-3, 5, 128), (-8, 6, 128), (-8, 7, 256), (-8, 7, 100), (-1, 0, 128)]
    assert all(bench.spec_uses_w4_search(*c) for c in w4)
    assert not any(bench.spec_uses_w4_search(*c) for c in general)
