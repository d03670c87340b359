#!/usr/bin/env python
"""Throughput of exact minimax FP16 group-scale selection (W4, group 128).

One step = one call of the C ABI over the whole 0.8B-scale sweep workload
(30,336 x 16,384 fp16 weights = 3,883,008 groups, E=4 per-column diagonals),
inputs already resident in HBM.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cq|reference]

N > 1 runs under torch.distributed (one process per GPU, NCCL used only for
the barrier and the max-over-ranks time): the sweep's 30,336 rows split into
contiguous blocks of whole rows, one per rank, each rank holding the whole
[4, 16384] diagonal set, so the job is the same 3,883,008 groups at every N
(strong scaling) and no data crosses between ranks.
The reference arm (--impl reference) times the exhaustive CPU oracle on the
host cores over bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "groups/sec (and % of binding roofline) for W4/G128 minimax scale selection"
WORKLOAD = 3
SMS, FP32_LANES, FP64_LANES = 148, 128, 64


def flop_run(E: int) -> int:
    """Counted FP32 flops per constant-code run: transition update 4E, vertices
    E, pairwise roots 12 E(E-1)/2, and a closed-form max over E environments
    (2 FMA + 1 max each) at the two run ends, E vertices, E(E-1) roots and two
    grid neighbours."""
    return 4 * E + E + 12 * E * (E - 1) // 2 + (E * E + 4) * (5 * E - 1)


def counted_flops(Wg: np.ndarray, E: int, qmin: int = -8, qmax: int = 7):
    """(fp32 flops, fp64 flops) of the method's candidate work for these groups:
    per non-trivial group (T_g + 1) runs with T_g = qmax #(w>0) + |qmin| #(w<0)
    code transitions (7 and 8 for W4), plus fp64 rescoring of two finalists
    (2 * n * E * 5)."""
    n = Wg.shape[1]
    nz = (Wg & 0x7FFF) != 0
    neg = nz & ((Wg & 0x8000) != 0)
    pos = nz & ~neg
    T = qmax * pos.sum(axis=1, dtype=np.int64) + (-qmin) * neg.sum(axis=1, dtype=np.int64)
    live = nz.any(axis=1)
    f32 = int(((T + 1) * live).sum()) * flop_run(E)
    f64 = int(live.sum()) * 2 * n * E * 5
    return f32, f64


def peaks():
    """(fp32 TFLOP/s, fp64 TFLOP/s, clock MHz, source) from unit counts and the max SM clock."""
    mhz, src = 1965.0, "recipe clocks.max.sm 1965 MHz"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
        if mp.get("sm_max_mhz"):
            mhz, src = float(mp["sm_max_mhz"]), "MEASURED_PEAKS.json sm_max_mhz"
    except OSError:
        pass
    p32 = SMS * FP32_LANES * 2 * mhz * 1e6 / 1e12
    p64 = SMS * FP64_LANES * 2 * mhz * 1e6 / 1e12
    return p32, p64, mhz, f"148 SMs x {FP32_LANES} FP32 / {FP64_LANES} FP64 lanes x 2 x {mhz:.0f} MHz ({src})"


def objective_roofline(G: int, E: int, ms: float, hbm: float, hsrc: str = "") -> dict:
    """Roofline of the objective of given scales over G groups in `ms`: the
    slower of its bytes (256 + 2 + 8E + 8 per group) at the HBM peak `hbm`
    (GB/s) and its fp64 operations at one per FP64 lane per clock.  The
    definition fixes 2 + 2E of them per weight: r = w - s q, r*r, and d*rr plus
    the running sum for each environment."""
    bpg = 256 + 2 + 8 * E + 8
    byt = G * bpg
    ops = G * 128 * (2 + 2 * E)
    _, _, mhz, csrc = peaks()
    p64ops = SMS * FP64_LANES * mhz * 1e6 / 1e12  # T operations/s
    hbm_gbs = byt / ms / 1e6
    ops_t = ops / ms / 1e9
    if ops / (p64ops * 1e12) >= byt / (hbm * 1e9):  # the fp64 pipe binds
        roof = {"bound": "alu", "achieved": ops_t, "peak": p64ops, "unit": "Top/s (fp64 operations)",
                "frac": ops_t / p64ops, "hbm_achieved_gbs": hbm_gbs, "hbm_frac": hbm_gbs / hbm,
                "peak_note": f"{SMS} SMs x {FP64_LANES} FP64 lanes x {mhz:.0f} MHz ({csrc})"}
    else:
        roof = {"bound": "hbm", "achieved": hbm_gbs, "peak": hbm, "unit": "GB/s", "frac": hbm_gbs / hbm,
                "alu_frac": ops_t / p64ops, "peak_note": hsrc}
    roof.update({"bytes_per_group": bpg, "fp64_ops": ops})
    return roof


def kernel_source_hash() -> str:
    """Hash of the main kernel's sources (its file and the device header it includes)."""
    h = hashlib.sha256()
    for name in ("cq_select.cu", "cq_device.cuh"):
        h.update(open(os.path.join(ROOT, "minimax_scale_search_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def main_kernel_record():
    """The committed ncu record of the main kernel (profiles/select_kernel_traffic.txt)
    as a dict, or None when the kernel's source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "select_kernel_traffic.txt")
    try:
        kv = dict(tok.split("=", 1) for tok in open(path).read().split() if "=" in tok)
    except OSError:
        return None
    if kv.get("kernel_sha") != kernel_source_hash():
        return None
    return kv


def recorded_traffic(groups: int):
    """DRAM bytes per launch of the main kernel from the committed ncu summary,
    scaled to `groups`; None when the kernel changed since the capture."""
    kv = main_kernel_record()
    if kv is None:
        return None
    return float(kv["dram_bytes"]) / float(kv["groups"]) * groups


def recorded_issue():
    """The main kernel's hardware utilisation from the same ncu capture: issue
    slots active, pipe utilisation and warp instructions per group; None when
    the kernel changed since the capture.  The counted-FLOP fraction compares
    the kernel with the pages' candidate method; these say how busy the SMs
    actually are."""
    kv = main_kernel_record()
    if kv is None or "issue_active_pct" not in kv:
        return None
    keys = ("issue_active_pct", "fma_pipe_pct", "fp64_pipe_pct", "alu_pipe_pct", "lsu_pipe_pct",
            "warp_inst_per_group")
    out = {k: float(kv[k]) for k in keys if k in kv}
    out["source"] = "profiles/" + kv.get("capture", "select_kernel_sweep.md")
    return out


def recorded_kernel_traffic(kernel: str, units: int):
    """DRAM bytes of one launch of a secondary kernel over `units` units, from the
    committed ncu record (profiles/secondary_kernels_traffic.txt) scaled by
    units; None when the kernel's source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "secondary_kernels_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    for ln in lines:
        kv = dict(tok.split("=", 1) for tok in ln.split() if "=" in tok)
        if kv.get("kernel") != kernel:
            continue
        src = os.path.join(ROOT, "minimax_scale_search_b200", "csrc", kv["src"])
        if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != kv.get("sha"):
            return None
        return float(kv["dram_bytes"]) / float(kv["units"]) * units
    return None


class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-i", gpu_index, "-lms", "200"], stdout=self.tmp,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        for ln in open(self.tmp.name).read().splitlines():
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append((ts, float(parts[1].split()[0]), float(parts[2].split()[0]), parts[4:]))
            except (ValueError, IndexError):
                continue
        os.unlink(self.tmp.name)
        inside = [r for r in rows if t0 - 0.25 <= r[0] <= t1 + 0.25] or rows
        if not inside:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in inside for n, v in zip(names, r[3][1:]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


def max_over_ranks(values, dist=None, device=None):
    """Elementwise max of per-rank timings (the job's time is its slowest rank)."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def sum_over_ranks(counts: dict, dist=None, device=None) -> dict:
    """Per-key sum of integer counters over ranks (every rank solves its own
    matrix, so the job's counts are the sums)."""
    if dist is None:
        return {k: int(v) for k, v in counts.items()}
    import torch
    keys = sorted(counts)
    t = torch.tensor([int(counts[k]) for k in keys], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return {k: int(v) for k, v in zip(keys, t.cpu())}


def job_rate(groups_total: int, seconds: float) -> float:
    """Whole-job groups per second: every rank's groups over the slowest rank's time."""
    return groups_total / seconds


def gpu_index_for(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


def oracle_rate(Wg, D, K, groups_target_s: float, seed: int = 5):
    """Time the oracle, as it stands, on a bounded sample; returns (groups/s, n, seconds, threads)."""
    import oracle
    threads = os.cpu_count() or 1
    rng = np.random.default_rng(seed)
    probe = rng.choice(Wg.shape[0], size=min(Wg.shape[0], 2 * threads), replace=False)
    t0 = time.perf_counter()
    oracle.solve(Wg, D, K=K, sel=np.sort(probe), threads=threads)
    per = (time.perf_counter() - t0) / len(probe)
    n = int(max(len(probe), min(Wg.shape[0], groups_target_s / max(per, 1e-6))))
    sel = np.sort(rng.choice(Wg.shape[0], size=n, replace=False))
    t0 = time.perf_counter()
    oracle.solve(Wg, D, K=K, sel=sel, threads=threads)
    dt = time.perf_counter() - t0
    return n / dt, n, dt, threads


def oracle_rate_one_thread(Wg, D, K, seconds: float = 3.0, seed: int = 6):
    """The oracle on one host thread, on a sample of about `seconds` of work;
    returns groups/s."""
    import oracle
    rng = np.random.default_rng(seed)
    probe = np.sort(rng.choice(Wg.shape[0], size=min(Wg.shape[0], 4), replace=False))
    t0 = time.perf_counter()
    oracle.solve(Wg, D, K=K, sel=probe, threads=1)
    per = (time.perf_counter() - t0) / len(probe)
    n = int(max(len(probe), min(Wg.shape[0], seconds / max(per, 1e-6))))
    sel = np.sort(rng.choice(Wg.shape[0], size=n, replace=False))
    t0 = time.perf_counter()
    oracle.solve(Wg, D, K=K, sel=sel, threads=1)
    return n / (time.perf_counter() - t0)


def run_reference(args, wl):
    """The oracle arm: each step solves a bounded sample on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from minimax_scale_search_b200 import synth
    import oracle
    W = synth.make_weights(WORKLOAD, 0, 512)  # 65,536 groups drawn like the full workload
    D = synth.make_diagonals(WORKLOAD)
    Wg = W.reshape(-1, 128)
    threads = os.cpu_count() or 1
    per_step_s = max(1.0, 150.0 / (args.steps + args.warmup))
    _, n_probe, dt_probe, _ = oracle_rate(Wg, D, wl.cols, 2.0)
    n = max(threads, int(n_probe / dt_probe * per_step_s))
    n = min(n, Wg.shape[0])
    rng = np.random.default_rng(17)
    times = []
    for s in range(args.warmup + args.steps):
        sel = np.sort(rng.choice(Wg.shape[0], size=n, replace=False))
        t0 = time.perf_counter()
        oracle.solve(Wg, D, K=wl.cols, sel=sel, threads=threads)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
    tot = sum(times)
    value = n * len(times) / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "groups/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "groups_per_step": n, "E": wl.E, "K": wl.cols},
            "cpu_baseline": {"value": value, "unit": "groups/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} groups per step drawn from rows 0-511 (65,536 groups) of the "
                                       f"{wl.name} workload, exhaustive fp64 over 31,743 scales"},
            "e2e": {"value": value, "unit": "groups/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def hbm_peak():
    """(GB/s, source): the measured copy bandwidth, else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "of measured (MEASURED_PEAKS.json hbm_gbs)"
    except (OSError, KeyError, ValueError):
        return 6650.0, "of fallback (6.65 TB/s)"


def time_calls(fn, steps: int, warmup: int, stream):
    """Mean device ms per call of fn() (CUDA events on the launching stream)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def bench_policies(args, wl, W, D, Wd, Dd, dev):
    """One JSON line per comparison-policy kernel on the same workload: AbsMax
    (HBM-bound), Pooled-WMSE (pooling + the search at E = 1), the objective of
    given scales (HBM-bound) and the three-policy reconstruction proxy on its
    own 4,096-group input."""
    import torch
    from minimax_scale_search_b200 import cq, synth
    stream = torch.cuda.current_stream()
    G = W.size // 128
    hbm, hsrc = hbm_peak()
    p32, p64, _, psrc = peaks()
    base = {"n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "data": "synthetic",
            "config": {"workload": wl.name, "groups": G, "E": wl.E, "K": wl.cols,
                       "l2": "inputs (994 MB of W) larger than the 126 MB L2; no flush"}}
    lines = []
    s_abs = torch.empty(G, dtype=torch.int16, device=dev)
    c_abs = torch.empty((G, 16), dtype=torch.int32, device=dev)
    ms = time_calls(lambda: cq.absmax_scales(Wd, out_scales=s_abs, out_codes=c_abs), args.steps, args.warmup,
                    stream)
    byt = G * (256 + 2 + 64)
    lines.append(dict(base, metric="AbsMax policy groups/sec", op="absmax", value=G / ms * 1e3, unit="groups/s",
                      ms_per_step=ms, higher_is_better=True, dtype="f64", gpu_launches=args.steps,
                      roofline={"bound": "hbm", "achieved": byt / ms / 1e6, "peak": hbm, "unit": "GB/s",
                                "frac": byt / ms / 1e6 / hbm, "traffic": recorded_kernel_traffic("absmax_kernel", G),
                                "kernel": "absmax_kernel",
                                "bytes_per_group": 322, "peak_note": hsrc}))

    s_pool = torch.empty(G, dtype=torch.int16, device=dev)
    c_pool = torch.empty((G, 16), dtype=torch.int32, device=dev)
    ws = torch.empty(cq.workspace_bytes(G, 1), dtype=torch.uint8, device=dev)
    kev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    kms = []

    def pooled():
        cq.select_scales_pooled(Wd, Dd, wl.cols, out_scales=s_pool, out_codes=c_pool, workspace=ws,
                                main_events=kev)
    for _ in range(args.warmup):
        pooled()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        pooled()
        kev[1].synchronize()
        kms.append(kev[0].elapsed_time(kev[1]))
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    f32, f64 = counted_flops(W.reshape(-1, 128), 1)
    kernel_ms = statistics.mean(kms)
    ach = (f32 + f64 * p32 / p64) / (kernel_ms / 1e3) / 1e12
    lines.append(dict(base, metric="Pooled-WMSE policy groups/sec", op="pooled_wmse", value=G / ms * 1e3,
                      unit="groups/s", ms_per_step=ms, higher_is_better=True, dtype="f64",
                      gpu_launches=3 * args.steps,
                      note="per-step host sync to read the main kernel's events; value from the outer events",
                      roofline={"bound": "alu", "achieved": ach, "peak": p32, "unit": "TFLOP/s", "frac": ach / p32,
                                "traffic": None, "kernel": "select_kernel<1>", "kernel_ms": kernel_ms,
                                "fp32_flops": f32, "fp64_flops": f64, "peak_note": psrc}))

    scales = cq.select_scales(Wd, Dd, wl.cols).scales
    per_env = torch.empty((G, wl.E), dtype=torch.float64, device=dev)
    obj = torch.empty(G, dtype=torch.float64, device=dev)
    ms = time_calls(lambda: cq.group_objective(Wd, Dd, scales, wl.cols, per_env=per_env, out=obj), args.steps,
                    args.warmup, stream)
    roof = objective_roofline(G, wl.E, ms, hbm, hsrc)
    roof.update({"traffic": recorded_kernel_traffic("objective_kernel<4,", G),
                 "kernel": "objective_kernel<4, per-column>"})
    lines.append(dict(base, metric="objective of given scales groups/sec", op="objective", value=G / ms * 1e3,
                      unit="groups/s", ms_per_step=ms, higher_is_better=True, dtype="f64",
                      gpu_launches=2 * args.steps, roofline=roof))

    Wp, Dp, offsets = synth.make_proxy_inputs()
    Wpd = torch.from_numpy(Wp.view(np.int16)).to(dev)
    Dpd = torch.from_numpy(Dp).to(dev)
    t = []
    for k in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        res = cq.evaluate_policies(Wpd, Dpd, offsets)
        if k >= args.warmup:
            t.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(t)
    lines.append(dict(base, metric="reconstruction proxy, three policies, ms per evaluation", op="proxy",
                      value=ms, unit="ms", ms_per_step=ms, higher_is_better=False, dtype="f64",
                      gpu_launches=18 * args.steps,
                      config={"workload": "proxy-4096-groups-150-modules-E4", "groups": int(Wp.shape[0]),
                              "modules": len(offsets) - 1, "E": 4, "diagonals": "per-group [4, 4096, 128] fp32"},
                      timing="host wall clock per call, including three device-to-host reads",
                      proxy={p: v[0] for p, v in res.items()}))
    for ln in lines:
        print(json.dumps(ln), flush=True)


def bench_gptq(args, wl, dev):
    """One JSON line each for the GPTQ v1 export and dequantisation of the
    sweep's layer shape (random codes and scales: the format steps do not
    depend on their values)."""
    import torch
    from minimax_scale_search_b200 import cq, synth
    stream = torch.cuda.current_stream()
    R, K = wl.rows, wl.cols
    G = R * K // 128
    hbm, hsrc = hbm_peak()
    scales, codes = synth.make_codes(G)
    S = torch.from_numpy(scales.view(np.int16)).to(dev)
    C = torch.from_numpy(codes.view(np.int32)).to(dev)
    t = cq.gptq_export(S, C, R, K)
    base = {"n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "data": "synthetic", "unit": "groups/s",
            "higher_is_better": True, "dtype": "u32",
            "config": {"workload": f"gptq-v1-{R}x{K}", "groups": G, "R": R, "K": K,
                       "l2": "tensors (>= 248 MB each) larger than the 126 MB L2; no flush"}}
    lines = []
    ms = time_calls(lambda: cq.gptq_export(S, C, R, K), args.steps, args.warmup, stream)
    bpg = 64 + 2 + 64 + 2 + 0.5  # codes and scales in, qweight, scales and qzeros out
    lines.append(dict(base, metric="GPTQ v1 export groups/sec", op="gptq_export", value=G / ms * 1e3,
                      ms_per_step=ms, gpu_launches=args.steps,
                      roofline={"bound": "hbm", "achieved": G * bpg / ms / 1e6, "peak": hbm, "unit": "GB/s",
                                "frac": G * bpg / ms / 1e6 / hbm,
                                "traffic": recorded_kernel_traffic("export_kernel", G),
                                "kernel": "export_kernel (word and scale transposes, fills)",
                                "bytes_per_group": bpg, "peak_note": hsrc}))
    for half in (True, False):
        out = torch.empty((R, K), dtype=torch.float16 if half else torch.float32, device=dev)
        fn = lambda: cq.lib.cq_gptq_dequantize(  # noqa: E731
            cq._ptr(t.qweight), cq._ptr(t.qzeros), cq._ptr(t.scales), cq._ptr(t.g_idx), R, K, int(half),
            cq._ptr(out), cq._stream_handle(stream))
        ms = time_calls(fn, args.steps, args.warmup, stream)
        bpg = 64 + 2 + 0.5 + 128 * (2 if half else 4)
        lines.append(dict(base, metric=f"GPTQ v1 dequantisation to {'fp16' if half else 'fp32'} groups/sec",
                          op="gptq_dequant_fp16" if half else "gptq_dequant_fp32", value=G / ms * 1e3,
                          ms_per_step=ms, gpu_launches=args.steps, dtype="f16" if half else "f32",
                          roofline={"bound": "hbm", "achieved": G * bpg / ms / 1e6, "peak": hbm, "unit": "GB/s",
                                    "frac": G * bpg / ms / 1e6 / hbm,
                                    "traffic": recorded_kernel_traffic(
                                        f"dequant_kernel<{'fp16' if half else 'fp32'}>", G),
                                    "kernel": f"dequant_kernel<{'true' if half else 'false'}>",
                                    "bytes_per_group": bpg, "peak_note": hsrc}))
        del out
    for ln in lines:
        print(json.dumps(ln), flush=True)


DIAG_ENVS, DIAG_TOKENS = 4, 16384


def bench_diag(args, wl, dev):
    """Diagonal estimation from bf16 calibration inputs: 4 environments of
    16,384 tokens over the sweep's 16,384 input columns (2.1 GB, drawn on the
    device from a seeded generator)."""
    import torch
    from minimax_scale_search_b200 import cq
    stream = torch.cuda.current_stream()
    K, E, N = wl.cols, DIAG_ENVS, DIAG_TOKENS
    g = torch.Generator(device=dev)
    g.manual_seed(1010)
    col = torch.exp(torch.randn(K, generator=g, device=dev))
    X = (torch.randn((E * N, K), generator=g, device=dev) * col).to(torch.bfloat16)
    off = np.arange(E + 1, dtype=np.int64) * N
    means = torch.empty((E, K), dtype=torch.float64, device=dev)
    D = torch.empty((E, K), dtype=torch.float32, device=dev)
    hbm, hsrc = hbm_peak()
    ms = time_calls(lambda: cq.estimate_diagonals(X, off, means=means, out=D), args.steps, args.warmup, stream)
    byt = E * N * K * 2 + E * K * (8 + 8 + 4)
    line = {"metric": "diagonal estimation tokens/sec", "op": "diag", "value": E * N / ms * 1e3, "unit": "tokens/s",
            "ms_per_step": ms, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": "f64", "data": "synthetic", "gpu_launches": 2 * args.steps,
            "config": {"workload": f"diag-{E}x{N}x{K}-bf16", "environments": E, "tokens_per_env": N, "K": K,
                       "l2": "inputs (2.1 GB) larger than the 126 MB L2; no flush"},
            "roofline": {"bound": "hbm", "achieved": byt / ms / 1e6, "peak": hbm, "unit": "GB/s",
                         "frac": byt / ms / 1e6 / hbm,
                         "traffic": recorded_kernel_traffic("column_squares_kernel<bf16>", E * N),
                         "kernel": "column_squares_kernel<bf16> + normalise_kernel",
                         "bytes_per_token": K * 2, "peak_note": hsrc}}
    print(json.dumps(line), flush=True)


SPEC_ROWS = 4096
SPEC_CASES = ((-8, 7, 128), (-4, 3, 128), (-2, 1, 128), (-8, 7, 64), (-16, 15, 128))


def spec_uses_w4_search(qmin: int, qmax: int, n: int) -> bool:
    """Whether cq_select_scales_spec runs the W4 kernel's search for this spec
    (|qmin| = qmax or qmax + 1; at most 16 at group size 128, 8 at 64)."""
    return (n == 128 and -qmin <= 16 or n == 64 and -qmin <= 8) and qmax >= 1 and -qmin in (qmax, qmax + 1)


def bench_spec(args, wl, dev):
    """The general-spec path on the first 4,096 rows of the sweep (524,288
    groups of 128; 1,048,576 of 64), one JSON line per spec and kernel: specs
    the W4 kernel's search serves get a second line forced onto the general
    kernel, for comparison."""
    import torch
    from minimax_scale_search_b200 import cq, synth
    stream = torch.cuda.current_stream()
    W = synth.make_weights(WORKLOAD, 0, SPEC_ROWS)
    D = synth.make_diagonals(WORKLOAD)
    Wd = torch.from_numpy(W.view(np.int16)).to(dev)
    Dd = torch.from_numpy(D).to(dev)
    p32, p64, _, psrc = peaks()
    for qmin, qmax, n in SPEC_CASES:
        G = W.size // n
        f32, f64 = counted_flops(W.reshape(-1, n), wl.E, qmin, qmax)
        kernels = (False, True) if spec_uses_w4_search(qmin, qmax, n) else (True,)
        for general in kernels:
            ms = time_calls(lambda: cq.select_scales_spec(Wd, Dd, wl.cols, qmin=qmin, qmax=qmax, group_size=n,
                                                          general_kernel=general),
                            args.steps, args.warmup, stream)
            ach = (f32 + f64 * p32 / p64) / (ms / 1e3) / 1e12
            layers = 16 if -qmin > 8 else 8
            kname = "spec_kernel" if general else f"select_kernel<{wl.E}, false, true, {n}, {layers}> (W4 search)"
            if general:
                traffic = recorded_kernel_traffic("spec_kernel<4>", W.size)
            elif n == 128:  # recorded at (-4, 3) on the 8-layer kernel, (-16, 15) on the 16-layer one
                traffic = recorded_kernel_traffic(
                    "select_kernel<4,false,true>" if layers == 8 else "select_kernel<4,false,true,128,16>", W.size)
            else:
                traffic = None
            line = {"metric": "general-spec minimax scale selection groups/sec", "op": "spec",
                    "value": G / ms * 1e3, "unit": "groups/s", "ms_per_step": ms, "n_gpus": 1,
                    "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "dtype": "f64",
                    "data": "synthetic", "gpu_launches": args.steps * (1 if general else 2),
                    "config": {"workload": f"sweep-rows0-{SPEC_ROWS}-q[{qmin},{qmax}]-n{n}", "groups": G,
                               "E": wl.E, "K": wl.cols, "qmin": qmin, "qmax": qmax, "group_size": n,
                               "kernel": "general" if general else "w4-search"},
                    "roofline": {"bound": "alu", "achieved": ach, "peak": p32, "unit": "TFLOP/s",
                                 "frac": ach / p32, "traffic": traffic, "kernel": kname,
                                 "fp32_flops": f32, "fp64_flops": f64, "peak_note": psrc}}
            print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cq", choices=["cq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--op", default="select", choices=["select", "policies", "gptq", "diag", "spec"],
                    help="select: the headline line; policies / gptq: one line per kernel of those rows")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    from minimax_scale_search_b200 import synth
    wl = synth.workload(WORKLOAD)
    if args.impl == "reference":
        run_reference(args, wl)
        return

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from minimax_scale_search_b200 import cq, shard
    if args.op in ("gptq", "diag", "spec"):
        if world > 1:
            ap.error(f"--op {args.op} runs on one GPU")
        {"gptq": bench_gptq, "diag": bench_diag, "spec": bench_spec}[args.op](args, wl, dev)
        return
    r0, r1 = shard.row_block(rank, world, wl.rows)
    W = synth.make_weights(WORKLOAD, r0, r1)
    D = synth.make_diagonals(WORKLOAD)
    Wg = W.reshape(-1, 128)
    G = Wg.shape[0]
    G_job = wl.groups_per_matrix
    f32, f64 = counted_flops(Wg, wl.E)
    Wd = torch.from_numpy(W.view(np.int16)).to(dev)
    Dd = torch.from_numpy(D).to(dev)
    out_s = torch.empty(G, dtype=torch.int16, device=dev)
    out_c = torch.empty((G, 16), dtype=torch.int32, device=dev)
    ws = torch.empty(cq.workspace_bytes(G, wl.E), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    if args.op == "policies":
        if world > 1:
            ap.error("--op policies runs on one GPU")
        bench_policies(args, wl, W, D, Wd, Dd, dev)
        return

    def step(evs=None):
        return cq.select_scales(Wd, Dd, wl.cols, out_scales=out_s, out_codes=out_c, workspace=ws,
                                main_events=evs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    counters = sum_over_ranks(cq.read_counters(ws), dist, dev)  # one call per rank, summed over the job

    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_index_for(local))
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    t_start.record(stream)
    for k in range(args.steps):
        step(kev[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    if dist:
        dist.barrier()
    clocks = sampler.stop(w0, w1)
    ms_total = t_start.elapsed_time(t_end)
    kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)  # this rank's own launches
    ms_total = max_over_ranks([ms_total], dist, dev)[0]
    ms_step = ms_total / args.steps
    value = job_rate(G_job, ms_step / 1e3)

    # ---- end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        Wp = torch.from_numpy(W.view(np.int16)).pin_memory()
        Dp = torch.from_numpy(D).pin_memory()
        sp = torch.empty(G, dtype=torch.int16).pin_memory()
        cp = torch.empty((G, 16), dtype=torch.int32).pin_memory()
        Wn, Dn, sn, cn = Wp.numpy(), Dp.numpy(), sp.numpy().view(np.uint16), cp.numpy().view(np.uint32)
        for _ in range(2):
            cq.select_scales_host(Wn, Dn, out_scales=sn, out_codes=cn)
        n_e2e = max(3, min(args.steps, 10))
        if dist:
            dist.barrier()
        t0 = time.perf_counter()
        for _ in range(n_e2e):
            cq.select_scales_host(Wn, Dn, out_scales=sn, out_codes=cn)
        e2e_s = max_over_ranks([(time.perf_counter() - t0) / n_e2e], dist, dev)[0]
        dev_s = out_s.cpu().numpy().view(np.uint16)
        assert np.array_equal(dev_s, sn), "host entry point disagrees with the device entry point"
        io = sum_over_ranks({"h2d": W.nbytes + D.nbytes, "d2h": sn.nbytes + cn.nbytes}, dist, dev)
        e2e = {"value": job_rate(G_job, e2e_s), "unit": "groups/s", "h2d_bytes_per_step": io["h2d"],
               "d2h_bytes_per_step": io["d2h"], "ms_per_step": 1e3 * e2e_s, "steps": n_e2e}

    p32, p64, mhz, psrc = peaks()
    t_roof = f32 / (p32 * 1e12) + f64 / (p64 * 1e12)
    achieved = (f32 + f64 * p32 / p64) / (kernel_ms / 1e3) / 1e12
    traffic = recorded_traffic(G)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, dt, threads = oracle_rate(Wg, D, wl.cols, 12.0)
        cpu = {"value": rate, "unit": "groups/s", "cores": threads, "kind": "oracle",
               "value_one_thread": oracle_rate_one_thread(Wg, D, wl.cols),
               "sample": f"{n} groups sampled from the {wl.name} workload (rank 0's matrix), exhaustive "
                         f"fp64 over 31,743 scales, {dt:.1f} s"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "groups/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": wl.name, "groups": G_job, "weights": G_job * 128, "E": wl.E,
                           "K": wl.cols, "diagonals": "per-column [4, 16384] fp32, replicated on every rank",
                           "parallelism": f"row blocks x{world}" if world > 1 else "one GPU",
                           "rows_rank0": [r0, r1], "groups_rank0": G,
                           "l2": f"inputs ({W.nbytes / 1e6:.0f} MB of W per GPU) larger than the 126 MB L2; "
                                 "no flush"},
                "weights_per_s": value * 128,
                "roofline": {"bound": "alu", "achieved": achieved, "peak": p32, "unit": "TFLOP/s",
                             "frac": achieved / p32, "traffic": traffic,
                             "kernel": f"select_kernel<{wl.E}>", "kernel_ms": kernel_ms,
                             "roofline_ms": 1e3 * t_roof, "fp32_flops": f32, "fp64_flops": f64,
                             "peak_note": f"fp32-equivalent (fp64 flops weighted x{p32 / p64:.0f}); {psrc}",
                             "count_basis": "the pages' candidate method on every constant-code run of every "
                                            "group (vertices, pairwise environment intersections, closed-form "
                                            "max), not the kernel's own instructions: the kernel skips most runs "
                                            "by a certified window and screen, so frac compares it with that "
                                            "method; 'issue' gives the hardware utilisation",
                             "issue": recorded_issue()},
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps,
                "clocks": clocks, "counters": counters}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
