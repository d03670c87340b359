"""Command-line runner for synthetic workloads on the GPU.

    python -m minimax_scale_search_b200 --workload 2 [--rows R] [--repeat N]
        [--matrix M] [--force-exhaustive] [--intersections]
    python -m minimax_scale_search_b200 --workload 3 --rows 1024 --qmin -4 --qmax 3 [--group-size 128]
    python -m minimax_scale_search_b200 --ops

The first form selects scales for one synthetic workload and prints one JSON
line with the device time per call (CUDA events), groups/s and the kernel
counters; with --qmin/--qmax/--group-size it runs the general-spec path
instead.  --ops runs each of the other kernels once (AbsMax, objective of
given scales, GPTQ export and dequantisation, diagonal estimation, the
three-policy reconstruction proxy) on inputs larger than L2 and prints their
device times.
"""
from __future__ import annotations

import argparse
import json
import time

import numpy as np


def timed(fn):
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    out = fn()
    e1.record()
    torch.cuda.synchronize()
    return out, round(e0.elapsed_time(e1), 3)


def run_ops():
    """Each secondary kernel once: the first 4,096 sweep rows (524,288 groups,
    134 MB of W), 4 x 8,192 bf16 activation rows of 16,384 columns (1.07 GB),
    and the 4,096-group proxy input."""
    import torch

    from minimax_scale_search_b200 import cq, synth
    W = synth.make_weights(3, 0, 4096)
    D = synth.make_diagonals(3)
    Wd = torch.from_numpy(W.view(np.int16)).cuda()
    Dd = torch.from_numpy(D).cuda()
    ms = {}
    (s_abs, c_abs), ms["absmax"] = timed(lambda: cq.absmax_scales(Wd))
    _, ms["objective"] = timed(lambda: cq.group_objective(Wd, Dd, s_abs, 16384))
    t, ms["gptq_export"] = timed(lambda: cq.gptq_export(s_abs, c_abs, 4096, 16384))
    _, ms["gptq_dequant_fp16"] = timed(lambda: cq.gptq_dequantize(t, half=True))
    _, ms["gptq_dequant_fp32"] = timed(lambda: cq.gptq_dequantize(t))
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    X = torch.randn((4 * 8192, 16384), generator=g, device="cuda").to(torch.bfloat16)
    _, ms["diagonals"] = timed(lambda: cq.estimate_diagonals(X, np.arange(5, dtype=np.int64) * 8192))
    Wp, Dp, off = synth.make_proxy_inputs()
    res, ms["proxy_three_policies"] = timed(lambda: cq.evaluate_policies(
        torch.from_numpy(Wp.view(np.int16)).cuda(), torch.from_numpy(Dp).cuda(), off))
    print(json.dumps({"groups": int(W.size // 128), "ms": ms, "proxy": {k: v[0] for k, v in res.items()}}),
          flush=True)


def main():
    ap = argparse.ArgumentParser(prog="python -m minimax_scale_search_b200")
    ap.add_argument("--workload", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--rows", type=int, default=0, help="only the first R rows of the matrix")
    ap.add_argument("--matrix", type=int, default=0)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--force-exhaustive", action="store_true")
    ap.add_argument("--intersections", action="store_true",
                    help="search surviving runs with the pairwise environment-intersection solver")
    ap.add_argument("--ops", action="store_true", help="run each of the other kernels once")
    ap.add_argument("--qmin", type=int, default=None, help="general spec: smallest code")
    ap.add_argument("--qmax", type=int, default=None, help="general spec: largest code")
    ap.add_argument("--group-size", type=int, default=128, help="general spec: weights per group")
    a = ap.parse_args()
    if a.ops:
        run_ops()
        return

    import torch

    from minimax_scale_search_b200 import cq, synth

    wl = synth.workload(a.workload)
    rows = a.rows or wl.rows
    t0 = time.perf_counter()
    W = synth.make_weights(a.workload, 0, rows, matrix=a.matrix)
    D = synth.make_diagonals(a.workload, a.matrix)
    gen_s = time.perf_counter() - t0
    Wd = torch.from_numpy(W.view(np.int16)).cuda()
    Dd = torch.from_numpy(D).cuda()
    if a.qmin is not None or a.qmax is not None:
        qmin = -8 if a.qmin is None else a.qmin
        qmax = 7 if a.qmax is None else a.qmax
        n = a.group_size
        times = []
        for _ in range(a.repeat):
            _, t = timed(lambda: cq.select_scales_spec(Wd, Dd, wl.cols, qmin=qmin, qmax=qmax, group_size=n))
            times.append(t)
        G = W.size // n
        print(json.dumps({"workload": wl.name, "rows": rows, "groups": G, "E": wl.E, "qmin": qmin, "qmax": qmax,
                          "group_size": n, "ms": times, "groups_per_s": G / (min(times) / 1e3)}), flush=True)
        return
    G = W.size // 128
    ws = torch.empty(cq.workspace_bytes(G, wl.E), dtype=torch.uint8, device="cuda")
    times = []
    res = None
    for _ in range(a.repeat):
        res, t = timed(lambda: cq.select_scales(Wd, Dd, wl.cols, workspace=ws, force_exhaustive=a.force_exhaustive,
                                                intersections=a.intersections))
        times.append(t)
    out = {"workload": wl.name, "rows": rows, "groups": G, "E": wl.E, "gen_s": round(gen_s, 2),
           "ms": times, "groups_per_s": G / (min(times) / 1e3), "counters": res.counters()}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
