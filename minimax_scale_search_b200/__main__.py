"""Command-line runner: select scales for one synthetic workload on the GPU.

    python -m minimax_scale_search_b200 --workload 2 [--rows R] [--repeat N]
        [--matrix M] [--check N] [--force-exhaustive]

Prints one JSON line with the device time per call (CUDA events), groups/s and
the kernel counters.  --check N compares N sampled groups with the exhaustive
CPU oracle (test infrastructure; needs the oracle's C library).
"""
from __future__ import annotations

import argparse
import json
import time

import numpy as np


def main():
    ap = argparse.ArgumentParser(prog="python -m minimax_scale_search_b200")
    ap.add_argument("--workload", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--rows", type=int, default=0, help="only the first R rows of the matrix")
    ap.add_argument("--matrix", type=int, default=0)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--check", type=int, default=0)
    ap.add_argument("--force-exhaustive", action="store_true")
    a = ap.parse_args()

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
    G = W.size // 128
    ws = torch.empty(cq.workspace_bytes(G, wl.E), dtype=torch.uint8, device="cuda")
    times = []
    res = None
    for _ in range(a.repeat):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        res = cq.select_scales(Wd, Dd, wl.cols, workspace=ws, force_exhaustive=a.force_exhaustive,
                               want_objective=a.check > 0)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    out = {"workload": wl.name, "rows": rows, "groups": G, "E": wl.E, "gen_s": round(gen_s, 2),
           "ms": [round(t, 3) for t in times], "groups_per_s": G / (min(times) / 1e3),
           "counters": res.counters()}
    if a.check:
        import oracle
        scales, codes = cq.to_numpy_bits(res)
        sel = synth.sample_groups(a.workload, min(a.check, G), seed=3)
        sel = sel[sel < G]
        Wg = W.reshape(-1, 128)
        o = oracle.solve(Wg, D, K=wl.cols, sel=sel)
        strict = (o["best_obj"] == 0) | (np.abs(o["runner_obj"] - o["best_obj"]) >
                                         1e-12 * np.maximum(np.abs(o["best_obj"]), np.abs(o["runner_obj"])))
        same = scales[sel] == o["best_bits"]
        out["check"] = {"groups": int(len(sel)), "strict": int(strict.sum()),
                        "strict_mismatch": int((strict & ~same).sum())}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
