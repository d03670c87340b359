"""Shared helpers for the GPU parity tests (not a test module)."""
import os

import numpy as np

import oracle

NEAR_TIE = 1e-12

# (workload, counts) of the parity checks run in this session, printed in the
# terminal summary so a run's log shows how many groups met the oracle
REPORT = []


def record(where, **counts):
    REPORT.append((where, counts))


def oracle_threads():
    return max(1, os.cpu_count() or 1)


def run_gpu(W_bits, D, K=None, **kw):
    """Run the CUDA path through the binding; returns host numpy outputs."""
    import torch
    from minimax_scale_search_b200 import cq
    W = torch.from_numpy(np.ascontiguousarray(W_bits).view(np.int16)).cuda()
    Dt = torch.from_numpy(np.ascontiguousarray(D, dtype=np.float32)).cuda()
    res = cq.select_scales(W, Dt, K, want_objective=True, want_flags=True, **kw)
    torch.cuda.synchronize()
    scales, codes = cq.to_numpy_bits(res)
    out = dict(scales=scales, codes=codes, obj=res.objective.cpu().numpy(),
               flags=res.flags.cpu().numpy(), counters=res.counters())
    del W, Dt, res
    return out


def groups_and_diag(W_bits, D, K):
    """Per-group views: W [G,128] and D [E,G,128] (D expanded only when K > 0)."""
    Wg = np.ascontiguousarray(W_bits).reshape(-1, 128)
    if K:
        gpr = K // 128
        E = D.shape[0]
        Dg = D.reshape(E, gpr, 128)[:, np.arange(Wg.shape[0]) % gpr, :]
    else:
        Dg = D
    return Wg, np.ascontiguousarray(Dg, dtype=np.float32)


def check_against_oracle(Wg, Dg, gpu, sel=None, where=""):
    """Parity rule: scale bits and packed codes identical wherever the oracle's
    best and runner-up differ by more than 1e-12 relative (or the best is 0);
    elsewhere the oracle's objective at the GPU scale is within 1e-12 of the
    oracle minimum.  Returns the oracle result."""
    sel = np.arange(Wg.shape[0]) if sel is None else np.asarray(sel)
    o = oracle.solve(Wg, Dg, sel=sel, threads=oracle_threads())
    bad = []
    for k, g in enumerate(sel):
        ob, orun = o["best_obj"][k], o["runner_obj"][k]
        gs = int(gpu["scales"][g])
        strict = ob == 0.0 or oracle.rel_gap(ob, orun) > NEAR_TIE
        if strict:
            if gs != int(o["best_bits"][k]):
                bad.append((int(g), "scale", gs, int(o["best_bits"][k]), ob, orun))
                continue
            words = oracle.pack_codes(o["codes"][k])
            if not np.array_equal(words, gpu["codes"][g]):
                bad.append((int(g), "codes"))
                continue
        else:
            f, _, q = oracle.objective(Wg[g], Dg[:, g, :], gs)
            if not (f <= ob * (1 + NEAR_TIE)):
                bad.append((int(g), "near-tie objective", f, ob))
                continue
            if not np.array_equal(oracle.pack_codes(q), gpu["codes"][g]):
                bad.append((int(g), "near-tie codes"))
                continue
        # the reported objective is the fp64 objective at the chosen scale
        f_at = ob if gs == int(o["best_bits"][k]) else oracle.objective(Wg[g], Dg[:, g, :], gs)[0]
        if oracle.rel_gap(gpu["obj"][g], f_at) > 1e-13:
            bad.append((int(g), "objective", gpu["obj"][g], f_at))
    assert not bad, f"{where}: {len(bad)} mismatches, first: {bad[:5]}"
    return o


def recompute_codes(Wg, scales):
    """clip(round-half-even(w/s), -8, 7) in fp64 (exact decisions), packed."""
    w = Wg.view(np.float16).astype(np.float64)
    s = scales.view(np.float16).astype(np.float64)[:, None]
    q = np.clip(np.rint(w / s), -8, 7).astype(np.int64) + 8
    sh = (4 * np.arange(8, dtype=np.uint64))[None, None, :]
    return (q.reshape(-1, 16, 8).astype(np.uint64) << sh).sum(axis=2).astype(np.uint32)


def objective_np(Wg, Dg, scales):
    """max_e sum_i d (w - s q)^2 in fp64 (vectorised; order differs from the oracle)."""
    w = Wg.view(np.float16).astype(np.float64)
    s = scales.view(np.float16).astype(np.float64)[:, None]
    q = np.clip(np.rint(w / s), -8, 7)
    r2 = (w - s * q) ** 2
    return np.max(np.einsum("egi,gi->eg", Dg.astype(np.float64), r2), axis=0)


def seed_range(var: str, default: int):
    """Seeds of a seeded-case test: range(default), or the range an environment
    variable names as "N" (0..N-1) or "A:B" (A..B-1), so a larger campaign runs
    the same committed cases, e.g. CQ_FUZZ_FAST_SEEDS=100:4500."""
    import os
    v = os.environ.get(var, "").strip()
    if not v:
        return range(default)
    if ":" in v:
        a, b = v.split(":", 1)
        return range(int(a), int(b))
    return range(int(v))
