"""Comparison scale policies and the reconstruction proxy, plain CPU versions
(test infrastructure: only the tests, the smoke check and the benchmark's CPU
leg use this module; it shares no code with the CUDA path).

CliffQuant project page, "Held-out reconstruction proxy" (and the model card's
section of the same name): three scale policies are compared on the
module-macro worst-environment weighted MSE over sampled groups.

* CliffQuant: the exact minimax scale (``oracle.solve``).
* Pooled-WMSE: the environments' diagonals averaged first, then the same exact
  search with that single environment.  Reading: the pooled diagonal is the
  arithmetic mean over environments, accumulated in fp64 in environment order
  and rounded once to fp32 (the diagonals' own precision).
* AbsMax: the matched baseline checkpoint's scale, fp16(max |w| / 7) with the
  division in fp64 and one round-to-nearest-even; raised to the smallest
  positive pattern when that rounds to zero, since a scale must be positive.

The proxy (reading): for module m and environment e, the weighted MSE is the
sum over the module's groups of sum_i d_{e,i} (w_i - s q_i)^2, divided by the
number of weights (128 per group); a module's worst-environment value is the
largest over e; the macro value is the plain mean over modules.
"""
from __future__ import annotations

import math

import numpy as np

from . import absmax_scale, objective, pack_codes, solve

GROUP = 128


def pool_diagonals(D) -> np.ndarray:
    """[E, ...] float32 -> [1, ...] float32: fp64 sum over e = 0..E-1 in that
    order, divided by E, rounded to nearest even fp32."""
    D = np.asarray(D, dtype=np.float32)
    acc = np.zeros(D.shape[1:], dtype=np.float64)
    for e in range(D.shape[0]):
        acc = acc + D[e].astype(np.float64)
    return (acc / float(D.shape[0])).astype(np.float32)[None]


def _is_finite_group(w_bits) -> bool:
    return bool(np.all((np.asarray(w_bits, dtype=np.uint16) & 0x7FFF) < 0x7C00))


def absmax_policy(W):
    """AbsMax scales and packed codes: (uint16 [G], uint32 [G, 16]).  A group
    holding a non-finite weight gets scale 0x0001 and zero codes."""
    W = np.asarray(W, dtype=np.uint16).reshape(-1, GROUP)
    G = W.shape[0]
    scales = np.ones(G, dtype=np.uint16)
    codes = np.zeros((G, GROUP), dtype=np.int8)
    ones = np.ones((1, GROUP), dtype=np.float32)
    for g in range(G):
        if not _is_finite_group(W[g]):
            continue
        s = max(absmax_scale(W[g]), 1)
        scales[g] = s
        codes[g] = objective(W[g], ones, s)[2]
    return scales, pack_codes(codes)


def group_diagonal(D, K: int, g: int, G: int) -> np.ndarray:
    """[E, 128] diagonals of group g: per column (K > 0, D [E, K], groups run
    along each row of K / 128 groups) or per group (K == 0, D [E, G, 128])."""
    if K > 0:
        c = (g % (K // GROUP)) * GROUP
        return D[:, c:c + GROUP]
    return D[:, g, :]


def group_objectives(W, D, K: int, scales) -> np.ndarray:
    """Per-environment objectives [G, E] (float64) of the given scales."""
    W = np.asarray(W, dtype=np.uint16).reshape(-1, GROUP)
    D = np.asarray(D, dtype=np.float32)
    G = W.shape[0]
    out = np.zeros((G, D.shape[0]), dtype=np.float64)
    for g in range(G):
        out[g] = objective(W[g], group_diagonal(D, K, g, G), int(scales[g]))[1]
    return out


def pooled_policy(W, D, K: int = 0, threads: int | None = None) -> np.ndarray:
    """Pooled-WMSE scales: the exact search over the pooled diagonal."""
    W = np.asarray(W, dtype=np.uint16).reshape(-1, GROUP)
    return solve(W, pool_diagonals(D), K, threads=threads)["best_bits"]


def reconstruction_proxy(per_env, offsets, scale: float = 1.0 / GROUP):
    """(module_env [nmod, E], module_worst [nmod], macro) from per-environment
    group objectives and module offsets, with correctly rounded sums
    (math.fsum).  A module without groups gives NaN."""
    per_env = np.asarray(per_env, dtype=np.float64)
    offsets = [int(o) for o in offsets]
    nmod, E = len(offsets) - 1, per_env.shape[1]
    module_env = np.zeros((nmod, E), dtype=np.float64)
    for m in range(nmod):
        a, b = offsets[m], offsets[m + 1]
        for e in range(E):
            module_env[m, e] = (math.fsum(per_env[a:b, e]) / (b - a) * scale) if b > a else math.nan
    module_worst = module_env.max(axis=1) if nmod else np.zeros(0)
    macro = math.fsum(module_worst) / nmod if nmod else math.nan
    return module_env, module_worst, macro
