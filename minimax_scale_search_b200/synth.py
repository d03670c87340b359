"""Seeded synthetic inputs for W4/G128 minimax scale selection.

This module only draws inputs: fp16 weight matrices and per-column environment
diagonals with the shapes and value distributions of the five workloads below.
It holds none of the selection method's arithmetic, so both the CUDA path and
the CPU oracle may take their inputs from it.

Recipe (CliffQuant project page, "What CliffQuant changes": weights w_i and
separately normalised environment diagonals d_{e,i}):

* every value is drawn in fp64 with NumPy's PCG64, then cast once (weights to
  binary16 with round-to-nearest-even, diagonals to fp32);
* each diagonal environment is lognormal, divided by its own fp64 mean over
  the K columns ("separately normalized"), then cast to fp32;
* a stream is keyed by ``SeedSequence(seed, spawn_key=(kind, matrix, block))``
  so that any row range regenerates bit-identically however it is chunked;
* groups run along the input dimension: group ``g`` of a row-major ``W[R, K]``
  is row ``g // (K/128)``, columns ``(g % (K/128))*128 .. +127``.

Workloads (sizes follow the 0.8B model card's scale run of 3,883,008 groups):

1. tiny       64 x 512, N(0, 0.02), 1% of entries x10, E=4, lognormal(0, 1)
2. projection 3072 x 1024, N(0, 0.02), 0.5% x8, E=4, lognormal(0, 1.5)
3. sweep      30336 x 16384, 0.02 * Student-t(5), E=4, lognormal(0, 1.5)
4. tie/stress 8192 x 16384, E=8, lognormal(0, 2.5); groups split by a seeded
              permutation: 65% N(0, 0.02); 25% exact multiples m_i * s0 of an
              fp16 step s0 = 2^U{-12..-4} * (1 + j/128) with m_i ~ U{-8..7}
              (first half) or U{-4..3} (second half); 5% all zero; 5% a single
              nonzero N(0, 0.02) weight at a uniform position
5. large      32 matrices of 14336 x 4096, N(0, 0.015), 0.2% x12, E=4,
              lognormal(0, 1.5), one diagonal set per matrix

Proxy inputs (``make_proxy_inputs``; project page, "Held-out reconstruction
proxy": 4,096 groups sampled across 150 target matrices): the groups are split
over the modules as evenly as possible, the first ``groups % modules`` modules
taking one more.  Module m draws N(0, sigma_m) weights, sigma_m = 0.02 *
2^U(-1, 1), with 0.5% of entries x8, and its own E lognormal(0, 1.5)
diagonals over 4096 columns, each environment divided by its fp64 mean; each
of its groups takes a uniformly drawn 128-column block of those diagonals.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

GROUP = 128
ROW_BLOCK = 256

_KIND_DIAG = 0
_KIND_ROWS = 1
_KIND_CLASS = 2
_KIND_PROXY = 3
_KIND_CODES = 4
_KIND_GPTQ = 5
_KIND_ACT = 6


@dataclass(frozen=True)
class Workload:
    idx: int
    name: str
    rows: int
    cols: int
    E: int
    n_matrices: int
    d_sigma: float
    seed: int

    @property
    def groups_per_matrix(self) -> int:
        return self.rows * self.cols // GROUP

    @property
    def groups(self) -> int:
        return self.groups_per_matrix * self.n_matrices

    @property
    def groups_per_row(self) -> int:
        return self.cols // GROUP


WORKLOADS = {
    1: Workload(1, "tiny-64x512-E4", 64, 512, 4, 1, 1.0, 1001),
    2: Workload(2, "projection-3072x1024-E4", 3072, 1024, 4, 1, 1.5, 1002),
    3: Workload(3, "sweep-30336x16384-E4", 30336, 16384, 4, 1, 1.5, 1003),
    4: Workload(4, "tie-stress-8192x16384-E8", 8192, 16384, 8, 1, 2.5, 1004),
    5: Workload(5, "large-32x14336x4096-E4", 14336, 4096, 4, 32, 1.5, 1005),
}


def workload(idx: int) -> Workload:
    return WORKLOADS[idx]


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence(seed, spawn_key=tuple(key)))


def make_diagonals(idx: int, matrix: int = 0) -> np.ndarray:
    """fp32 [E, K] per-column environment diagonals, each env mean 1 in fp64."""
    wl = WORKLOADS[idx]
    rng = _rng(wl.seed, _KIND_DIAG, matrix)
    d = rng.lognormal(0.0, wl.d_sigma, size=(wl.E, wl.cols))
    d = d / d.mean(axis=1, keepdims=True)
    return d.astype(np.float32)


def _outliers(rng, w, frac, factor):
    mask = rng.random(w.shape) < frac
    w[mask] *= factor
    return w


def _stress_classes(wl: Workload) -> np.ndarray:
    """Per-group class for workload 4: 0 gaussian, 1 multiples U{-8..7},
    2 multiples U{-4..3}, 3 all zero, 4 single nonzero."""
    G = wl.groups_per_matrix
    perm = _rng(wl.seed, _KIND_CLASS, 0).permutation(G)
    n_gauss = int(round(0.65 * G))
    n_mult = int(round(0.25 * G))
    n_zero = int(round(0.05 * G))
    cls = np.empty(G, dtype=np.int8)
    c = 0
    for label, count in ((0, n_gauss), (1, n_mult // 2), (2, n_mult - n_mult // 2), (3, n_zero)):
        cls[perm[c:c + count]] = label
        c += count
    cls[perm[c:]] = 4
    return cls


_CLASS_CACHE: dict[int, np.ndarray] = {}


def stress_classes() -> np.ndarray:
    if 4 not in _CLASS_CACHE:
        _CLASS_CACHE[4] = _stress_classes(WORKLOADS[4])
    return _CLASS_CACHE[4]


def _block(wl: Workload, matrix: int, b: int) -> np.ndarray:
    """fp16 bits [rows, K] of row block b (rows b*ROW_BLOCK .. +ROW_BLOCK)."""
    r0 = b * ROW_BLOCK
    nr = min(ROW_BLOCK, wl.rows - r0)
    rng = _rng(wl.seed, _KIND_ROWS, matrix, b)
    shape = (nr, wl.cols)
    if wl.idx == 1:
        w = _outliers(rng, rng.normal(0.0, 0.02, shape), 0.01, 10.0)
    elif wl.idx == 2:
        w = _outliers(rng, rng.normal(0.0, 0.02, shape), 0.005, 8.0)
    elif wl.idx == 3:
        w = 0.02 * rng.standard_t(5, shape)
    elif wl.idx == 5:
        w = _outliers(rng, rng.normal(0.0, 0.015, shape), 0.002, 12.0)
    elif wl.idx == 4:
        w = rng.normal(0.0, 0.02, shape)
        gpr = wl.groups_per_row
        cls = stress_classes()[r0 * gpr:(r0 + nr) * gpr]
        wg = w.reshape(-1, GROUP)
        for gl in np.nonzero(cls)[0]:
            c = cls[gl]
            if c in (1, 2):
                p = rng.integers(-12, -3)
                j = rng.integers(0, 128)
                s0 = np.ldexp(1.0 + j / 128.0, int(p))
                lo, hi = (-8, 8) if c == 1 else (-4, 4)
                wg[gl] = rng.integers(lo, hi, GROUP).astype(np.float64) * s0
            elif c == 3:
                wg[gl] = 0.0
            else:
                wg[gl] = 0.0
                wg[gl, rng.integers(0, GROUP)] = rng.normal(0.0, 0.02)
        w = wg.reshape(shape)
    else:
        raise ValueError(idx)
    return w.astype(np.float16).view(np.uint16)


def make_weights(idx: int, row0: int = 0, row1: int | None = None, matrix: int = 0,
                 threads: int | None = None) -> np.ndarray:
    """fp16 bit patterns (uint16) [row1-row0, K] of one matrix of workload idx."""
    wl = WORKLOADS[idx]
    row1 = wl.rows if row1 is None else row1
    if not (0 <= row0 <= row1 <= wl.rows):
        raise ValueError("row range out of bounds")
    out = np.empty((row1 - row0, wl.cols), dtype=np.uint16)
    if row1 == row0:
        return out
    b0, b1 = row0 // ROW_BLOCK, (row1 - 1) // ROW_BLOCK + 1

    def fill(b):
        blk = _block(wl, matrix, b)
        lo = max(row0, b * ROW_BLOCK)
        hi = min(row1, b * ROW_BLOCK + blk.shape[0])
        out[lo - row0:hi - row0] = blk[lo - b * ROW_BLOCK:hi - b * ROW_BLOCK]

    nthr = threads or min(32, os.cpu_count() or 1)
    if b1 - b0 == 1 or nthr == 1:
        for b in range(b0, b1):
            fill(b)
    else:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(fill, range(b0, b1)))
    return out


def make_inputs(idx: int, matrix: int = 0):
    """(W bits uint16 [R, K], D fp32 [E, K]) for one matrix of workload idx."""
    return make_weights(idx, matrix=matrix), make_diagonals(idx, matrix)


def group_rows(idx: int, groups: np.ndarray, matrix: int = 0):
    """Weights (uint16 [n, 128]) and per-group diagonals (fp32 [E, n, 128]) of
    selected groups of one matrix, regenerating only the row blocks they touch."""
    wl = WORKLOADS[idx]
    groups = np.asarray(groups, dtype=np.int64)
    gpr = wl.groups_per_row
    rows = groups // gpr
    cols = (groups % gpr) * GROUP
    D = make_diagonals(idx, matrix)
    Wg = np.empty((len(groups), GROUP), dtype=np.uint16)
    for b in np.unique(rows // ROW_BLOCK):
        blk = _block(wl, matrix, int(b))
        sel = np.nonzero(rows // ROW_BLOCK == b)[0]
        for k in sel:
            r = rows[k] - b * ROW_BLOCK
            Wg[k] = blk[r, cols[k]:cols[k] + GROUP]
    Dg = np.stack([D[:, c:c + GROUP] for c in cols], axis=1) if len(groups) else \
        np.empty((wl.E, 0, GROUP), dtype=np.float32)
    return Wg, np.ascontiguousarray(Dg)


def sample_groups(idx: int, count: int, seed: int = 7, matrix: int = 0) -> np.ndarray:
    """Sorted, seeded sample of distinct group indices of one matrix."""
    wl = WORKLOADS[idx]
    count = min(count, wl.groups_per_matrix)
    rng = _rng(seed, 9, idx, matrix)
    return np.sort(rng.choice(wl.groups_per_matrix, size=count, replace=False))


PROXY_GROUPS = 4096
PROXY_MODULES = 150
_PROXY_COLS = 4096


def proxy_offsets(groups: int = PROXY_GROUPS, modules: int = PROXY_MODULES) -> np.ndarray:
    """int64 [modules + 1]: module m holds groups offsets[m] .. offsets[m+1]-1."""
    base, extra = divmod(groups, modules)
    sizes = np.full(modules, base, dtype=np.int64)
    sizes[:extra] += 1
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)


def make_proxy_inputs(groups: int = PROXY_GROUPS, modules: int = PROXY_MODULES, E: int = 4,
                      seed: int = 1006):
    """(W uint16 [G, 128], per-group D fp32 [E, G, 128], offsets int64 [modules + 1])."""
    offsets = proxy_offsets(groups, modules)
    W = np.empty((groups, GROUP), dtype=np.uint16)
    D = np.empty((E, groups, GROUP), dtype=np.float32)
    for m in range(modules):
        a, b = int(offsets[m]), int(offsets[m + 1])
        rng = _rng(seed, _KIND_PROXY, m)
        sigma = 0.02 * 2.0 ** rng.uniform(-1.0, 1.0)
        w = _outliers(rng, rng.normal(0.0, sigma, (b - a, GROUP)), 0.005, 8.0)
        W[a:b] = w.astype(np.float16).view(np.uint16)
        d = rng.lognormal(0.0, 1.5, size=(E, _PROXY_COLS))
        d = (d / d.mean(axis=1, keepdims=True)).astype(np.float32)
        blocks = rng.integers(0, _PROXY_COLS // GROUP, b - a)
        for k, c in enumerate(blocks):
            D[:, a + k, :] = d[:, c * GROUP:(c + 1) * GROUP]
    return W, D, offsets


def make_codes(G: int, seed: int = 1007):
    """Random selection outputs for format tests: (positive finite binary16 scale
    bits uint16 [G], code words uint32 [G, 16]); every nibble is a valid code."""
    rng = _rng(seed, _KIND_CODES, 0)
    scales = rng.integers(1, 0x7C00, G, dtype=np.int64).astype(np.uint16)
    codes = rng.integers(0, 1 << 32, (G, 16), dtype=np.uint64).astype(np.uint32)
    return scales, codes


def make_gptq_tensors(R: int, K: int, seed: int = 1008, act_order: bool = False):
    """Random GPTQ v1 tensors of an [R, K] layer (qweight int32 [K/8, R], qzeros
    int32 [K/128, R/8] with arbitrary zero nibbles, scales binary16 bits uint16
    [K/128, R], g_idx int32 [K]: i // 128, or a random permutation of it)."""
    rng = _rng(seed, _KIND_GPTQ, 0)
    qweight = rng.integers(0, 1 << 32, (K // 8, R), dtype=np.uint64).astype(np.uint32).view(np.int32)
    qzeros = rng.integers(0, 1 << 32, (K // GROUP, R // 8), dtype=np.uint64).astype(np.uint32).view(np.int32)
    scales = rng.integers(1, 0x7C00, (K // GROUP, R), dtype=np.int64).astype(np.uint16)
    g_idx = (np.arange(K) // GROUP).astype(np.int32)
    if act_order:
        g_idx = rng.permutation(g_idx).astype(np.int32)
    return qweight, qzeros, scales, g_idx


def to_bf16_bits(x) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even (finite inputs)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def make_activations(tokens, K: int, dtype: int = 0, seed: int = 1009):
    """Calibration inputs for diagonal estimation: (X [sum(tokens), K] as bf16 /
    fp16 bit patterns (uint16, dtype 0 / 1) or float32 (dtype 2), row offsets
    int64 [E + 1]).  Environment e draws N(0, 1) scaled per column by
    lognormal(0, 1) shared across environments times an environment factor
    lognormal(0, 0.5), with 0.5% of columns (outlier channels) x16."""
    tokens = [int(n) for n in np.atleast_1d(tokens)]
    shared = _rng(seed, _KIND_ACT, 0).lognormal(0.0, 1.0, K)
    outl = _rng(seed, _KIND_ACT, 1).random(K) < 0.005
    shared = np.where(outl, shared * 16.0, shared)
    parts = []
    for e, n in enumerate(tokens):
        rng = _rng(seed, _KIND_ACT, 2 + e)
        scale = shared * rng.lognormal(0.0, 0.5, K)
        x = (rng.standard_normal((n, K)) * scale).astype(np.float32)
        if dtype == 0:
            parts.append(to_bf16_bits(x))
        elif dtype == 1:
            parts.append(x.astype(np.float16).view(np.uint16))
        else:
            parts.append(x)
    offsets = np.concatenate([[0], np.cumsum(tokens)]).astype(np.int64)
    empty = np.zeros((0, K), dtype=np.float32 if dtype == 2 else np.uint16)
    return (np.concatenate(parts, axis=0) if parts else empty), offsets
