"""Per-environment sensitivity diagonals from calibration activations, plain
CPU version (test infrastructure: only the tests, the smoke check and the
benchmark's CPU leg use this module; it shares no code with the CUDA path).

CliffQuant project page, "What CliffQuant changes" and "The negative result
that changed the method": the solver takes "separately normalized environment
diagonals" d_{e,i}, estimated as empirical activation-weighted sensitivity with
every calibration environment kept apart.  Reading: for the inputs X_e
(tokens x K) of environment e,

    m_{e,k} = (1 / N_e) * sum_t x_{t,k}^2          (column mean of squares)
    d_{e,k} = m_{e,k} / ((1 / K) * sum_j m_{e,j})   (each environment to mean 1)

computed from the exact values of the inputs; the sums here are correctly
rounded (math.fsum), d is rounded once to fp32.  An environment without tokens,
or whose activations are all zero, gives NaN.
"""
from __future__ import annotations

import math

import numpy as np

BF16, FP16, FP32 = 0, 1, 2


def decode(X, dtype: int) -> np.ndarray:
    """Exact float64 values of bf16 / fp16 bit patterns (uint16) or fp32 values."""
    X = np.asarray(X)
    if dtype == BF16:
        return (X.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == FP16:
        return X.astype(np.uint16).view(np.float16).astype(np.float64)
    if dtype == FP32:
        return X.astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


def column_means(X, dtype: int, offsets) -> np.ndarray:
    """m [E, K] float64: per environment e (rows offsets[e] .. offsets[e+1]-1),
    the correctly rounded sum of squares of each column divided by N_e."""
    x = decode(X, dtype)
    offsets = [int(o) for o in offsets]
    E, K = len(offsets) - 1, x.shape[1]
    m = np.zeros((E, K), dtype=np.float64)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        sq = x[a:b] * x[a:b]  # exact: at most 48 significant bits
        for k in range(K):
            m[e, k] = math.fsum(sq[:, k]) / (b - a) if b > a else math.nan
    return m


def normalise(m) -> np.ndarray:
    """d [E, K] float32: each environment divided by its mean over columns."""
    m = np.asarray(m, dtype=np.float64)
    out = np.zeros(m.shape, dtype=np.float64)
    for e in range(m.shape[0]):
        mean = math.fsum(m[e]) / m.shape[1]
        out[e] = m[e] / mean if mean != 0 else math.nan
    return out.astype(np.float32)


def estimate(X, dtype: int, offsets):
    """(m float64 [E, K], d float32 [E, K])."""
    m = column_means(X, dtype, offsets)
    return m, normalise(m)
