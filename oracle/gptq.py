"""GPTQ v1 checkpoint tensors, plain CPU versions (test infrastructure: only
the tests, the smoke check and the benchmark's CPU leg use this module; it
shares no code with the CUDA path).

CliffQuant project page and the FriendliAI model card, "Quantization
configuration": the released checkpoint is GPTQ v1, 4-bit, group size 128,
symmetric, act-order off.  The pages do not print the tensor layout; this
follows the public GPTQ v1 format for a linear layer with weight [R, K]
(R output features, K input features):

* ``qweight`` int32 [K/8, R]: word (k, r) holds the unsigned codes u of
  inputs 8k .. 8k+7 of output r, input 8k + j in bits 4j .. 4j+3;
* ``qzeros``  int32 [K/128, R/8]: word (g, c) holds the stored zeros of
  outputs 8c .. 8c+7, output 8c + j in bits 4j .. 4j+3; v1 stores the zero
  point minus one, so a symmetric 4-bit zero of 8 is stored as 7;
* ``scales``  fp16 [K/128, R];
* ``g_idx``   int32 [K]: the group of each input, i // 128 with act-order off.

Dequantisation (v1): w[r, i] = scales[g, r] * (u[r, i] - (z[g, r] + 1)) with
g = g_idx[i].  The selection's codes are u = q + 8, so the zero point is 8
and the dequantised weight is s * q.
"""
from __future__ import annotations

import numpy as np

GROUP = 128
ZERO = 8  # symmetric 4-bit zero point


def unpack_group_codes(codes) -> np.ndarray:
    """Packed selection codes uint32 [G, 16] -> unsigned nibbles u uint8 [G, 128]
    (element i of a group in word i // 8, bits 4 (i % 8) ..)."""
    codes = np.asarray(codes, dtype=np.uint32)
    G = codes.shape[0]
    u = np.zeros((G, GROUP), dtype=np.uint8)
    for i in range(GROUP):
        u[:, i] = (codes[:, i // 8] >> np.uint32(4 * (i % 8))) & np.uint32(0xF)
    return u


def export_v1(scales, codes, R: int, K: int):
    """(qweight, qzeros, scales, g_idx) of an [R, K] weight whose groups run along
    rows (group g = row g // (K/128), columns (g % (K/128)) * 128 ..).
    scales: binary16 bits uint16 [G]; codes uint32 [G, 16]."""
    if K % GROUP or R % 8:
        raise ValueError("K must be a multiple of 128 and R a multiple of 8")
    gpr = K // GROUP
    u = unpack_group_codes(codes).reshape(R, gpr, GROUP).reshape(R, K)
    qweight = np.zeros((K // 8, R), dtype=np.uint32)
    for i in range(K):
        qweight[i // 8, :] |= u[:, i].astype(np.uint32) << np.uint32(4 * (i % 8))
    qzeros = np.zeros((gpr, R // 8), dtype=np.uint32)
    for r in range(R):
        qzeros[:, r // 8] |= np.uint32(ZERO - 1) << np.uint32(4 * (r % 8))
    gscales = np.asarray(scales, dtype=np.uint16).reshape(R, gpr).T.copy()
    g_idx = (np.arange(K) // GROUP).astype(np.int32)
    return qweight.view(np.int32), qzeros.view(np.int32), gscales, g_idx


def dequantize_v1(qweight, qzeros, scales, g_idx) -> np.ndarray:
    """float64 [R, K] by the v1 definition (every value is exact: an 11-bit
    scale times an integer below 16 in magnitude)."""
    qweight = np.asarray(qweight).view(np.uint32)
    qzeros = np.asarray(qzeros).view(np.uint32)
    s = np.asarray(scales, dtype=np.uint16).view(np.float16).astype(np.float64)
    g_idx = np.asarray(g_idx, dtype=np.int64)
    K = qweight.shape[0] * 8
    R = qweight.shape[1]
    out = np.zeros((R, K), dtype=np.float64)
    for i in range(K):
        g = g_idx[i]
        u = (qweight[i // 8, :] >> np.uint32(4 * (i % 8))) & np.uint32(0xF)
        z = np.array([(qzeros[g, r // 8] >> np.uint32(4 * (r % 8))) & np.uint32(0xF) for r in range(R)],
                     dtype=np.int64)
        out[:, i] = s[g, :] * (u.astype(np.int64) - (z + 1))
    return out
