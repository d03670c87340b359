"""How a selection job splits over ranks (one process per GPU).

Groups are independent (CliffQuant project page, "What CliffQuant changes": each
128-weight group picks its own scale), so a job splits with no exchange on the
data path:

* one matrix (the 0.8B-scale sweep) splits into contiguous blocks of whole
  rows; every rank keeps the whole per-column ``[E, K]`` diagonal set, so a
  block's groups see exactly the diagonals they see in the whole matrix;
* a job of several matrices (32 matrices of 14,336 x 4,096) splits into
  contiguous blocks of whole matrices.

The blocks are as even as possible; the first ``n % world`` ranks take one
more.  Concatenating the ranks' outputs in rank order gives the whole job's
output, byte for byte, because each group's result depends on its own inputs
only.  ``gather_rows`` does that concatenation over a process group (NCCL
on GPUs, gloo on CPU) for callers that want every output on every rank.
"""
from __future__ import annotations

import math


def block(rank: int, world: int, n: int) -> tuple[int, int]:
    """Half-open range [lo, hi) of n items owned by `rank` of `world`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    if n < 0:
        raise ValueError("n must be >= 0")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def row_block(rank: int, world: int, rows: int) -> tuple[int, int]:
    """Rows [r0, r1) of one matrix solved by `rank`."""
    return block(rank, world, rows)


def matrix_block(rank: int, world: int, n_matrices: int) -> tuple[int, int]:
    """Matrices [m0, m1) of a several-matrix job solved by `rank`."""
    return block(rank, world, n_matrices)


def gather_rows(local, world: int, rows_total: int, dist, dim0_per_row: int = 1):
    """Every rank's block of a per-row output, concatenated in rank order on
    every rank.  `local` is a tensor whose first dimension covers this rank's
    rows times `dim0_per_row` (groups per row for per-group outputs).  The
    bytes travel as uint8, which every backend carries (NCCL has no 16-bit
    integer type)."""
    import torch
    sizes = [(block(r, world, rows_total)[1] - block(r, world, rows_total)[0]) * dim0_per_row
             for r in range(world)]
    pad = max(sizes)
    item = local.contiguous()
    inner = tuple(item.shape[1:])
    row_bytes = item.element_size() * math.prod(inner)
    buf = torch.zeros((pad, row_bytes), dtype=torch.uint8, device=item.device)
    buf[:item.shape[0]] = item.view(torch.uint8).reshape(item.shape[0], row_bytes)
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf)
    out = torch.cat([p[:n] for p, n in zip(parts, sizes)], dim=0)
    return out.view(item.dtype).reshape((sum(sizes),) + inner)
