"""Multi-rank host logic on CPU: two gloo ranks on 127.0.0.1.

* The benchmark's helpers: the job time is the max over ranks, the job rate
  counts the whole job's groups, counters are summed.
* The partition of a real workload: each rank solves its contiguous block of
  whole rows (tiny workload, and the first 96 rows of the projection
  workload) with the diagonals replicated; the per-rank solver here is the
  CPU oracle, the checker, not the product path.  The blocks, gathered in rank
  order over the process group, equal the single-rank result byte for byte.
* The several-matrix job (32 matrices) splits into whole matrices that cover
  every matrix exactly once.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_rows(idx, r0, r1):
    """Oracle scales (int16 view) and packed codes (int32 view) of rows [r0, r1)."""
    import oracle
    from minimax_scale_search_b200 import synth
    wl = synth.workload(idx)
    W = synth.make_weights(idx, r0, r1)
    D = synth.make_diagonals(idx)
    o = oracle.solve(W.reshape(-1, 128), D, K=wl.cols, threads=max(1, (os.cpu_count() or 2) // 2))
    return o["best_bits"].view(np.int16), oracle.pack_codes(o["codes"]).view(np.int32)


WORKLOADS = ((1, 64), (2, 96))  # (workload, rows solved)


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    from minimax_scale_search_b200 import shard, synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        times = bench.max_over_ranks([10.0 + rank, 3.0 - rank], dist, "cpu")
        counts = bench.sum_over_ranks({"fallback": rank + 1, "near_tie": 10 * rank}, dist, "cpu")
        res = {"times": times, "rate": bench.job_rate(2000, times[0]), "counts": counts}
        for idx, rows in WORKLOADS:
            r0, r1 = shard.row_block(rank, world, rows)
            s, c = _oracle_rows(idx, r0, r1)
            gpr = synth.workload(idx).groups_per_row
            res[f"block{idx}"] = (r0, r1)
            res[f"scales{idx}"] = shard.gather_rows(torch.from_numpy(s), world, rows, dist, gpr).numpy()
            res[f"codes{idx}"] = shard.gather_rows(torch.from_numpy(c), world, rows, dist, gpr).numpy()
        res["matrices"] = shard.matrix_block(rank, world, synth.workload(5).n_matrices)
        dist.barrier()
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    return dict(out[0]), dict(out[1])


def test_two_gloo_ranks_take_max_and_sum(two_ranks):
    a, b = two_ranks
    assert a["times"] == b["times"] == [11.0, 3.0]        # max over ranks, identical on every rank
    assert a["rate"] == b["rate"] == 2000 / 11.0           # the whole job's groups over the slowest rank
    assert a["counts"] == b["counts"] == {"fallback": 3, "near_tie": 10}


@pytest.mark.parametrize("idx,rows", WORKLOADS)
def test_row_blocks_gathered_equal_single_rank(two_ranks, idx, rows):
    a, b = two_ranks
    assert a[f"block{idx}"] == (0, rows // 2) and b[f"block{idx}"] == (rows // 2, rows)
    s1, c1 = _oracle_rows(idx, 0, rows)
    for r in (a, b):
        assert np.array_equal(r[f"scales{idx}"], s1)
        assert np.array_equal(r[f"codes{idx}"], c1)


def test_matrix_blocks_cover_the_job(two_ranks):
    a, b = two_ranks
    assert a["matrices"] == (0, 16) and b["matrices"] == (16, 32)


def test_blocks_partition_exactly():
    from minimax_scale_search_b200 import shard
    for n in (0, 1, 7, 32, 30336):
        for world in (1, 2, 3, 4, 8):
            spans = [shard.block(r, world, n) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[k][1] == spans[k + 1][0] for k in range(world - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    assert [shard.matrix_block(r, 8, 32) for r in range(8)] == [(4 * r, 4 * r + 4) for r in range(8)]
    assert [shard.row_block(r, 8, 30336) for r in range(8)] == [(3792 * r, 3792 * (r + 1)) for r in range(8)]
    with pytest.raises(ValueError):
        shard.block(2, 2, 10)
