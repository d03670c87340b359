"""Host-side logic of the multi-GPU benchmark on CPU: two gloo ranks on
127.0.0.1.  Every rank solves its own matrix (no data exchange); the job time
is the max over ranks; the job rate counts every rank's groups."""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    from minimax_scale_search_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        m = bench.rank_matrix(rank)
        W = synth.make_weights(5, 0, 4, matrix=m)  # first rows of this rank's matrix
        times = bench.max_over_ranks([10.0 + rank, 3.0 - rank], dist, "cpu")
        counts = bench.sum_over_ranks({"fallback": rank + 1, "near_tie": 10 * rank}, dist, "cpu")
        dist.barrier()
        out[rank] = (m, int(W.astype(np.int64).sum()), times[0], times[1],
                     bench.job_rate(world, 1000, times[0]), counts)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_take_max():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    (m0, s0, t0a, t0b, v0, c0), (m1, s1, t1a, t1b, v1, c1) = out[0], out[1]
    assert (m0, m1) == (0, 1) and s0 != s1          # different matrices per rank
    assert t0a == t1a == 11.0 and t0b == t1b == 3.0  # max over ranks, identical on every rank
    assert v0 == v1 == 2 * 1000 / 11.0
    assert c0 == c1 == {"fallback": 3, "near_tie": 10}  # counters summed over ranks
