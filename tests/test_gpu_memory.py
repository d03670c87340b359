"""Device memory the allocating entry points keep, and how a caller returns it.

cq_select_scales takes its workspace from a library pool whose freed blocks
stay reserved for the next call; cq_trim_memory hands them back to the
device.  Measured with the device-wide free-memory count, which the torch
caching allocator does not affect."""
import numpy as np
import pytest

from minimax_scale_search_b200 import synth

pytestmark = pytest.mark.gpu


def test_pool_keeps_the_workspace_until_trimmed():
    import torch
    from minimax_scale_search_b200 import cq
    rows = 16384  # 2,097,152 groups: a 16 MiB workspace
    W = synth.make_weights(3, 0, rows)
    D = synth.make_diagonals(3)
    Wt = torch.from_numpy(W.view(np.int16)).cuda()
    Dt = torch.from_numpy(D).cuda()
    s = torch.empty(W.size // 128, dtype=torch.int16, device="cuda")
    c = torch.empty((W.size // 128, 16), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    cq.trim_memory()
    free0 = torch.cuda.mem_get_info()[0]
    cq.select_scales_plain(Wt, Dt, out_scales=s, out_codes=c)
    torch.cuda.synchronize()
    kept = free0 - torch.cuda.mem_get_info()[0]
    ws = cq.workspace_bytes(W.size // 128, 4)
    assert kept >= ws  # the freed workspace stays reserved by the pool
    cq.trim_memory()
    back = torch.cuda.mem_get_info()[0] - (free0 - kept)
    assert back >= ws  # and is returned by the trim
    # the pool is reused: a second call reserves no more than the first
    cq.select_scales_plain(Wt, Dt, out_scales=s, out_codes=c)
    cq.select_scales_plain(Wt, Dt, out_scales=s, out_codes=c)
    torch.cuda.synchronize()
    assert free0 - torch.cuda.mem_get_info()[0] <= kept
    cq.trim_memory()
