"""The allocation-free entry point, cq_select_scales_noalloc.

It serves callers that cannot allocate device memory when they call in (code
inside an allocator callback or under a fixed memory budget, runtimes that
plan device memory up front): its scratch is one fixed array compiled into
libcq.so instead of a workspace from the caller or a pool.  These tests call
it through the C ABI and check that it returns exactly what the regular entry
point returns, on two calls in a row that share (and so reuse) that array.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from minimax_scale_search_b200 import synth


@pytest.fixture(scope="module")
def cq():
    """The binding, after an in-tree build of libcq.so (a fresh checkout has none)."""
    from minimax_scale_search_b200 import build
    build.build()
    from minimax_scale_search_b200 import cq as binding
    return binding


def _noalloc(cq, Wt, G, Dt, E, K, S, C, stream_handle):
    vp = ctypes.c_void_p
    return cq.lib.cq_select_scales_noalloc(vp(Wt), G, vp(Dt), E, K, vp(S), vp(C), vp(stream_handle))


def test_noalloc_rejects_more_groups_than_its_scratch_holds(cq):
    # returns before anything is enqueued, so plain (never dereferenced) addresses suffice
    fake = 0x10000
    G = cq.NOALLOC_MAX_GROUPS + 1
    assert _noalloc(cq, fake, G, fake, 4, 0, fake, fake, None) == cq.CQ_ERR_TOO_LARGE
    assert "fixed scratch" in cq.status_string(cq.CQ_ERR_TOO_LARGE)
    assert _noalloc(cq, fake, 8, fake, 9, 0, fake, fake, None) == cq.CQ_ERR_UNSUPPORTED
    assert _noalloc(cq, 0, 0, 0, 4, 0, 0, 0, None) == cq.CQ_OK


@pytest.mark.gpu
def test_noalloc_matches_regular_entry_point_on_two_calls(cq):
    import torch
    stream = torch.cuda.current_stream()
    for idx, rows in ((4, 256), (2, 3072)):  # E=8 with exhaustive-fallback groups, then E=4
        wl = synth.workload(idx)
        W = synth.make_weights(idx, 0, rows)
        D = synth.make_diagonals(idx)
        Wt = torch.from_numpy(W.view(np.int16)).cuda()
        Dt = torch.from_numpy(D).cuda()
        G = W.size // 128
        ref = cq.select_scales(Wt, Dt, want_flags=True)
        S = torch.full((G,), -1, dtype=torch.int16, device="cuda")
        C = torch.full((G, 16), -1, dtype=torch.int32, device="cuda")
        st = _noalloc(cq, Wt.data_ptr(), G, Dt.data_ptr(), wl.E, wl.cols, S.data_ptr(), C.data_ptr(),
                      stream.cuda_stream)
        assert st == cq.CQ_OK, cq.status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(S, ref.scales)
        assert torch.equal(C, ref.codes)
        if idx == 4:
            assert int((ref.flags & cq.FLAG_FALLBACK).sum()) > 0  # the fixed queue was used
