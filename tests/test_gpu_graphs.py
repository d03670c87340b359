"""The device entry points inside a captured CUDA graph.

With its workspace and outputs supplied, cq_select_scales_ex only enqueues a
counter reset and its kernels on the caller's stream: no allocation, no host
synchronisation.  So a serving loop can capture it once and replay it on new
inputs written into the same buffers.  The general-spec path and the policy
kernels are checked the same way.  Each replay must equal a direct call on the
same inputs, byte for byte."""
import numpy as np
import pytest

from minimax_scale_search_b200 import synth

pytestmark = pytest.mark.gpu


def _second_input(W, seed):
    rng = np.random.default_rng(seed)
    return np.clip(rng.normal(0, 0.03, W.shape), -1, 1).astype(np.float16).view(np.uint16)


def test_selection_replays_in_a_cuda_graph():
    import torch
    from minimax_scale_search_b200 import cq
    W, D = synth.make_inputs(1)
    G = W.size // 128
    Wt = torch.from_numpy(W.view(np.int16)).cuda()
    Dt = torch.from_numpy(D).cuda()
    s = torch.empty(G, dtype=torch.int16, device="cuda")
    c = torch.empty((G, 16), dtype=torch.int32, device="cuda")
    ws = torch.empty(cq.workspace_bytes(G, D.shape[0]), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture
        cq.select_scales(Wt, Dt, out_scales=s, out_codes=c, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    ref_s, ref_c = s.clone(), c.clone()
    s.zero_()
    c.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cq.select_scales(Wt, Dt, out_scales=s, out_codes=c, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(s, ref_s) and torch.equal(c, ref_c)
    # new weights in the captured buffer: the replay follows them
    W2 = _second_input(W, 11)
    Wt.copy_(torch.from_numpy(W2.view(np.int16)))
    g.replay()
    torch.cuda.synchronize()
    direct = cq.select_scales(torch.from_numpy(W2.view(np.int16)).cuda(), Dt)
    torch.cuda.synchronize()
    assert torch.equal(s, direct.scales) and torch.equal(c, direct.codes)
    assert cq.read_counters(ws)["nonfinite"] == 0


def test_general_spec_and_policies_replay_in_a_cuda_graph():
    import torch
    from minimax_scale_search_b200 import cq
    W, D = synth.make_inputs(1)
    Wt = torch.from_numpy(W.view(np.int16)).cuda()
    Dt = torch.from_numpy(D).cuda()
    K = W.shape[1]

    def work():
        r = cq.select_scales_spec(Wt, Dt, K, qmin=-4, qmax=3, group_size=128)
        a_s, a_c = cq.absmax_scales(Wt)
        obj, per_env = cq.group_objective(Wt, Dt, a_s, K)
        return r.scales, r.codes, a_s, a_c, obj, per_env

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        work()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        outs = work()
    W2 = _second_input(W, 12)
    Wt.copy_(torch.from_numpy(W2.view(np.int16)))
    g.replay()
    torch.cuda.synchronize()
    ref = work()
    torch.cuda.synchronize()
    for got, want in zip(outs, ref):
        assert torch.equal(got.view(torch.uint8), want.view(torch.uint8))
