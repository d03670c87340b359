"""GPU parity of the GPTQ v1 export and dequantisation (csrc/cq_gptq.cu)
against the oracle's element-by-element versions (oracle/gptq.py), on seeded
random inputs: bit-exact for every tensor and every output value."""
import numpy as np
import pytest

from oracle import gptq as OQ
from minimax_scale_search_b200 import synth

pytestmark = pytest.mark.gpu


def _cuda(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(a).cuda()


def _bits(t, dtype):
    return t.cpu().numpy().view(dtype)


@pytest.mark.parametrize("R,K", [(8, 128), (40, 384), (264, 1024), (3072, 1024), (8, 16384)])
def test_export_bit_exact(R, K):
    from minimax_scale_search_b200 import cq
    G = R * K // 128
    scales, codes = synth.make_codes(G, seed=R * 7 + K)
    t = cq.gptq_export(_cuda(scales), _cuda(codes), R, K)
    qw, qz, gs, gi = OQ.export_v1(scales, codes, R, K)
    assert np.array_equal(_bits(t.qweight, np.uint32), qw.view(np.uint32))
    assert np.array_equal(_bits(t.qzeros, np.uint32), qz.view(np.uint32))
    assert np.array_equal(_bits(t.scales, np.uint16), gs)
    assert np.array_equal(t.g_idx.cpu().numpy(), gi)


@pytest.mark.parametrize("R,K", [(40, 384), (264, 1024)])
def test_export_unaligned_words_take_the_three_launch_path(R, K):
    """Code words that start 4 bytes past a 16-byte boundary: the export runs
    its scalar transposes, with the same bytes as the oracle."""
    import torch
    from minimax_scale_search_b200 import cq
    G = R * K // 128
    scales, codes = synth.make_codes(G, seed=R + 3 * K)
    buf = torch.zeros(G * 16 + 1, dtype=torch.int32, device="cuda")
    buf[1:] = _cuda(codes).reshape(-1)
    words = buf[1:].view(G, 16)
    assert words.data_ptr() % 16 == 4
    t = cq.gptq_export(_cuda(scales), words, R, K)
    qw, qz, gs, gi = OQ.export_v1(scales, codes, R, K)
    assert np.array_equal(_bits(t.qweight, np.uint32), qw.view(np.uint32))
    assert np.array_equal(_bits(t.qzeros, np.uint32), qz.view(np.uint32))
    assert np.array_equal(_bits(t.scales, np.uint16), gs)
    assert np.array_equal(t.g_idx.cpu().numpy(), gi)


def test_export_sweep_size_sampled_rows():
    """The sweep's layer shape (30,336 x 16,384): rows sampled in blocks of 8,
    each compared with the oracle's export of just those rows."""
    from minimax_scale_search_b200 import cq
    R, K = 30336, 16384
    G = R * K // 128
    scales, codes = synth.make_codes(G, seed=5)
    t = cq.gptq_export(_cuda(scales), _cuda(codes), R, K)
    qw = _bits(t.qweight, np.uint32)
    gs = _bits(t.scales, np.uint16)
    gpr = K // 128
    for r0 in (0, 8, 15000, R - 8):
        rows = np.arange(r0, r0 + 8)
        sel = (rows[:, None] * gpr + np.arange(gpr)[None, :]).ravel()
        oqw, _, ogs, _ = OQ.export_v1(scales[sel], codes[sel], 8, K)
        assert np.array_equal(qw[:, rows], oqw.view(np.uint32)), r0
        assert np.array_equal(gs[:, rows], ogs), r0
    assert np.all(_bits(t.qzeros, np.uint32) == 0x77777777)


@pytest.mark.parametrize("act_order", [False, True])
@pytest.mark.parametrize("R,K", [(8, 128), (40, 384), (1024, 2048)])
def test_dequantize_bit_exact(R, K, act_order):
    import torch
    from minimax_scale_search_b200 import cq
    qw, qz, gs, gi = synth.make_gptq_tensors(R, K, seed=R + K, act_order=act_order)
    t = cq.GPTQTensors(_cuda(qw), _cuda(qz), _cuda(gs).view(torch.float16), _cuda(gi))
    exp = OQ.dequantize_v1(qw, qz, gs, gi)
    got32 = cq.gptq_dequantize(t).cpu().numpy()
    assert np.array_equal(got32.astype(np.float64), exp)
    got16 = cq.gptq_dequantize(t, half=True).cpu().numpy()
    with np.errstate(over="ignore"):  # products above 65504 round to inf on both sides
        exp16 = exp.astype(np.float16)
    assert np.isinf(exp16).any() or R < 1024
    assert np.array_equal(got16.view(np.uint16), exp16.view(np.uint16))


def test_round_trip_to_s_times_q():
    """export then dequantise gives s * q of the selection's own codes."""
    from minimax_scale_search_b200 import cq
    R, K = 96, 512
    G = R * K // 128
    scales, codes = synth.make_codes(G, seed=77)
    w = cq.gptq_dequantize(cq.gptq_export(_cuda(scales), _cuda(codes), R, K)).cpu().numpy()
    q = OQ.unpack_group_codes(codes).astype(np.int64) - 8
    s = scales.view(np.float16).astype(np.float64)
    exp = (s[:, None] * q).reshape(R, K // 128, 128).reshape(R, K)
    assert np.array_equal(w.astype(np.float64), exp)
