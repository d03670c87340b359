"""GPU parity of the comparison policies and the reconstruction proxy
(CliffQuant project page, "Held-out reconstruction proxy"): AbsMax scales and
codes, pooled diagonals and the objective of given scales are bit-exact against
the oracle; the Pooled-WMSE selection follows the selection's parity rule; the
proxy's reductions agree with correctly rounded sums to 1e-12 relative."""
import numpy as np
import pytest

from oracle import policies as OP
from minimax_scale_search_b200 import synth
from parity import check_against_oracle, groups_and_diag

pytestmark = pytest.mark.gpu

PROXY_REL = 1e-12  # fp64 sums of <= 4096 non-negative terms in any order: < 4096 * 2^-53


def _cuda(a, dtype=None):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda() if dtype is None else torch.from_numpy(a).to(dtype).cuda()


def _host_bits(scales, codes):
    return scales.cpu().numpy().view(np.uint16), codes.cpu().numpy().view(np.uint32)


def _with_nonfinite(W):
    W = W.copy()
    W[1, 7] = 0x7C00   # +inf
    W[2, 0] = 0xFE00   # NaN
    W[3, 127] = 0xFC00  # -inf
    return W


def test_absmax_matches_oracle():
    from minimax_scale_search_b200 import cq
    wl4 = synth.workload(4)
    cls = synth.stress_classes()
    pick = np.concatenate([np.nonzero(cls == c)[0][:300] for c in range(5)])
    W4, _ = synth.group_rows(4, np.sort(pick))
    Wp, _, _ = synth.make_proxy_inputs()
    # tiny weights: max|w| / 7 lands in the subnormal range, where codes reach the clip
    sub = (np.random.default_rng(8).integers(-40, 41, (96, 128)) * 2.0 ** -24).astype(np.float16).view(np.uint16)
    for name, W in (("tiny", synth.make_weights(1).reshape(-1, 128)), ("stress", W4),
                    ("proxy", Wp), ("nonfinite", _with_nonfinite(Wp[:40])), ("subnormal scales", sub)):
        s, c = cq.absmax_scales(_cuda(W))
        gs, gc = _host_bits(s, c)
        es, ec = OP.absmax_policy(W)
        assert np.array_equal(gs, es), (name, np.nonzero(gs != es)[0][:5])
        assert np.array_equal(gc, ec), (name, np.nonzero((gc != ec).any(axis=1))[0][:5])
    assert wl4.E == 8


def test_absmax_ragged_and_empty():
    import torch
    from minimax_scale_search_b200 import cq
    Wp, _, _ = synth.make_proxy_inputs()
    for G in (1, 3, 5, 31, 33, 4095):  # partial four-group iterations and partial CTAs
        s, c = cq.absmax_scales(_cuda(Wp[:G]))
        gs, gc = _host_bits(s, c)
        es, ec = OP.absmax_policy(Wp[:G])
        assert np.array_equal(gs, es) and np.array_equal(gc, ec), G
    s, c = cq.absmax_scales(torch.empty((0, 128), dtype=torch.int16, device="cuda"))
    assert s.numel() == 0 and c.numel() == 0


def test_pool_diagonals_bit_exact():
    from minimax_scale_search_b200 import cq
    rng = np.random.default_rng(31)
    for E, n in ((1, 777), (2, 4096), (3, 1_000_003), (4, 16384), (7, 129), (8, 300_001)):
        D = (2.0 ** rng.uniform(-20, 20, (E, n)) * rng.uniform(1, 2, (E, n))).astype(np.float32)
        got = cq.pool_diagonals(_cuda(D)).cpu().numpy()
        assert got.shape == (1, n)
        assert np.array_equal(got.view(np.uint32), OP.pool_diagonals(D).view(np.uint32)), (E, n)
    _, Dp, _ = synth.make_proxy_inputs()
    got = cq.pool_diagonals(_cuda(Dp)).cpu().numpy()
    assert got.shape == (1,) + Dp.shape[1:]
    assert np.array_equal(got.view(np.uint32), OP.pool_diagonals(Dp).view(np.uint32))


def test_pooled_selection_parity():
    from minimax_scale_search_b200 import cq
    import torch
    wl = synth.workload(2)
    W = synth.make_weights(2, 0, 512)
    D = synth.make_diagonals(2)
    res = cq.select_scales_pooled(_cuda(W), _cuda(D), want_objective=True, want_flags=True)
    torch.cuda.synchronize()
    gs, gc = _host_bits(res.scales, res.codes)
    gpu = dict(scales=gs, codes=gc, obj=res.objective.cpu().numpy())
    Wg, Dg = groups_and_diag(W, OP.pool_diagonals(D), wl.cols)
    check_against_oracle(Wg, Dg, gpu, where="pooled workload 2")
    # the policy differs from minimax on real-shaped inputs
    mm = cq.select_scales(_cuda(W), _cuda(D))
    assert not torch.equal(mm.scales, res.scales)


def _objective_case(name):
    if name == "per_column_E4":
        W = synth.make_weights(1).reshape(-1, 128)
        D = synth.make_diagonals(1)
        return W, D, synth.workload(1).cols
    if name == "per_group_E1":
        W, D, _ = synth.make_proxy_inputs(groups=700, modules=9, E=1)
        return W, D, 0
    if name == "per_group_E8":
        W, D, _ = synth.make_proxy_inputs(groups=333, modules=5, E=8)
        return W, D, 0
    raise ValueError(name)


@pytest.mark.parametrize("name", ["per_column_E4", "per_group_E1", "per_group_E8"])
def test_group_objective_bit_exact(name):
    from minimax_scale_search_b200 import cq
    W, D, K = _objective_case(name)
    G = W.shape[0]
    Wt, Dt = _cuda(W), _cuda(D)
    rng = np.random.default_rng(33)
    absm, _ = cq.absmax_scales(Wt)
    mm = cq.select_scales(Wt, Dt, K or None).scales
    rand = rng.integers(1, 0x7C00, G).astype(np.uint16)
    rand[:4] = [0x0001, 0x7BFF, 0x03FF, 0x0400]  # grid ends and the subnormal boundary
    for label, S in (("absmax", absm), ("minimax", mm), ("random", _cuda(rand))):
        obj, per_env = cq.group_objective(Wt, Dt, S, K or None)
        s_host = S.cpu().numpy().view(np.uint16)
        exp = OP.group_objectives(W, D, K, s_host)
        got = per_env.cpu().numpy()
        assert np.array_equal(got.view(np.uint64), exp.view(np.uint64)), (name, label)
        assert np.array_equal(obj.cpu().numpy(), exp.max(axis=1)), (name, label)


def test_reconstruction_proxy_three_policies():
    """The proxy on 4,096 groups over 150 modules for each policy: the GPU's
    CliffQuant and Pooled-WMSE scales pass the selection parity rule, the
    AbsMax scales are bit-exact, and the proxy values agree with the oracle's
    (evaluated at the GPU's scales) to 1e-12."""
    from minimax_scale_search_b200 import cq
    W, D, offsets = synth.make_proxy_inputs()
    res = cq.evaluate_policies(_cuda(W), _cuda(D), offsets)
    assert set(res) == set(cq.POLICIES)
    macros = {}
    for pol, (macro, worst, scales) in res.items():
        s_host = scales.cpu().numpy().view(np.uint16)
        per_env = OP.group_objectives(W, D, 0, s_host)
        _, e_worst, e_macro = OP.reconstruction_proxy(per_env, offsets)
        assert worst.shape == (len(offsets) - 1,)
        assert np.all(np.abs(worst - e_worst) <= PROXY_REL * e_worst), pol
        assert abs(macro - e_macro) <= PROXY_REL * e_macro, pol
        macros[pol] = macro
    # scale parity of the two searched policies (sampled: the exhaustive oracle is slow)
    sel = np.arange(0, W.shape[0], 8)
    for pol, Dsel in (("cliffquant", D), ("pooled_wmse", OP.pool_diagonals(D))):
        s_host = res[pol][2].cpu().numpy().view(np.uint16)
        codes = cq.policy_scales(pol, _cuda(W), _cuda(D))[1].cpu().numpy().view(np.uint32)
        objs = OP.group_objectives(W, Dsel, 0, s_host).max(axis=1)
        gpu = dict(scales=s_host, codes=codes, obj=objs)
        check_against_oracle(W, Dsel, gpu, sel=sel, where=f"proxy {pol}")
    s_abs, _ = OP.absmax_policy(W)
    assert np.array_equal(res["absmax"][2].cpu().numpy().view(np.uint16), s_abs)
    # per group, the minimax scale is never worse in the worst environment
    f = {p: OP.group_objectives(W, D, 0, res[p][2].cpu().numpy().view(np.uint16)).max(axis=1)
         for p in cq.POLICIES}
    assert np.all(f["cliffquant"] <= f["pooled_wmse"] * (1 + 1e-12))
    assert np.all(f["cliffquant"] <= f["absmax"] * (1 + 1e-12))
    assert macros["cliffquant"] < macros["absmax"]


def test_reconstruction_proxy_ragged_modules():
    import torch
    from minimax_scale_search_b200 import cq
    rng = np.random.default_rng(34)
    for E, offsets in ((4, [0, 0, 5, 5, 300, 301, 1000]), (1, [0, 1]), (8, [0, 129, 257, 4000]),
                       (3, list(range(0, 600, 3)))):
        G = offsets[-1]
        per_env = rng.lognormal(-8, 2, (G, E))
        env, worst, macro = cq.reconstruction_proxy(_cuda(per_env), offsets)
        e_env, e_worst, e_macro = OP.reconstruction_proxy(per_env, offsets)
        env, worst = env.cpu().numpy(), worst.cpu().numpy()
        nan = np.isnan(e_env)
        assert np.array_equal(np.isnan(env), nan)
        assert np.all(np.abs(env[~nan] - e_env[~nan]) <= PROXY_REL * e_env[~nan])
        assert np.array_equal(np.isnan(worst), np.isnan(e_worst))
        ok = ~np.isnan(e_worst)
        assert np.all(np.abs(worst[ok] - e_worst[ok]) <= PROXY_REL * e_worst[ok])
        m = float(macro.cpu()[0])
        assert (np.isnan(m) and np.isnan(e_macro)) or abs(m - e_macro) <= PROXY_REL * e_macro
        # deterministic: a second call gives identical bits
        env2, worst2, macro2 = cq.reconstruction_proxy(_cuda(per_env), offsets)
        assert np.array_equal(env2.cpu().numpy().view(np.uint64), env.view(np.uint64))
    empty = cq.reconstruction_proxy(torch.empty((0, 4), dtype=torch.float64, device="cuda"), [0])
    assert empty[1].numel() == 0 and np.isnan(float(empty[2].cpu()[0]))
