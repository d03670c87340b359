"""C-ABI checks that need no GPU: the library loads, exports every function
include/cq.h declares, and rejects bad arguments before enqueuing anything."""
import ctypes

import numpy as np
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cq.h")


@pytest.fixture(scope="module")
def cq():
    from minimax_scale_search_b200 import build
    build.build()
    from minimax_scale_search_b200 import cq as mod
    return mod


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(cq_\w+)\s*\(", src, flags=re.M)


def test_header_declares_expected_entry_points(cq):
    names = declared_functions()
    assert set(names) == set(cq.EXPORTS)


def test_library_exports_every_declared_symbol(cq):
    out = subprocess.run(["nm", "-D", "--defined-only", cq.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(cq.lib, name)


def test_allocating_entry_points_document_the_pool(cq):
    """cq_select_scales says that it allocates, from which pool, that the pool
    keeps its blocks, and how to return them; the trim call is exported."""
    src = open(HEADER).read()
    head = src[:src.index("cq_status cq_select_scales(")]
    doc = head[head.rindex("/*"):]
    for phrase in ("allocates", "pool", "release", "cq_trim_memory", "cq_select_scales_ex"):
        assert phrase in doc, phrase
    assert hasattr(cq.lib, "cq_trim_memory")
    noalloc = src[src.index("Allocation-free variant"):src.index("cq_status cq_select_scales_noalloc(")]
    assert "only status" in noalloc  # the allocation-free call reports no counters


def test_status_strings_and_version(cq):
    assert cq.status_string(0) == "CQ_OK"
    for st in range(1, 6):
        assert cq.status_string(st).startswith("CQ_ERR_")
    assert "unknown" in cq.status_string(99)
    assert cq.version() >= 100


def test_workspace_size(cq):
    assert cq.workspace_bytes(0, 4) == 256
    assert cq.workspace_bytes(1, 4) == 512
    assert cq.workspace_bytes(3883008, 4) == 256 + 3883008 * 8


FAKE = 0x10000  # 16-byte aligned fake device address: every call below fails validation first


def call_ex(cq, W=FAKE, G=8, D=FAKE, E=4, K=0, S=FAKE, C=FAKE, opts=None, ws=FAKE, wsb=1 << 20):
    vp = ctypes.c_void_p
    return cq.lib.cq_select_scales_ex(vp(W), G, vp(D), E, K, vp(S), vp(C), vp(None),
                                      ctypes.byref(opts) if opts is not None else None, vp(ws), wsb,
                                      vp(None), vp(None))


def test_argument_errors_are_synchronous(cq):
    assert call_ex(cq, E=0) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, E=9) == cq.CQ_ERR_UNSUPPORTED
    assert call_ex(cq, G=-1) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, K=-128) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, K=100) == cq.CQ_ERR_INVALID_ARG          # K % 128 != 0
    assert call_ex(cq, G=9, K=256) == cq.CQ_ERR_INVALID_ARG     # G not whole rows of K/128 groups
    assert call_ex(cq, G=1 << 32) == cq.CQ_ERR_UNSUPPORTED
    assert call_ex(cq, W=0) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, D=0) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, S=0) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, C=0) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, W=FAKE + 8) == cq.CQ_ERR_INVALID_ARG     # W not 16-byte aligned
    assert call_ex(cq, D=FAKE + 4) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, C=FAKE + 2) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, ws=0) == cq.CQ_ERR_WORKSPACE
    assert call_ex(cq, wsb=100) == cq.CQ_ERR_WORKSPACE
    assert call_ex(cq, ws=FAKE + 16) == cq.CQ_ERR_WORKSPACE     # not 256-byte aligned
    assert call_ex(cq, opts=cq.Opts(65, 0, 0.0, None, None)) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, opts=cq.Opts(-1, 0, 0.0, None, None)) == cq.CQ_ERR_INVALID_ARG
    assert call_ex(cq, opts=cq.Opts(0, 0, -1.0, None, None)) == cq.CQ_ERR_INVALID_ARG


def test_plain_and_host_entry_points_validate(cq):
    vp = ctypes.c_void_p
    assert cq.lib.cq_select_scales(vp(FAKE), 8, vp(FAKE), 0, 0, vp(FAKE), vp(FAKE), vp(None)) == \
        cq.CQ_ERR_INVALID_ARG
    assert cq.lib.cq_select_scales(vp(None), 0, vp(None), 4, 0, vp(None), vp(None), vp(None)) == cq.CQ_OK
    assert cq.lib.cq_select_scales_host(vp(None), 8, vp(FAKE), 4, 0, vp(FAKE), vp(FAKE), vp(None)) == \
        cq.CQ_ERR_INVALID_ARG
    assert cq.lib.cq_select_scales_host(vp(None), 0, vp(None), 4, 0, vp(None), vp(None), vp(None)) == cq.CQ_OK
    assert cq.lib.cq_read_counters(vp(None), vp(FAKE), vp(None)) == cq.CQ_ERR_INVALID_ARG
    assert cq.lib.cq_get_status(vp(None), vp(None)) == cq.CQ_ERR_INVALID_ARG


def test_policy_entry_points_validate(cq):
    vp, L = ctypes.c_void_p, cq.lib
    f = vp(FAKE)
    # AbsMax: W [G][128] binary16, 16-byte aligned
    assert L.cq_absmax_scales(f, -1, f, f, vp(None)) == cq.CQ_ERR_INVALID_ARG
    assert L.cq_absmax_scales(f, 1 << 32, f, f, vp(None)) == cq.CQ_ERR_UNSUPPORTED
    assert L.cq_absmax_scales(vp(None), 0, vp(None), vp(None), vp(None)) == cq.CQ_OK
    assert L.cq_absmax_scales(vp(FAKE + 8), 4, f, f, vp(None)) == cq.CQ_ERR_INVALID_ARG
    assert L.cq_absmax_scales(f, 4, f, vp(FAKE + 2), vp(None)) == cq.CQ_ERR_INVALID_ARG
    assert L.cq_absmax_scales(f, 4, f, vp(FAKE + 4), vp(None)) == cq.CQ_ERR_INVALID_ARG  # codes need 16 B
    assert L.cq_absmax_scales(f, 4, vp(None), f, vp(None)) == cq.CQ_ERR_INVALID_ARG
    # pooling: 1 <= E <= 8
    assert L.cq_pool_diagonals(f, 0, 10, f, vp(None)) == cq.CQ_ERR_INVALID_ARG
    assert L.cq_pool_diagonals(f, 9, 10, f, vp(None)) == cq.CQ_ERR_UNSUPPORTED
    assert L.cq_pool_diagonals(f, 4, -1, f, vp(None)) == cq.CQ_ERR_INVALID_ARG
    assert L.cq_pool_diagonals(vp(None), 4, 0, vp(None), vp(None)) == cq.CQ_OK
    assert L.cq_pool_diagonals(vp(None), 4, 10, f, vp(None)) == cq.CQ_ERR_INVALID_ARG
    # objective of given scales
    obj = lambda G=8, E=4, K=0, W=FAKE, D=FAKE, S=FAKE, P=FAKE, O=FAKE: L.cq_group_objective(  # noqa: E731
        vp(W), G, vp(D), E, K, vp(S), vp(P), vp(O), vp(None))
    assert obj(E=0) == cq.CQ_ERR_INVALID_ARG
    assert obj(E=9) == cq.CQ_ERR_UNSUPPORTED
    assert obj(G=-1) == cq.CQ_ERR_INVALID_ARG
    assert obj(K=100) == cq.CQ_ERR_INVALID_ARG
    assert obj(G=9, K=256) == cq.CQ_ERR_INVALID_ARG
    assert obj(S=0) == cq.CQ_ERR_INVALID_ARG
    assert obj(P=FAKE + 4) == cq.CQ_ERR_INVALID_ARG
    assert obj(D=FAKE + 4) == cq.CQ_ERR_INVALID_ARG
    assert obj(W=FAKE + 8) == cq.CQ_ERR_INVALID_ARG
    assert obj(G=0, W=0, D=0, S=0, P=0, O=0) == cq.CQ_OK
    # proxy reductions
    prox = lambda G=8, E=4, nmod=3, scale=1.0, X=FAKE, off=FAKE: L.cq_reconstruction_proxy(  # noqa: E731
        vp(X), G, E, nmod, vp(off), scale, f, f, f, vp(None))
    assert prox(G=-1) == cq.CQ_ERR_INVALID_ARG
    assert prox(E=0) == cq.CQ_ERR_INVALID_ARG
    assert prox(E=9) == cq.CQ_ERR_UNSUPPORTED
    assert prox(nmod=-1) == cq.CQ_ERR_INVALID_ARG
    assert prox(scale=float("nan")) == cq.CQ_ERR_INVALID_ARG
    assert prox(X=FAKE + 4) == cq.CQ_ERR_INVALID_ARG
    assert prox(off=0) == cq.CQ_ERR_INVALID_ARG
    assert prox(nmod=0, X=0, off=0) == cq.CQ_OK


def test_gptq_entry_points_validate(cq):
    vp, L, f = ctypes.c_void_p, cq.lib, ctypes.c_void_p(FAKE)
    exp = lambda R=8, K=128, S=FAKE, C=FAKE: L.cq_gptq_export(vp(S), vp(C), R, K, f, f, f, f, vp(None))  # noqa: E731
    assert exp(R=4) == cq.CQ_ERR_INVALID_ARG      # R % 8
    assert exp(K=100) == cq.CQ_ERR_INVALID_ARG    # K % 128
    assert exp(R=-8) == cq.CQ_ERR_INVALID_ARG
    assert exp(R=1 << 31) == cq.CQ_ERR_UNSUPPORTED
    assert exp(S=0) == cq.CQ_ERR_INVALID_ARG
    assert exp(C=FAKE + 2) == cq.CQ_ERR_INVALID_ARG
    assert exp(R=0, S=0, C=0) == cq.CQ_OK
    deq = lambda R=8, K=128, half=0, out=FAKE: L.cq_gptq_dequantize(f, f, f, f, R, K, half, vp(out), vp(None))  # noqa: E731
    assert deq(half=2) == cq.CQ_ERR_INVALID_ARG
    assert deq(out=FAKE + 8) == cq.CQ_ERR_INVALID_ARG  # out must be 16-byte aligned
    assert deq(K=64) == cq.CQ_ERR_INVALID_ARG
    assert deq(R=0, out=0) == cq.CQ_OK


def test_diagonal_entry_point_validates(cq):
    vp, L = ctypes.c_void_p, cq.lib
    off = np.array([0, 10, 20], dtype=np.int64)
    bad = np.array([0, 20, 10], dtype=np.int64)
    f = vp(FAKE)
    est = lambda dt=0, K=256, o=off, E=2, X=FAKE, M=FAKE: L.cq_estimate_diagonals(  # noqa: E731
        vp(X), dt, K, vp(o.ctypes.data), E, vp(M), f, vp(None))
    assert est(dt=3) == cq.CQ_ERR_INVALID_ARG
    assert est(E=0) == cq.CQ_ERR_INVALID_ARG
    assert est(E=9) == cq.CQ_ERR_UNSUPPORTED
    assert est(K=12) == cq.CQ_ERR_INVALID_ARG            # K % 8
    assert est(o=bad) == cq.CQ_ERR_INVALID_ARG           # offsets must ascend
    assert est(X=FAKE + 8) == cq.CQ_ERR_INVALID_ARG      # X 16-byte aligned
    assert est(M=FAKE + 4) == cq.CQ_ERR_INVALID_ARG
    assert est(K=0) == cq.CQ_OK
    assert L.cq_estimate_diagonals(f, 0, 256, vp(None), 2, f, f, vp(None)) == cq.CQ_ERR_INVALID_ARG


def test_spec_entry_point_validates(cq):
    vp, L, f = ctypes.c_void_p, cq.lib, ctypes.c_void_p(FAKE)

    def call(qmin=-4, qmax=3, n=64, G=8, E=2, K=0, W=FAKE, obj=0):
        spec = cq.QuantizerSpec(qmin, qmax, n)
        return L.cq_select_scales_spec(vp(W), G, f, E, K, ctypes.byref(spec), f, f, vp(obj), vp(None), vp(None))
    assert call(qmin=0) == cq.CQ_ERR_INVALID_ARG
    assert call(qmax=0) == cq.CQ_ERR_INVALID_ARG
    assert call(n=0) == cq.CQ_ERR_INVALID_ARG
    assert call(qmin=-129) == cq.CQ_ERR_UNSUPPORTED
    assert call(qmax=128) == cq.CQ_ERR_UNSUPPORTED
    assert call(n=2048) == cq.CQ_ERR_UNSUPPORTED
    assert call(E=9) == cq.CQ_ERR_UNSUPPORTED
    assert call(K=100) == cq.CQ_ERR_INVALID_ARG     # K % n
    assert call(G=3, K=128) == cq.CQ_ERR_INVALID_ARG  # G not whole rows of K/n groups
    assert call(W=FAKE + 1) == cq.CQ_ERR_INVALID_ARG
    assert call(obj=FAKE + 4) == cq.CQ_ERR_INVALID_ARG
    assert call(G=0, W=0) == cq.CQ_OK
    assert L.cq_select_scales_spec(f, 8, f, 2, 0, None, f, f, vp(None), vp(None), vp(None)) == cq.CQ_ERR_INVALID_ARG


def test_no_cpu_fallback_in_binding():
    """The binding refuses to run without its CUDA library, and no module of the
    package uses the oracle (test infrastructure only)."""
    pkg = os.path.join(ROOT, "minimax_scale_search_b200")
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            src = open(os.path.join(pkg, name)).read()
            assert "import oracle" not in src and "from oracle" not in src, name
    src = open(os.path.join(pkg, "cq.py")).read()
    assert "raise ImportError" in src


def test_binding_raises_without_its_library(tmp_path):
    """Imported from a directory without libcq.so, the binding raises at import
    instead of running anything on the CPU."""
    import importlib.util
    import shutil
    src = os.path.join(ROOT, "minimax_scale_search_b200", "cq.py")
    dst = tmp_path / "cq_copy.py"
    shutil.copy(src, dst)
    spec = importlib.util.spec_from_file_location("cq_copy_without_library", dst)
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="libcq.so"):
        spec.loader.exec_module(mod)
