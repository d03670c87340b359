"""ctypes binding of libcq.so (argument marshalling only).

Every step of the selection runs in the library's CUDA kernels; PyTorch is used
for device memory, pinned host memory and streams.  Importing this module loads
``libcq.so`` from this package's directory and raises if it is missing: there
is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcq.so")

CQ_OK, CQ_ERR_INVALID_ARG, CQ_ERR_UNSUPPORTED, CQ_ERR_CUDA, CQ_ERR_NONFINITE, CQ_ERR_WORKSPACE, CQ_ERR_TOO_LARGE = range(7)
NOALLOC_MAX_GROUPS = 1 << 20
CQ_NUM_COUNTERS = 8
COUNTER_NAMES = ("fallback", "near_tie", "nonfinite", "trivial", "finalists", "uncertain", "queue", "survivors")
FLAG_TRIVIAL, FLAG_FALLBACK, FLAG_NEAR_TIE, FLAG_NONFINITE = 0x01, 0x02, 0x04, 0x08
GROUP = 128
WORDS = 16
MAX_E = 8

# Symbols the C header declares, in declaration order.
EXPORTS = ("cq_workspace_bytes", "cq_select_scales", "cq_select_scales_ex", "cq_select_scales_host",
           "cq_absmax_scales", "cq_pool_diagonals", "cq_group_objective", "cq_reconstruction_proxy",
           "cq_gptq_export", "cq_gptq_dequantize", "cq_estimate_diagonals", "cq_select_scales_spec",
           "cq_select_scales_noalloc", "cq_trim_memory", "cq_read_counters", "cq_get_status", "cq_status_string",
           "cq_version")


class CQError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}" if where else status_string(status))


class QuantizerSpec(ctypes.Structure):
    """Codes in [qmin, qmax], groups of group_size weights (the pages' QuantizerSpec)."""
    _fields_ = [("qmin", ctypes.c_int32), ("qmax", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("kernel", ctypes.c_int32)]


SPEC_MAX_GROUP = 1024


class Opts(ctypes.Structure):
    _fields_ = [("finalist_cap", ctypes.c_int32), ("force_exhaustive", ctypes.c_int32),
                ("flag_rel_gap", ctypes.c_double), ("ev_main_begin", ctypes.c_void_p),
                ("ev_main_end", ctypes.c_void_p), ("intersections", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m minimax_scale_search_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.cq_workspace_bytes.restype = ctypes.c_size_t
    L.cq_workspace_bytes.argtypes = [i64, i32]
    L.cq_select_scales.restype = i32
    L.cq_select_scales.argtypes = [vp, i64, vp, i32, i64, vp, vp, vp]
    L.cq_select_scales_ex.restype = i32
    L.cq_select_scales_ex.argtypes = [vp, i64, vp, i32, i64, vp, vp, vp, ctypes.POINTER(Opts), vp,
                                      ctypes.c_size_t, vp, vp]
    L.cq_select_scales_host.restype = i32
    L.cq_select_scales_host.argtypes = [vp, i64, vp, i32, i64, vp, vp, vp]
    L.cq_absmax_scales.restype = i32
    L.cq_absmax_scales.argtypes = [vp, i64, vp, vp, vp]
    L.cq_pool_diagonals.restype = i32
    L.cq_pool_diagonals.argtypes = [vp, i32, i64, vp, vp]
    L.cq_group_objective.restype = i32
    L.cq_group_objective.argtypes = [vp, i64, vp, i32, i64, vp, vp, vp, vp]
    L.cq_reconstruction_proxy.restype = i32
    L.cq_reconstruction_proxy.argtypes = [vp, i64, i32, i64, vp, ctypes.c_double, vp, vp, vp, vp]
    L.cq_gptq_export.restype = i32
    L.cq_gptq_export.argtypes = [vp, vp, i64, i64, vp, vp, vp, vp, vp]
    L.cq_gptq_dequantize.restype = i32
    L.cq_gptq_dequantize.argtypes = [vp, vp, vp, vp, i64, i64, i32, vp, vp]
    L.cq_estimate_diagonals.restype = i32
    L.cq_estimate_diagonals.argtypes = [vp, i32, i64, vp, i32, vp, vp, vp]
    L.cq_select_scales_spec.restype = i32
    L.cq_select_scales_spec.argtypes = [vp, i64, vp, i32, i64, ctypes.POINTER(QuantizerSpec), vp, vp, vp, vp, vp]
    L.cq_select_scales_noalloc.restype = i32
    L.cq_select_scales_noalloc.argtypes = [vp, i64, vp, i32, i64, vp, vp, vp]
    L.cq_trim_memory.restype = i32
    L.cq_trim_memory.argtypes = []
    L.cq_read_counters.restype = i32
    L.cq_read_counters.argtypes = [vp, vp, vp]
    L.cq_get_status.restype = i32
    L.cq_get_status.argtypes = [vp, vp]
    L.cq_status_string.restype = ctypes.c_char_p
    L.cq_status_string.argtypes = [i32]
    L.cq_version.restype = i32
    L.cq_version.argtypes = []
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.cq_status_string(int(status)).decode()


def version() -> int:
    return int(lib.cq_version())


def workspace_bytes(G: int, E: int) -> int:
    return int(lib.cq_workspace_bytes(int(G), int(E)))


def _check(status: int, where: str):
    if status != CQ_OK:
        raise CQError(status, where)


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(None)
    if isinstance(t, np.ndarray):
        return ctypes.c_void_p(t.ctypes.data)
    return ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class Result:
    scales: "object"          # torch.int16 [G]: binary16 bit patterns
    codes: "object"           # torch.int32 [G, 16]: packed nibble words (uint32 bits)
    objective: "object" = None  # torch.float64 [G]
    flags: "object" = None      # torch.uint8 [G]
    workspace: "object" = None  # torch.uint8: counters + fallback queue

    def counters(self, stream=None) -> dict:
        return read_counters(self.workspace, stream)


def _shapes(W, D, K):
    if W.dim() != 2 or W.shape[-1] % GROUP:
        raise ValueError("W must be 2-D with a multiple of 128 columns")
    G = W.numel() // GROUP
    if D.dim() == 2:
        E, Kd = D.shape
        if K is not None and K != Kd:
            raise ValueError("K does not match D")
        K = Kd
    elif D.dim() == 3:
        E = D.shape[0]
        if D.shape[1:] != (G, GROUP):
            raise ValueError("per-group D must be [E, G, 128]")
        K = 0
    else:
        raise ValueError("D must be [E, K] or [E, G, 128]")
    return G, E, K


def select_scales(W, D, K: int | None = None, *, stream=None, finalist_cap: int = 0,
                  force_exhaustive: bool = False, flag_rel_gap: float = 0.0,
                  out_scales=None, out_codes=None, want_objective: bool = False,
                  want_flags: bool = False, workspace=None, main_events=None,
                  intersections: bool = False) -> Result:
    """Exact minimax FP16 scales and packed W4 codes for every 128-weight group.

    W: CUDA tensor of binary16 bit patterns (int16/uint16/float16), [R, K] grouped
       along rows or [G, 128].  D: CUDA float32, per column [E, K] or per group
       [E, G, 128].  Runs asynchronously on ``stream`` (default: current).
       main_events: optional pair of torch.cuda.Event (enable_timing=True)
       recorded just before and after the main selection kernel.
       intersections: search surviving runs with the pairwise
       environment-intersection solver (same results)."""
    import torch
    if not (W.is_cuda and D.is_cuda):
        raise ValueError("W and D must be CUDA tensors")
    if W.element_size() != 2:
        raise ValueError("W must hold 16-bit binary16 patterns")
    if D.dtype != torch.float32:
        raise ValueError("D must be float32")
    if not (W.is_contiguous() and D.is_contiguous()):
        raise ValueError("W and D must be contiguous")
    G, E, K = _shapes(W, D, K)
    dev = W.device
    if out_scales is None:
        out_scales = torch.empty(G, dtype=torch.int16, device=dev)
    if out_codes is None:
        out_codes = torch.empty((G, WORDS), dtype=torch.int32, device=dev)
    obj = torch.empty(G, dtype=torch.float64, device=dev) if want_objective else None
    flags = torch.empty(G, dtype=torch.uint8, device=dev) if want_flags else None
    wsb = workspace_bytes(G, E)
    if workspace is None or workspace.numel() < wsb:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    ev0 = ev1 = None
    if main_events is not None:  # (torch.cuda.Event, torch.cuda.Event) around the main kernel
        for e in main_events:  # torch creates the event lazily, at its first record
            if not e.cuda_event:
                e.record(stream)
        ev0, ev1 = (ctypes.c_void_p(e.cuda_event) for e in main_events)
    opts = Opts(int(finalist_cap), int(bool(force_exhaustive)), float(flag_rel_gap), ev0, ev1,
                int(bool(intersections)))
    st = lib.cq_select_scales_ex(_ptr(W), G, _ptr(D), E, K, _ptr(out_scales), _ptr(out_codes),
                                 _stream_handle(stream), ctypes.byref(opts), _ptr(workspace), wsb,
                                 _ptr(obj), _ptr(flags))
    _check(st, "cq_select_scales_ex")
    return Result(out_scales, out_codes, obj, flags, workspace)


def select_scales_plain(W, D, K: int | None = None, *, stream=None, out_scales=None, out_codes=None):
    """The plain entry point (library-allocated workspace); returns (scales, codes)."""
    import torch
    G, E, K = _shapes(W, D, K)
    if out_scales is None:
        out_scales = torch.empty(G, dtype=torch.int16, device=W.device)
    if out_codes is None:
        out_codes = torch.empty((G, WORDS), dtype=torch.int32, device=W.device)
    st = lib.cq_select_scales(_ptr(W), G, _ptr(D), E, K, _ptr(out_scales), _ptr(out_codes),
                              _stream_handle(stream))
    _check(st, "cq_select_scales")
    return out_scales, out_codes


def select_scales_noalloc(W, D, K: int | None = None, *, stream=None, out_scales=None, out_codes=None):
    """The allocation-free entry point: the library allocates nothing (its
    scratch is a fixed array inside libcq.so, up to NOALLOC_MAX_GROUPS groups).
    The outputs are allocated here only when not passed in.  Calls that
    overlap on the GPU share that scratch and must be ordered on one stream."""
    import torch
    G, E, K = _shapes(W, D, K)
    if out_scales is None:
        out_scales = torch.empty(G, dtype=torch.int16, device=W.device)
    if out_codes is None:
        out_codes = torch.empty((G, WORDS), dtype=torch.int32, device=W.device)
    st = lib.cq_select_scales_noalloc(_ptr(W), G, _ptr(D), E, K, _ptr(out_scales), _ptr(out_codes),
                                      _stream_handle(stream))
    _check(st, "cq_select_scales_noalloc")
    return out_scales, out_codes


def select_scales_host(W, D, K: int | None = None, *, stream=None, out_scales=None, out_codes=None):
    """Host-buffer entry point: W, D and the outputs live in host memory (numpy
    arrays or CPU tensors; page-locked memory overlaps the copies).  Blocks
    until the results are on the host.  Returns (scales uint16 [G], codes uint32 [G, 16])."""
    W = W.numpy() if hasattr(W, "numpy") and not isinstance(W, np.ndarray) else W
    D = D.numpy() if hasattr(D, "numpy") and not isinstance(D, np.ndarray) else D
    if W.dtype.itemsize != 2 or W.ndim != 2 or W.shape[-1] % GROUP or not W.flags.c_contiguous:
        raise ValueError("W must be a contiguous 2-D array of 16-bit patterns")
    if D.dtype != np.float32 or not D.flags.c_contiguous:
        raise ValueError("D must be contiguous float32")
    G = W.size // GROUP
    if D.ndim == 2:
        E, K = D.shape
    else:
        E, K = D.shape[0], 0
    if out_scales is None:
        out_scales = np.empty(G, dtype=np.uint16)
    if out_codes is None:
        out_codes = np.empty((G, WORDS), dtype=np.uint32)
    st = lib.cq_select_scales_host(_ptr(W), G, _ptr(D), E, K, _ptr(out_scales), _ptr(out_codes),
                                   _stream_handle(stream))
    _check(st, "cq_select_scales_host")
    return out_scales, out_codes


def _check_w(W):
    if not W.is_cuda or W.element_size() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous CUDA tensor of 16-bit binary16 patterns")
    if W.dim() != 2 or W.shape[-1] % GROUP:
        raise ValueError("W must be 2-D with a multiple of 128 columns")


def absmax_scales(W, *, stream=None, out_scales=None, out_codes=None):
    """AbsMax policy: s = fp16(max|w| / 7) per group (at least the smallest
    positive pattern) and the codes at s.  Returns (scales int16 [G], codes int32 [G, 16])."""
    import torch
    _check_w(W)
    G = W.numel() // GROUP
    if out_scales is None:
        out_scales = torch.empty(G, dtype=torch.int16, device=W.device)
    if out_codes is None:
        out_codes = torch.empty((G, WORDS), dtype=torch.int32, device=W.device)
    _check(lib.cq_absmax_scales(_ptr(W), G, _ptr(out_scales), _ptr(out_codes), _stream_handle(stream)),
           "cq_absmax_scales")
    return out_scales, out_codes


def pool_diagonals(D, *, stream=None, out=None):
    """Mean of the environments' diagonals (fp64 sum in environment order,
    rounded once to fp32): [E, ...] -> [1, ...], the input of Pooled-WMSE."""
    import torch
    if not D.is_cuda or D.dtype != torch.float32 or not D.is_contiguous() or D.dim() < 2:
        raise ValueError("D must be a contiguous CUDA float32 tensor [E, ...]")
    E = D.shape[0]
    n = D.numel() // E
    if out is None:
        out = torch.empty((1,) + tuple(D.shape[1:]), dtype=torch.float32, device=D.device)
    _check(lib.cq_pool_diagonals(_ptr(D), E, n, _ptr(out), _stream_handle(stream)), "cq_pool_diagonals")
    return out


def select_scales_pooled(W, D, K: int | None = None, **kw) -> Result:
    """Pooled-WMSE policy: the exact search with one environment whose
    diagonal is the mean of D's environments."""
    return select_scales(W, pool_diagonals(D, stream=kw.get("stream")), K, **kw)


def group_objective(W, D, scales, K: int | None = None, *, stream=None, per_env=None, out=None):
    """Objective of given scales: (max_e objective float64 [G], per-environment
    objectives float64 [G, E]), each an fp64 sum over the group in index order."""
    import torch
    _check_w(W)
    if not D.is_cuda or D.dtype != torch.float32 or not D.is_contiguous():
        raise ValueError("D must be a contiguous CUDA float32 tensor")
    G, E, K = _shapes(W, D, K)
    if scales.numel() != G or scales.element_size() != 2 or not scales.is_contiguous():
        raise ValueError("scales must hold G 16-bit patterns")
    if per_env is None:
        per_env = torch.empty((G, E), dtype=torch.float64, device=W.device)
    if out is None:
        out = torch.empty(G, dtype=torch.float64, device=W.device)
    _check(lib.cq_group_objective(_ptr(W), G, _ptr(D), E, K, _ptr(scales), _ptr(per_env), _ptr(out),
                                  _stream_handle(stream)), "cq_group_objective")
    return out, per_env


def reconstruction_proxy(per_env, offsets, scale: float = 1.0 / GROUP, *, stream=None):
    """Module-macro worst-environment weighted MSE from per-environment group
    objectives [G, E] and module offsets (int64, nmod + 1).  Returns
    (module_env float64 [nmod, E], module_worst [nmod], macro [1]) on the device."""
    import torch
    if per_env.dtype != torch.float64 or per_env.dim() != 2 or not per_env.is_contiguous():
        raise ValueError("per_env must be a contiguous float64 [G, E] tensor")
    G, E = per_env.shape
    off = np.asarray(offsets.cpu() if hasattr(offsets, "cpu") else offsets, dtype=np.int64).ravel()
    if off.size < 1 or off[0] < 0 or off[-1] > G or np.any(np.diff(off) < 0):
        raise ValueError("offsets must ascend from >= 0 to <= the number of groups")
    offsets = torch.from_numpy(off).to(per_env.device)
    nmod = off.size - 1
    dev = per_env.device
    module_env = torch.empty((max(nmod, 0), E), dtype=torch.float64, device=dev)
    module_worst = torch.empty(max(nmod, 0), dtype=torch.float64, device=dev)
    macro = torch.full((1,), float("nan"), dtype=torch.float64, device=dev)
    _check(lib.cq_reconstruction_proxy(_ptr(per_env), G, E, nmod, _ptr(offsets), float(scale), _ptr(module_env),
                                       _ptr(module_worst), _ptr(macro), _stream_handle(stream)),
           "cq_reconstruction_proxy")
    return module_env, module_worst, macro


POLICIES = ("cliffquant", "pooled_wmse", "absmax")


def policy_scales(policy: str, W, D, K: int | None = None, *, stream=None):
    """(scales, codes) of one of POLICIES on the device."""
    if policy == "cliffquant":
        r = select_scales(W, D, K, stream=stream)
        return r.scales, r.codes
    if policy == "pooled_wmse":
        r = select_scales_pooled(W, D, K, stream=stream)
        return r.scales, r.codes
    if policy == "absmax":
        return absmax_scales(W, stream=stream)
    raise ValueError(f"unknown policy {policy!r}; expected one of {POLICIES}")


def evaluate_policies(W, D, offsets, K: int | None = None, *, policies=POLICIES, stream=None) -> dict:
    """The reconstruction proxy for each policy: {policy: (macro, module_worst
    numpy [nmod], scales)}; every step on the device, one host read per policy."""
    out = {}
    for pol in policies:
        scales, _ = policy_scales(pol, W, D, K, stream=stream)
        _, per_env = group_objective(W, D, scales, K, stream=stream)
        _, worst, macro = reconstruction_proxy(per_env, offsets, stream=stream)
        if stream is not None:
            stream.synchronize()
        out[pol] = (float(macro.cpu()[0]), worst.cpu().numpy(), scales)
    return out


@dataclass
class GPTQTensors:
    """GPTQ v1 tensors of one linear layer with weight [R, K] (R outputs, K inputs)."""
    qweight: "object"  # torch.int32 [K/8, R]
    qzeros: "object"   # torch.int32 [K/128, R/8]
    scales: "object"   # torch.float16 [K/128, R]
    g_idx: "object"    # torch.int32 [K]

    def as_dict(self) -> dict:
        return {"qweight": self.qweight, "qzeros": self.qzeros, "scales": self.scales, "g_idx": self.g_idx}


def gptq_export(scales, codes, R: int, K: int, *, stream=None) -> GPTQTensors:
    """GPTQ v1 tensors from the selection's scales [R*K/128] and codes [R*K/128, 16]
    (groups along the rows of an [R, K] weight)."""
    import torch
    G = R * K // GROUP
    if scales.numel() != G or codes.numel() != G * WORDS or not (scales.is_contiguous() and codes.is_contiguous()):
        raise ValueError("scales and codes must hold R*K/128 contiguous groups")
    dev = codes.device
    t = GPTQTensors(torch.empty((K // 8, R), dtype=torch.int32, device=dev),
                    torch.empty((K // GROUP, R // 8), dtype=torch.int32, device=dev),
                    torch.empty((K // GROUP, R), dtype=torch.float16, device=dev),
                    torch.empty(K, dtype=torch.int32, device=dev))
    _check(lib.cq_gptq_export(_ptr(scales), _ptr(codes), R, K, _ptr(t.qweight), _ptr(t.qzeros), _ptr(t.scales),
                              _ptr(t.g_idx), _stream_handle(stream)), "cq_gptq_export")
    return t


def gptq_dequantize(t: GPTQTensors, *, half: bool = False, stream=None):
    """[R, K] weights by the v1 rule: float32 (exact) or float16 (rounded to nearest even)."""
    import torch
    K = t.qweight.shape[0] * 8
    R = t.qweight.shape[1]
    out = torch.empty((R, K), dtype=torch.float16 if half else torch.float32, device=t.qweight.device)
    _check(lib.cq_gptq_dequantize(_ptr(t.qweight), _ptr(t.qzeros), _ptr(t.scales), _ptr(t.g_idx), R, K,
                                  int(bool(half)), _ptr(out), _stream_handle(stream)), "cq_gptq_dequantize")
    return out


def select_scales_spec(W, D, K: int | None = None, *, qmin: int = -8, qmax: int = 7, group_size: int = 128,
                       stream=None, want_objective: bool = False, want_flags: bool = False,
                       general_kernel: bool = False) -> Result:
    """Exact minimax scales for a general spec (codes in [qmin, qmax], groups of
    group_size weights).  W: CUDA 16-bit binary16 patterns whose last dimension
    is a multiple of group_size; D: float32 per column [E, K] or per group
    [E, G, group_size].  Returns scales int16 [G] and codes int8 [G, group_size]
    (the q values).  qmin = -qmax or -qmax - 1 with |qmin| <= 16 at group size
    128, or <= 8 at 64, runs the W4 kernel's search; general_kernel=True forces
    the general one."""
    import torch
    n = int(group_size)
    if not (W.is_cuda and D.is_cuda and W.is_contiguous() and D.is_contiguous()):
        raise ValueError("W and D must be contiguous CUDA tensors")
    if W.element_size() != 2 or D.dtype != torch.float32:
        raise ValueError("W must hold binary16 patterns and D float32")
    if n < 1 or W.shape[-1] % n:
        raise ValueError("the last dimension of W must be a multiple of group_size")
    G = W.numel() // n
    if D.dim() == 2:
        E, Kd = D.shape
        if K is not None and K != Kd:
            raise ValueError("K does not match D")
        K = Kd
    elif D.dim() == 3 and D.shape[1:] == (G, n):
        E, K = D.shape[0], 0
    else:
        raise ValueError("D must be [E, K] or [E, G, group_size]")
    dev = W.device
    scales = torch.empty(G, dtype=torch.int16, device=dev)
    codes = torch.empty((G, n), dtype=torch.int8, device=dev)
    obj = torch.empty(G, dtype=torch.float64, device=dev) if want_objective else None
    flags = torch.empty(G, dtype=torch.uint8, device=dev) if want_flags else None
    spec = QuantizerSpec(int(qmin), int(qmax), n, 1 if general_kernel else 0)
    _check(lib.cq_select_scales_spec(_ptr(W), G, _ptr(D), E, K, ctypes.byref(spec), _ptr(scales), _ptr(codes),
                                     _ptr(obj), _ptr(flags), _stream_handle(stream)), "cq_select_scales_spec")
    return Result(scales, codes, obj, flags)


DTYPE_BF16, DTYPE_FP16, DTYPE_FP32 = 0, 1, 2


def estimate_diagonals(X, row_offsets, *, dtype=None, stream=None, means=None, out=None):
    """Per-environment diagonals from calibration inputs X [rows, K] (CUDA
    bfloat16, float16 or float32; environment e owns rows row_offsets[e] ..
    row_offsets[e+1]-1).  Returns (means float64 [E, K], D float32 [E, K]);
    D is the per-column diagonal input of select_scales."""
    import torch
    if not X.is_cuda or X.dim() != 2 or not X.is_contiguous():
        raise ValueError("X must be a contiguous 2-D CUDA tensor")
    if dtype is None:
        dtype = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_FP16, torch.float32: DTYPE_FP32}.get(X.dtype)
        if dtype is None:
            raise ValueError("X must be bfloat16, float16 or float32 (or pass dtype for 16-bit patterns)")
    off = np.ascontiguousarray(np.asarray(row_offsets, dtype=np.int64).ravel())
    E, K = off.size - 1, X.shape[1]
    if E < 1 or off[-1] > X.shape[0]:
        raise ValueError("row_offsets must hold E + 1 offsets within X's rows")
    if means is None:
        means = torch.empty((E, K), dtype=torch.float64, device=X.device)
    if out is None:
        out = torch.empty((E, K), dtype=torch.float32, device=X.device)
    _check(lib.cq_estimate_diagonals(_ptr(X), int(dtype), K, _ptr(off), E, _ptr(means), _ptr(out),
                                     _stream_handle(stream)), "cq_estimate_diagonals")
    return means, out


def read_counters(workspace, stream=None) -> dict:
    """Synchronises ``stream`` and returns the counters of the last call."""
    host = np.zeros(CQ_NUM_COUNTERS, dtype=np.uint32)
    st = lib.cq_read_counters(_ptr(workspace), _ptr(host), _stream_handle(stream))
    if st not in (CQ_OK, CQ_ERR_NONFINITE):
        raise CQError(st, "cq_read_counters")
    return {n: int(v) for n, v in zip(COUNTER_NAMES, host)}


def trim_memory() -> None:
    """Return the device memory that select_scales_plain and the host-buffer
    path keep cached in the library's pool on the current device."""
    st = lib.cq_trim_memory()
    if st != CQ_OK:
        raise CQError(st, "cq_trim_memory")


def get_status(workspace, stream=None) -> int:
    """Synchronises ``stream``; CQ_OK, or CQ_ERR_NONFINITE when the last call
    on ``workspace`` saw non-finite or negative input."""
    st = lib.cq_get_status(_ptr(workspace), _stream_handle(stream))
    if st not in (CQ_OK, CQ_ERR_NONFINITE):
        raise CQError(st, "cq_get_status")
    return st


def to_numpy_bits(res: Result):
    """(scales uint16 [G], codes uint32 [G, 16]) on the host."""
    s = res.scales.cpu().numpy().view(np.uint16)
    c = res.codes.cpu().numpy().view(np.uint32)
    return s, c
