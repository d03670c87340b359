"""Build libcq.so in-tree for sm_100a (nvcc; cross-compiles without a GPU).

    python -m minimax_scale_search_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRCS = [os.path.join(PKG, "csrc", name) for name in ("cq_select.cu", "cq_policies.cu", "cq_gptq.cu", "cq_diag.cu",
                                                           "cq_spec.cu")]
DEPS = SRCS + [os.path.join(PKG, "csrc", "cq_device.cuh"), os.path.join(ROOT, "include", "cq.h")]
LIB = os.path.join(PKG, "libcq.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def build(force: bool = False, ptxas_verbose: bool = False, out: str = LIB) -> str:
    if not force and os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in DEPS):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", os.path.join(ROOT, "include"), "-o", tmp, *SRCS]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas))
    sys.exit(0)
