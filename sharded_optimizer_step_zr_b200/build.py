"""Build libzr.so in-tree: the sm_100a kernels and the C ABI (nvcc, no torch).

    python sharded_optimizer_step_zr_b200/build.py [--verbose-ptxas]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libzr.so")
SOURCES = ["zr_kernels.cu", "zr_scalars.cu", "zr_check.cu", "zr_gather.cu", "zr_no_alloc.cu",
           "planner.cpp", "api.cpp", "checkpoint.cpp", "peer.cpp"]
HEADERS = ["zr_internal.hpp", os.path.join(ROOT, "include", "zr.h"), "exports.map"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + \
        [h if os.path.isabs(h) else os.path.join(CSRC, h) for h in HEADERS] + [__file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not _stale() and not verbose_ptxas:
        return LIB
    cmd = [NVCC, "-std=c++17", "-O3", "-lineinfo", *ARCH,
           "-Xcompiler", "-fPIC", "-shared",
           "-I", os.path.join(ROOT, "include"),
           "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"),
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", LIB + ".tmp"]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
