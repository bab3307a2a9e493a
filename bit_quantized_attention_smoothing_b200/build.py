"""Builds the CUDA library ``libqattn.so`` in-tree for B200 (sm_100a) with nvcc.

No fast-math: the quantization kernels rely on correctly rounded binary32 division, reciprocal and
conversions, and on subnormals being kept, to stay bit-exact.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqattn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def nvcc_cmd(out: str, verbose: bool = False):
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC, "-o", out,
           os.path.join(CSRC, "qattn.cu"), "-lcudart"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if force or stale():
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(nvcc_cmd(tmp, verbose))
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
