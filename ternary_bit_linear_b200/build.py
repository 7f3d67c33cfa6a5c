"""Build libtq.so (the CUDA kernels + C ABI) in-tree for sm_100a.

    python -m ternary_bit_linear_b200.build [--verbose]

nvcc cross-compiles without a GPU.  No fast-math: the quantisers rely on
IEEE round-to-nearest-even fp32 multiplies and divides.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtq.so")
SOURCES = ["tq_api.cu"]
DEPS = ["tq_api.cu", "tq_common.cuh", "tq_pack.cuh", "tq_act.cuh", "tq_gemv.cuh", "tq_gemv_group.cuh", "tq_gemm.cuh",
        "tq_train.cuh", "tq_xorshift_jump.h"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(INCLUDE, "tq.h")]
    return any(os.path.getmtime(s) > t for s in srcs)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [
        nvcc(), "-O3", "-std=c++17", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
        "-I", INCLUDE, "-I", CSRC,
        "-o", tmp,
    ] + [os.path.join(CSRC, s) for s in SOURCES] + ["-lcudart"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
