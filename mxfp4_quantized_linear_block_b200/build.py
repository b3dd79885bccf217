"""Build libmxfp4.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmxfp4.so")
SOURCES = ["csrc/abi.cu", "csrc/quantize.cu", "csrc/quantize_wide.cu", "csrc/quantize_norm.cu",
           "csrc/gemm.cu", "csrc/gemm_smallm.cu", "csrc/noalloc.cu"]
DEPS = SOURCES + ["csrc/internal.h", "csrc/sm100.cuh", "csrc/block_quant.cuh",
                  "../include/mxfp4.h"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
    "-I" + os.path.join(ROOT, "include"),
]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(os.path.join(HERE, d)) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or needs_build():
        cmd = [NVCC, *FLAGS, *[os.path.join(HERE, s) for s in SOURCES], "-o", LIB]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd, cwd=HERE)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
