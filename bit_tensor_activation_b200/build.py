"""Compiles libhq.so (all CUDA kernels + the C ABI) in-tree for sm_100a."""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SO = os.path.join(PKG, "libhq.so")
SOURCES = [os.path.join(PKG, "csrc", "hq_api.cu")]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-fmad=false",           # every float op stays one IEEE operation (bit-exact with the spec)
    "-Xcompiler", "-fPIC", "-shared",
]


def build(verbose: bool = False, extra_flags=()) -> str:
    cmd = ["nvcc", *NVCC_FLAGS, *extra_flags, "-I", os.path.join(ROOT, "include"), *SOURCES, "-o", SO]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return SO


if __name__ == "__main__":
    build(verbose=True)
