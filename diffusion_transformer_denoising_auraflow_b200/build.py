"""Build the sm_100a shared library ``libaf.so`` in-tree with nvcc.

Usage: ``python diffusion_transformer_denoising_auraflow_b200/build.py``
(also called by ``__graft_entry__.build()``).  No GPU is needed: nvcc
cross-compiles for sm_100a.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libaf.so")
SOURCES = ["api.cu", "gemm.cu", "attention.cu", "kernels.cu", "init.cu", "fp32.cu", "exchange.cu", "noalloc.cu"]
HEADERS = ["af_internal.h", "ptx.cuh"]


def nvcc_cmd(out=LIB, extra=()):
    nvcc = os.environ.get("NVCC", "nvcc")
    return [nvcc, "-shared", "-Xcompiler", "-fPIC", "-std=c++17", "-O3", "-lineinfo",
            "-gencode", "arch=compute_100a,code=sm_100a",
            "-I", os.path.join(ROOT, "include"), "-I", CSRC,
            *extra, "-o", out] + [os.path.join(CSRC, s) for s in SOURCES]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "af.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = True) -> str:
    if force or needs_build():
        cmd = nvcc_cmd()
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv)
