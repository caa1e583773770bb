"""Build the sm_100a shared library libfp8_paged_decode.so in-tree with nvcc.

The library exports the C ABI of include/fp8_paged_decode.h.  Usage:
    python -m fp8_paged_decode_b200.build          (or build() from Python)
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libfp8_paged_decode.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
SOURCES = ["fpd_api.cu"]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(home, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES]


def deps():
    return sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
        os.path.join(INCLUDE, "fp8_paged_decode.h")]


def needs_build(out: str = LIB_PATH) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps())


def build(out: str = LIB_PATH, verbose_ptxas: bool = False, extra=()) -> str:
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
           "-shared", "-I", INCLUDE, "-I", CSRC, "-o", out, *sources(), *extra]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    build(verbose_ptxas="-v" in sys.argv)
    print("built", LIB_PATH)
