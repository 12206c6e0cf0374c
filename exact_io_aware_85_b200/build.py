"""Build step for libfa.so: one nvcc invocation for sm_100a, output in-tree."""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfa.so")
SOURCES = ["api.cu", "sm100.cuh", "fwd.cuh", "bwd.cuh", "fp8.cuh", "decode.cuh", "fwd256.cuh"]
HEADER = os.path.join(os.path.dirname(PKG), "include", "fa.h")


def nvcc_command(out: str = LIB, extra=()):
    return [
        "nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
        "-Xcompiler", "-fPIC", "-shared", "--cudart", "static", *extra,
        os.path.join(CSRC, "api.cu"), "-o", out,
    ]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + [HEADER]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build_library(force: bool = False, verbose: bool = False) -> str:
    if force or needs_build():
        extra = ("-Xptxas", "-v") if verbose else ()
        subprocess.run(nvcc_command(extra=extra), check=True)
    return LIB


if __name__ == "__main__":
    build_library(force=True, verbose=True)
    print(LIB)
