"""Build step for libfa.so: one nvcc invocation for sm_100a, output in-tree.

``build_library(debug=True)`` builds ``libfa_debug.so`` with ``-DFA_DEBUG``: the
same kernels with device-side argument checks on every TMA copy, tensor-memory
access and MMA (a failed check is reported as FA_ERR_CHECK by fa_check_status);
the Python binding loads it when the environment sets FA_DEBUG=1."""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfa.so")
LIB_DEBUG = os.path.join(PKG, "libfa_debug.so")
SOURCES = ["api.cu", "sm100.cuh", "fwd.cuh", "bwd.cuh", "fp8.cuh", "decode.cuh", "fwd256.cuh", "bwd256.cuh"]
HEADER = os.path.join(os.path.dirname(PKG), "include", "fa.h")


def nvcc_command(out: str = LIB, extra=()):
    return [
        "nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
        "-Xcompiler", "-fPIC", "-shared", "--cudart", "static", *extra,
        os.path.join(CSRC, "api.cu"), "-o", out,
    ]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + [HEADER]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build_library(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    out = LIB_DEBUG if debug else LIB
    if force or needs_build(out):
        extra = (("-Xptxas", "-v") if verbose else ()) + (("-DFA_DEBUG",) if debug else ())
        subprocess.run(nvcc_command(out=out, extra=extra), check=True)
    return out


if __name__ == "__main__":
    import sys
    dbg = "--debug" in sys.argv
    print(build_library(force=True, verbose=True, debug=dbg))
