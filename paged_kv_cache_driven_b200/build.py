"""Builds libpagedattn.so (sm_100a kernels + host allocator) into this package.

Usage: python -m paged_kv_cache_driven_b200.build [--verbose]
"""

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libpagedattn.so")
SOURCES = [os.path.join(CSRC, f) for f in ("pa_api.cu", "pa_alloc.cpp", "pa_stepper.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("pa_device.cuh", "pa_decode.cuh", "pa_append.cuh",
                                                      "pa_gqa.cuh", "pa_prefill.cuh",
                                                      "pa_tcgen05.cuh")] \
    + [os.path.join(ROOT, "include", "pagedattn.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def command(verbose=False):
    cmd = [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC,-O2", "-shared", "-I", os.path.join(ROOT, "include"),
           *SOURCES, "-o", LIB]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPS)


def build(force=False, verbose=False):
    if force or stale():
        subprocess.run(command(verbose), check=True)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
