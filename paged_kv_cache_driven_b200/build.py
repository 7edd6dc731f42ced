"""Builds libpagedattn.so (sm_100a kernels + host allocator) into this package.

The kernels are split over several translation units (csrc/pa_k_*.cu) that
compile in parallel into ``_build/``; a unit is recompiled when it or any
header is newer than its object, then everything is linked into one library.

Usage: python -m paged_kv_cache_driven_b200.build [--verbose] [--force]
"""

import concurrent.futures
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libpagedattn.so")
SOURCES = sorted(glob.glob(os.path.join(CSRC, "*.cu"))) + \
    [os.path.join(CSRC, f) for f in ("pa_alloc.cpp", "pa_stepper.cpp")]
HEADERS = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
    [os.path.join(ROOT, "include", "pagedattn.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC,-O2", "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def _obj(src):
    return os.path.join(OBJ, os.path.basename(src) + ".o")


def compile_command(src, verbose=False):
    cmd = [NVCC, *FLAGS, "-c", src, "-o", _obj(src)]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def link_command():
    return [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
            *[_obj(s) for s in SOURCES], "-o", LIB]


def _stale_obj(src):
    o = _obj(src)
    if not os.path.exists(o):
        return True
    t = os.path.getmtime(o)
    return any(os.path.getmtime(f) > t for f in [src, *HEADERS])


def stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(_stale_obj(s) or os.path.getmtime(_obj(s)) > t for s in SOURCES)


def build(force=False, verbose=False):
    os.makedirs(OBJ, exist_ok=True)
    todo = [s for s in SOURCES if force or _stale_obj(s)]
    if todo:
        workers = max(1, min(len(todo), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            runs = list(ex.map(lambda s: subprocess.run(compile_command(s, verbose),
                                                        capture_output=True, text=True), todo))
        failed = False
        for src, r in zip(todo, runs):
            if verbose or r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
            failed |= r.returncode != 0
        if failed:
            raise subprocess.CalledProcessError(1, "nvcc")
    if todo or force or stale():
        subprocess.run(link_command(), check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
