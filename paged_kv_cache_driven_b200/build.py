"""Builds libpagedattn.so (sm_100a kernels + host allocator) into this package.

The kernels are split over several translation units (csrc/pa_k_*.cu) that
compile in parallel into ``_build/``; a unit is recompiled when it or any
header is newer than its object, then everything is linked into one library.

With --trace it also builds libpagedattn_trace.so: the same library with the
prefill unit compiled with PA_PREFILL_TRACE, which adds clock stamps at the
prefill kernel's hand-offs and exports pa_prefill_trace_read / _clear (for
bench.py --workload prefill_trace; the library proper has none of it).

Usage: python -m paged_kv_cache_driven_b200.build [--verbose] [--force] [--trace]
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
TRACE_LIB = os.path.join(PKG, "libpagedattn_trace.so")
TRACE_SRC = os.path.join(CSRC, "pa_k_prefill.cu")
TRACE_OBJ = os.path.join(OBJ, "pa_k_prefill.trace.o")
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


def build_trace(force=False, verbose=False):
    """libpagedattn_trace.so: the objects of build(), with the prefill unit
    compiled with PA_PREFILL_TRACE instead."""
    build(force=force, verbose=verbose)
    fresh = os.path.exists(TRACE_OBJ) and all(
        os.path.getmtime(f) <= os.path.getmtime(TRACE_OBJ) for f in [TRACE_SRC, *HEADERS])
    if force or not fresh:
        cmd = [NVCC, *FLAGS, "-DPA_PREFILL_TRACE", "-c", TRACE_SRC, "-o", TRACE_OBJ]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise subprocess.CalledProcessError(r.returncode, "nvcc")
    objs = [TRACE_OBJ if s == TRACE_SRC else _obj(s) for s in SOURCES]
    subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs,
                    "-o", TRACE_LIB], check=True)
    return TRACE_LIB


if __name__ == "__main__":
    if "--trace" in sys.argv:
        build_trace(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    else:
        build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
