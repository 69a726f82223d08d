"""Build liblattice.so in-tree with nvcc for sm_100a (B200).

Usage: python -m orthogonal_update_recurrent_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liblattice.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# Each translation unit is compiled whole (no split compilation: nvcc's split mode
# gave different register allocations, and spills, from one build to the next) and
# the units are compiled in parallel.
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-Xptxas", "-warn-spills"]
LINK_FLAGS = [*ARCH, "-shared", "-cudart", "static"]
# the C ABI and one unit per kernel family (csrc/launch.h joins them)
UNITS = ["lattice_abi.cu", "tu_simt_exact.cu", "tu_simt_chunked.cu", "tu_step.cu", "tu_bwd.cu", "tu_tc.cu"]
OBJDIR = os.path.join(HERE, "_build")


def _nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    p = os.path.join(cuda, "bin", "nvcc")
    return p if os.path.exists(p) else "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not stale():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    tag = f"{os.getpid()}"
    jobs = []
    for unit in UNITS:
        obj = os.path.join(OBJDIR, unit[:-3] + f".{tag}.o")
        cmd = [_nvcc(), *COMPILE_FLAGS, *extra, "-I", INCLUDE, "-c", "-o", obj, os.path.join(CSRC, unit)]
        if verbose:
            print(" ".join(cmd), flush=True)
        jobs.append((subprocess.Popen(cmd), obj, cmd))
    failed = [cmd for p, _, cmd in jobs if p.wait() != 0]
    objs = [obj for _, obj, _ in jobs]
    try:
        if failed:
            raise subprocess.CalledProcessError(1, failed[0])
        tmp = LIB + f".tmp{tag}"
        cmd = [_nvcc(), *LINK_FLAGS, "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    finally:
        for obj in objs:
            if os.path.exists(obj):
                os.remove(obj)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
