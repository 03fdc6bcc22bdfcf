"""Build libgdn.so (all CUDA sources under csrc/) in-tree for sm_100a with nvcc.

Usage: python -m gated_deltanet_sequence_b200.build [--force] [--verbose-ptxas] [--debug-bounds]

--debug-bounds builds libgdn_debug.so instead: the same sources with -DGDN_DEBUG_BOUNDS, whose
kernels check the index of each thread-side global access of inputs, outputs and states against
the extent the launch implies and report GDN_ERR_BOUNDS (through gdn_sync_status) instead of
making it.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libgdn.so")
LIB_DEBUG = os.path.join(HERE, "libgdn_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
              "--expt-relaxed-constexpr", "-Xptxas", "-O3"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int = 0, debug_bounds: bool = False) -> str:
    """Compile every csrc/*.cu to an object, then link libgdn.so (libgdn_debug.so with
    debug_bounds). Returns its path."""
    LIB = LIB_DEBUG if debug_bounds else globals()["LIB"]
    if not force and not is_stale(LIB):
        return LIB
    objdir = os.path.join(HERE, "_build_debug" if debug_bounds else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs, procs = [], []
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DGDN_DEBUG_BOUNDS"] if debug_bounds else [])
    for src in _sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        cmd = [NVCC, *ARCH_FLAGS, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-c", src, "-o", obj]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = False
    for cmd, p in procs:
        out, _ = p.communicate()
        if out:
            sys.stdout.write(out.decode(errors="replace"))
        if p.returncode != 0:
            failed = True
            sys.stderr.write("FAILED: " + " ".join(cmd) + "\n")
    if failed:
        raise RuntimeError(f"nvcc failed building {os.path.basename(LIB)}")
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH_FLAGS, "-shared", "-o", tmp, *objs, "-lcudart"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv,
                debug_bounds="--debug-bounds" in sys.argv))
