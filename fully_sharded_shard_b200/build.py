"""Build libfsdpk.so in-tree with nvcc for sm_100a (B200).

Usage: ``python -m fully_sharded_shard_b200.build [--force] [--verbose] [--debug]``.
The library links the CUDA runtime statically, so it does not depend on the
runtime version torch ships with.  ``--debug`` builds libfsdpk_debug.so, the
same sources with -DFSDPK_DEBUG (every table-driven kernel checks its work
units against the extents of its buffers); ``FSDPK_DEBUG=1`` makes the
binding load it.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfsdpk.so")
LIB_DEBUG = os.path.join(PKG, "libfsdpk_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
          "--expt-relaxed-constexpr", "-DFSDPK_BUILDING_LIBRARY"]
LDFLAGS = ["-shared", "-Xcompiler", "-fPIC"]
OBJDIR = os.path.join(PKG, "_build")
OBJDIR_DEBUG = os.path.join(PKG, "_build_debug")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")) + \
        [os.path.abspath(__file__)]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: cannot build libfsdpk.so")


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every kernel file to an object in parallel (one nvcc per file),
    then link the shared library (the debug library with debug=True)."""
    lib = LIB_DEBUG if debug else LIB
    objdir = OBJDIR_DEBUG if debug else OBJDIR
    if (not force and os.path.exists(lib)
            and os.path.getmtime(lib) >= max(os.path.getmtime(p) for p in _inputs())):
        return lib
    os.makedirs(objdir, exist_ok=True)
    extra = (["-Xptxas=-v"] if verbose else []) + (["-DFSDPK_DEBUG"] if debug else [])

    def compile_one(src: str) -> str:
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc(), *ARCH, *CFLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
        return obj

    srcs = sources()
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + ".tmp"
    subprocess.run([nvcc(), *ARCH, *LDFLAGS, "-o", tmp, *objs], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                debug="--debug" in sys.argv))
