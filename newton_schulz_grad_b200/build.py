"""Build the sm_100a shared library ``libdmuon_b200.so`` in place.

Each CUDA/C++ source under ``csrc/`` is compiled by nvcc for
``arch=compute_100a,code=sm_100a`` (no other architecture) with line info,
then linked into one shared library next to this file (the CUDA runtime is
linked statically, so the library only needs the driver at run time).  Only
symbols declared ``DMUON_API`` in ``include/dmuon.h`` are exported.

Usage: ``python newton_schulz_grad_b200/build.py [--force] [--verbose] [--debug]`` (run by
path: importing the package loads the library this script produces).  ``--debug`` builds
``libdmuon_b200_debug.so`` instead, with ``-DDMUON_DEBUG``: every global access of the
kernels is checked against its buffer's extent and skipped, with DMUON_ERR_BOUNDS in the
status word, when it falls outside (load it with DMUON_LIBRARY=<path>).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from typing import List

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_NAME = "libdmuon_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
DEBUG_LIB_PATH = os.path.join(HERE, "libdmuon_b200_debug.so")

SOURCES = ["api.cu", "plan.cpp", "elementwise.cu", "simt_gemm.cu", "tc_gemm.cu", "noalloc.cu", "small_ns.cu", "clip.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
          "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps() -> List[str]:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "dmuon.h"))
    return files


def _newest(paths) -> float:
    return max(os.path.getmtime(p) for p in paths if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, extra: List[str] = None, debug: bool = False) -> str:
    """Compile and link if any source is newer than the library; return its path."""
    user_extra = list(extra or [])
    lib = DEBUG_LIB_PATH if debug else LIB_PATH
    build_dir = os.path.join(BUILD_DIR, "debug") if debug else BUILD_DIR
    if (not force and not user_extra and os.path.exists(lib)
            and os.path.getmtime(lib) >= _newest(_deps())):
        return lib
    extra = user_extra + (["-DDMUON_DEBUG"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()
    objs = []
    for src in SOURCES:
        obj = os.path.join(build_dir, src + ".o")
        cmd = [cc] + ARCH + COMMON + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
        if src.endswith(".cpp"):
            cmd = ["g++", "-O3", "-std=c++17", "-fPIC", "-fvisibility=hidden", "-I", INCLUDE,
                   "-I", CSRC, "-I", os.path.join(os.path.dirname(os.path.dirname(cc)), "include"),
                   "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + ".tmp"
    cmd = [cc] + ARCH + ["-shared", "-Xcompiler", "-fvisibility=hidden", "-o", tmp] + objs
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    force = "--force" in sys.argv
    verbose = "--verbose" in sys.argv
    debug = "--debug" in sys.argv
    extra = [a for a in sys.argv[1:] if a not in ("--force", "--verbose", "--debug")]
    print(build(force=force, verbose=verbose, extra=extra, debug=debug))
