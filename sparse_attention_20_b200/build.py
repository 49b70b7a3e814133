"""Build libdsa.so (the C-ABI library of the DSA hot path) in-tree for sm_100a.

    python -m sparse_attention_20_b200.build [--force]

One translation unit (csrc/dsa.cu) compiled by nvcc for
``-gencode arch=compute_100a,code=sm_100a``; the public header is
include/dsa.h at the repository root.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdsa.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-O2",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


# The debug build: the same source with the device-side index-set checks
# (csrc/debug_checks.cuh) compiled in.
DEBUG_LIB = os.path.join(PKG, "libdsa_debug.so")


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    """Compile libdsa.so (or, with debug=True, libdsa_debug.so with -DDSA_DEBUG)
    when a source is newer than it; returns its path."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DDSA_DEBUG"] if debug else []), *extra_flags, "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "dsa.cu"), "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force=force or bool(extra), verbose=True, extra_flags=extra, debug="--debug" in sys.argv))
