"""Builds libdsa.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

Usage: python -m indexed_sparse_attention_relu_b200.build [--force] [--verbose] [--debug]
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
LIB = os.path.join(PKG, "libdsa.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-O2",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(ROOT, "include", "dsa.h")])


DEBUG_LIB = os.path.join(PKG, "libdsa_debug.so")


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile csrc/dsa.cu into libdsa.so unless it is up to date.

    debug=True builds libdsa_debug.so with DSA_DEBUG defined: every gathered
    row index is checked on the host before the attention runs (the calls
    then synchronise), and the tensor-core kernels guard the end of their
    shared memory with a canary that reports DSA_ERR_DEVICE_LAYOUT."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DDSA_DEBUG"] if debug else []), "-I", os.path.join(ROOT, "include"),
           os.path.join(CSRC, "dsa.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true", help="build libdsa_debug.so (DSA_DEBUG)")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))
