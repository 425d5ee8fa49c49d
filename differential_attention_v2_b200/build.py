"""Build the CUDA library libdiffattn_v2.so in place (sm_100a).

    python -m differential_attention_v2_b200.build [--force] [--verbose] [--debug-bounds]

Compiles every kernel and the C ABI with nvcc for sm_100a into one shared library that
sits next to this file, where the Python binding loads it. nvcc cross-compiles, so this
runs on machines without a GPU. Rebuilds only when a source is newer than the library.

--debug-bounds also builds libdiffattn_v2_debug.so: the same library compiled with
-DDA2_DEBUG_BOUNDS, in which the kernels check their shared-memory, tensor-memory and global
indices against the extents they address and report a violation through the device error
word (code 4) instead of making the access. The tests load it directly.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_NAME = "libdiffattn_v2.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
DEBUG_LIB_PATH = os.path.join(PKG, "libdiffattn_v2_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + [
        os.path.join(ROOT, "include", "diffattn_v2.h"), os.path.abspath(__file__)]


def up_to_date(path=LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libdiffattn_v2.so")
    return exe


def build(force: bool = False, verbose: bool = False, extra_flags=None, debug_bounds: bool = False) -> str:
    """Build the library (or, with debug_bounds, its bounds-checking twin); returns its path."""
    out = DEBUG_LIB_PATH if debug_bounds else LIB_PATH
    if debug_bounds:
        extra_flags = list(extra_flags or []) + ["-DDA2_DEBUG_BOUNDS"]
    if not force and up_to_date(out):
        return out
    tmp = out + ".tmp"
    cmd = [nvcc()] + NVCC_FLAGS + list(extra_flags or []) + ["-I", os.path.join(ROOT, "include"), "-o", tmp] + _sources()
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)
    os.replace(tmp, out)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true", help="print register and spill counts")
    ap.add_argument("--debug-bounds", action="store_true", help="also build the bounds-checking library")
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_verbose else []
    path = build(force=a.force or a.ptxas_verbose, verbose=a.verbose or a.ptxas_verbose, extra_flags=extra)
    print(path)
    if a.debug_bounds:
        print(build(force=a.force, verbose=a.verbose, extra_flags=extra, debug_bounds=True))


if __name__ == "__main__":
    sys.exit(main())
