"""Compile the sm_100a CUDA library (csrc/*.cu) into libfm_b200.so, in-tree.

Plain nvcc, no torch extension machinery: the library has a C ABI and the
Python binding loads it with ctypes.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libfm_b200.so")
# FM_DEBUG variant: device-side index checks and shared-memory canaries (see fm_common.cuh)
LIB_DEBUG = os.path.join(HERE, "libfm_b200_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh"))) + [
        os.path.join(ROOT, "include", "fm.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in deps())


def build(force: bool = False, verbose: bool = False, ptxas_v: bool = False, debug: bool = False) -> str:
    """Compile csrc/*.cu into libfm_b200.so (debug=True: libfm_b200_debug.so with -DFM_DEBUG)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [NVCC] + FLAGS + ["-I", os.path.join(ROOT, "include")] + (["-DFM_DEBUG"] if debug else [])
    if ptxas_v:
        cmd += ["-Xptxas", "-v"]
    cmd += sources() + ["-o", lib]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose or ptxas_v:
        sys.stderr.write(r.stdout + r.stderr)
    return lib


if __name__ == "__main__":
    build(force=True, verbose=True, ptxas_v="-v" in sys.argv, debug="--debug" in sys.argv)
