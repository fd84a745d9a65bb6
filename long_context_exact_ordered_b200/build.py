"""Build the in-tree shared library ``libringattn.so`` for sm_100a.

Usage: ``python -m long_context_exact_ordered_b200.build`` (or ``build()``).
The library is one translation unit (``csrc/ra_api.cu`` includes every
kernel header); the CUDA runtime is linked statically and the driver entry
point for tensor-map encoding is looked up at run time, so the library
loads on machines without a GPU driver.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libringattn.so")
# Debug build: the kernels also count visible pairs per row (-DRA_DEBUG_COUNT,
# include/ringattn_debug.h); used only by the mask bit-exactness tests.
LIB_COUNT = os.path.join(HERE, "libringattn_count.so")
ROOT = os.path.dirname(HERE)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = _sources() + [os.path.join(ROOT, "include", h) for h in ("ringattn.h", "ringattn_debug.h")]
    return any(os.path.getmtime(s) > t for s in deps)


def _compile(lib: str, extra: list, verbose: bool) -> str:
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    tmp = lib + ".tmp"
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-o", tmp, os.path.join(CSRC, "ra_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile ``libringattn.so`` if a source changed (or ``force``); return its path."""
    if force or needs_build(LIB):
        _compile(LIB, [], verbose)
    return LIB


def build_count(force: bool = False, verbose: bool = False) -> str:
    """Compile the debug build ``libringattn_count.so`` (-DRA_DEBUG_COUNT); return its path."""
    if force or needs_build(LIB_COUNT):
        _compile(LIB_COUNT, ["-DRA_DEBUG_COUNT"], verbose)
    return LIB_COUNT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build_count(force="--force" in sys.argv, verbose="-v" in sys.argv))
