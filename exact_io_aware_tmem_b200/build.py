"""Build libfa_b200.so in-tree with nvcc for sm_100a.

``python -m exact_io_aware_tmem_b200.build`` (or ``build()``) compiles every
``csrc/*.cu`` to an object under ``_build/`` and links the shared library
next to this file. cudart is linked statically, so the library loads on a
machine without a GPU driver (calls then fail with a CUDA error).

``build(debug=True)`` (``--debug``) builds the same sources with -DFA_DEBUG
into ``_build_debug/`` and ``libfa_b200_debug.so``: kernels with index
checks and event stamps (include/fa.h, "Debug build").
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
BUILD = os.path.join(PKG, "_build")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libfa_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
DEBUG_BUILD = os.path.join(PKG, "_build_debug")
DEBUG_LIB_PATH = os.path.join(PKG, "libfa_b200_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest(paths) -> float:
    return max((os.path.getmtime(p) for p in paths), default=0.0)


def build(force: bool = False, verbose: bool = False, extra_flags=None,
          debug: bool = False) -> str:
    """Compile stale objects and relink; returns the library path."""
    build_dir = DEBUG_BUILD if debug else BUILD
    lib_path = DEBUG_LIB_PATH if debug else LIB_PATH
    extra_flags = list(extra_flags or []) + (["-DFA_DEBUG"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    header_time = max(_newest(headers), os.path.getmtime(__file__))
    flags = NVCC_FLAGS + list(extra_flags or [])
    objects = []
    relink = force or not os.path.exists(lib_path)
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objects.append(obj)
        if (force or not os.path.exists(obj) or os.path.getmtime(obj) < max(
                os.path.getmtime(src), header_time)):
            cmd = [nvcc()] + ARCH + flags + ["-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
            relink = True
    if relink or os.path.getmtime(lib_path) < _newest(objects):
        tmp = lib_path + ".tmp"
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objects
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
