"""Build the fp4q CUDA library (sm_100a) in place.

The shared library is written next to this file (``libfp4q.so``) so that it
travels with the source tree; it links the CUDA runtime statically and
exports only the C ABI of ``include/fp4q.h``.  ``build_debug`` writes a second
library, ``libfp4q_debug.so``, from the same sources with ``FP4Q_DEBUG``: its
kernels bounds-check every global access they make by hand and record the
first violation in the device error word instead of making it.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfp4q.so")
DEBUG_LIB = os.path.join(PKG, "libfp4q_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                     "-Xcompiler", "-Wall", "-cudart", "static"]


def nvcc() -> str:
    cand = [shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"]
    for c in cand:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: the fp4q CUDA library cannot be built")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def stale(lib: str | None = None) -> bool:
    lib = lib or LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None, lib: str | None = None) -> str:
    """Compile every ``csrc/*.cu`` into ``libfp4q.so`` (or ``lib``) for sm_100a; return its path."""
    lib = lib or LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(extra or []), "-I", INCLUDE, "-I", CSRC, "-shared", *sources(), "-o", tmp]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build_debug(force: bool = False, verbose: bool = False) -> str:
    """The bounds-checking library, ``libfp4q_debug.so``: the same sources built with FP4Q_DEBUG=1."""
    return build(force=force, verbose=verbose, extra=["-DFP4Q_DEBUG=1"], lib=DEBUG_LIB)


if __name__ == "__main__":
    build(force=True, verbose=True)
