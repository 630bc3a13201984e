"""Build libckv.so (all CUDA sources of csrc/) for sm_100a with nvcc, and
libckv_debug.so, the same sources with -DCKV_DEBUG_BOUNDS (the kernels'
range checks of community segments, and the fault-injection entry point of
include/ckv_debug.h)."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libckv.so")
LIB_DEBUG = os.path.join(HERE, "libckv_debug.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def _start(lib: str, extra, verbose: bool):
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd))
    return subprocess.Popen(cmd), tmp


def _finish(lib: str, job):
    proc, tmp = job
    if proc.wait() != 0:
        raise subprocess.CalledProcessError(proc.returncode, proc.args)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    """Compile every .cu of csrc/ into one shared library next to this file
    (libckv_debug.so with the range checks when debug is set)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not stale(lib):
        return lib
    flags = [*extra, "-DCKV_DEBUG_BOUNDS"] if debug else list(extra)
    _finish(lib, _start(lib, flags, verbose))
    return lib


def build_all(force: bool = False, verbose: bool = False):
    """Both libraries, the two nvcc runs side by side."""
    jobs = [(lib, _start(lib, flags, verbose)) for lib, flags in ((LIB, []), (LIB_DEBUG, ["-DCKV_DEBUG_BOUNDS"]))
            if force or stale(lib)]
    for lib, job in jobs:
        _finish(lib, job)
    return LIB, LIB_DEBUG


if __name__ == "__main__":
    import sys
    if "--all" in sys.argv:
        print(build_all(force="--force" in sys.argv, verbose=True))
    else:
        print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv,
                    extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else []))
