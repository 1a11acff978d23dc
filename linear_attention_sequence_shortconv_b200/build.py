"""Build ``libprism.so`` and its debug build ``libprism_debug.so`` in-tree with nvcc for
sm_100a (no JIT cache).  The debug build is compiled with PRISM_DEBUG_BOUNDS: its kernels
check the global indices they compute and record PRISM_ERR_BOUNDS instead of faulting."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libprism.so")
LIB_DEBUG = os.path.join(PKG, "libprism_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def needs_rebuild(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def _command(lib: str, debug: bool) -> list[str]:
    flags = NVCC_FLAGS + (["-DPRISM_DEBUG_BOUNDS"] if debug else [])
    return [nvcc(), *flags, "-I", INCLUDE, "-I", CSRC, *sources(), "-o", lib + ".tmp"]


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile both libraries (side by side) when a source is newer; returns the release
    library's path."""
    todo = [(lib, debug) for lib, debug in ((LIB, False), (LIB_DEBUG, True)) if force or needs_rebuild(lib)]
    procs = []
    for lib, debug in todo:
        cmd = _command(lib, debug)
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((lib, cmd, subprocess.Popen(cmd)))
    failed = [cmd for _, cmd, proc in procs if proc.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    for lib, _, _ in procs:
        os.replace(lib + ".tmp", lib)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
    print(LIB_DEBUG)
