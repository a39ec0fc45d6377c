"""Builds the sm_100a shared library in-tree (``libmuon_b200.so`` beside this file)."""

from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmuon_b200.so")
# The same library with the device bounds checks compiled in (MUON_DEBUG_BOUNDS):
# every GEMM role checks each tile it takes against its class, matrix and tile
# grid before touching memory for it.  For tests and debugging, not the product path.
LIB_DEBUG = os.path.join(HERE, "libmuon_b200_debug.so")
SOURCES = [os.path.join(HERE, "csrc", "muon_api.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in ("kernels.cuh", "ptx.cuh")] + [
    os.path.join(ROOT, "include", "muon.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def _compile(lib: str, extra: list, verbose: bool) -> subprocess.Popen:
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-o", lib + ".tmp", *SOURCES]
    if verbose:
        print(" ".join(cmd))
    return subprocess.Popen(cmd)


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds the library and its bounds-checking twin (in parallel); returns the library's path."""
    jobs = [(lib, extra) for lib, extra in ((LIB, []), (LIB_DEBUG, ["-DMUON_DEBUG_BOUNDS"]))
            if force or not up_to_date(lib)]
    procs = [(lib, _compile(lib, extra, verbose)) for lib, extra in jobs]
    failed = [lib for lib, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc", output=f"building {failed} failed")
    for lib, _ in procs:
        os.replace(lib + ".tmp", lib)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
