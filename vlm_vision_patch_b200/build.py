"""Build the sm_100a shared library libpe.so in-tree with nvcc (no GPU needed).

`--debug-bounds` builds libpe_debug.so instead: the same sources with
-DPE_DEBUG_BOUNDS, whose kernels check every data-dependent global access
against the buffer it indexes and report PE_ERR_DEVICE_BOUNDS instead of
touching memory outside it.  Load it by setting PE_LIB to its path before
importing the package."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpe.so")
DEBUG_LIB = os.path.join(HERE, "libpe_debug.so")
SOURCES = [os.path.join(CSRC, "pe_api.cu")]
# every file the build reads: a change to any of them makes the library stale
DEPS = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))) + \
    [os.path.join(os.path.dirname(HERE), "include", "pe.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    lib = DEBUG_LIB if debug_bounds else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    extra = ["-DPE_DEBUG_BOUNDS"] if debug_bounds else []
    cmd = [nvcc(), *NVCC_FLAGS, *extra, *SOURCES, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug_bounds="--debug-bounds" in sys.argv))
