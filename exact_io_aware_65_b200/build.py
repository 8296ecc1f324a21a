"""Build libfa.so (the CUDA library behind include/fa.h) for sm_100a, in tree.

    python -m exact_io_aware_65_b200.build [--force] [--verbose] [--debug-bounds]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver only through the runtime's entry-point
query, so it loads on any machine with an NVIDIA driver.

``--debug-bounds`` builds libfa_debug.so instead: the same library compiled
with FA_DEBUG_BOUNDS, whose kernels check every raw-pointer global access
against its buffer and report a failed check as FA_ERR_BOUNDS through
fa_device_status().  Load it with FA_LIBRARY=<path> in the environment.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libfa.so")
DEBUG_LIB = os.path.join(HERE, "libfa_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O3",
         "-Xptxas", "-warn-spills"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(f) > t for f in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug_bounds: bool = False) -> str:
    lib = DEBUG_LIB if debug_bounds else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    defs = ["-DFA_DEBUG_BOUNDS"] if debug_bounds else []
    cmd = [NVCC, *ARCH, *FLAGS, *defs, "-shared", "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources(), "-ldl"]
    if ptxas_info:
        cmd[1:1] = ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                ptxas_info="--ptxas-info" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
