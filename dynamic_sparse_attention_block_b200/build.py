"""Build the PRR decode-step library (libprr_b200.so) in-tree with nvcc for sm_100a.

Runs on a machine without a GPU: nvcc cross-compiles.  The CUDA runtime is linked
statically and the driver entry point for TMA descriptors is resolved at run time,
so the library also loads (without running anything) where no driver is present.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libprr_b200.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
]


def sources():
    """CUDA sources plus host-only C++ (the budget model), all compiled by nvcc."""
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                              + glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date(output: str = LIBRARY) -> bool:
    if not os.path.exists(output):
        return False
    t = os.path.getmtime(output)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, output: str = LIBRARY, verbose: bool = False, extra=()) -> str:
    if not force and up_to_date(output):
        return output
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, *extra, f"-I{INCLUDE}", f"-I{CSRC}", "-o", output, *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return output


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
