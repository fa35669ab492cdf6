"""Build the CUDA library libqsa_b200.so in-tree for sm_100a (B200).

nvcc cross-compiles without a GPU.  The library exports the C ABI of
include/qsa.h and links only against the CUDA runtime.
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
LIB = os.path.join(PKG, "libqsa_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-cudart", "shared", f"-I{INCLUDE}", f"-I{CSRC}"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "qsa.h")])


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libqsa_b200.so if any source is newer than it; return its path."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose else []),
           os.path.join(CSRC, "qsa_api.cu"), "-o", LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
