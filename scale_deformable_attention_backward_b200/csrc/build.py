"""Build ``libmsda.so`` (the C-ABI library of include/msda.h) for sm_100a.

    python scale_deformable_attention_backward_b200/csrc/build.py [--force]

nvcc cross-compiles without a GPU.  The library lands next to the Python
binding (``scale_deformable_attention_backward_b200/libmsda.so``), in-tree, so
it travels with the source tree; the CUDA runtime is linked statically.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

CSRC = os.path.dirname(os.path.abspath(__file__))
PACKAGE = os.path.dirname(CSRC)
ROOT = os.path.dirname(PACKAGE)
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PACKAGE, "libmsda.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
              "-Xcompiler", "-fPIC,-O2,-Wall", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmsda.so")
    return path


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every ``csrc/*.cu`` into ``libmsda.so``; skip if up to date."""
    if not force and os.path.exists(LIBRARY):
        newest = max(os.path.getmtime(p) for p in _inputs())
        if os.path.getmtime(LIBRARY) >= newest:
            return LIBRARY
    tmp = LIBRARY + ".tmp"
    cmd = [nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-shared",
           "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
