"""Build ``libmsda.so`` (the C-ABI library of include/msda.h) for sm_100a.

    python scale_deformable_attention_backward_b200/csrc/build.py [--force] [--debug]

nvcc cross-compiles without a GPU.  The library lands next to the Python
binding (``scale_deformable_attention_backward_b200/libmsda.so``), in-tree, so
it travels with the source tree; the CUDA runtime is linked statically.

``--debug`` builds ``libmsda_debug.so`` instead: the same sources with
MSDA_DEBUG_BOUNDS defined, so that every gather and scatter checks its address
against the call's buffers (msda_debug_bounds_check in include/msda.h).  Its
kernels share one record of refused accesses, which needs relocatable device
code (-rdc=true) across the translation units.
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
DEBUG_LIBRARY = os.path.join(PACKAGE, "libmsda_debug.so")
DEBUG_FLAGS = ["-DMSDA_DEBUG_BOUNDS", "-rdc=true"]

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


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every ``csrc/*.cu`` into ``libmsda.so`` (``libmsda_debug.so`` with
    ``debug``); skip if up to date."""
    target = DEBUG_LIBRARY if debug else LIBRARY
    if not force and os.path.exists(target):
        newest = max(os.path.getmtime(p) for p in _inputs())
        if os.path.getmtime(target) >= newest:
            return target
    tmp = target + ".tmp"
    cmd = [nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, *(DEBUG_FLAGS if debug else []), "-I", INCLUDE,
           "-I", CSRC, "-shared", "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
