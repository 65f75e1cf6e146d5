"""Compile the float64 CPU oracle (``msda_oracle.c``) into a shared library.

Test infrastructure: the library this builds is loaded only by the tests, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``.

Run ``python oracle/build.py`` or call :func:`build`.  Plain ``gcc``, no
OpenMP and no fast-math: the oracle's arithmetic stays IEEE float64.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "msda_oracle.c")
LIBRARY = os.path.join(HERE, "_build", "libmsda_oracle.so")


def compile_source(source: str, output: str) -> str:
    """Compile one C file of oracle arithmetic into a shared library at ``output``."""
    os.makedirs(os.path.dirname(output), exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c99", "-Wall", "-Wextra", "-fPIC", "-shared",
           "-ffp-contract=off", "-o", output, source, "-lm"]
    subprocess.run(cmd, check=True)
    return output


def build(force: bool = False) -> str:
    """Build ``_build/libmsda_oracle.so`` if it is missing or older than the source."""
    stale = (not os.path.exists(LIBRARY)
             or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE))
    if force or stale:
        compile_source(SOURCE, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
