"""The debug build (libmsda_debug.so, compiled with MSDA_DEBUG_BOUNDS): its
kernels check every gather and scatter address against the call's buffers.
The checks run in a child process (debug_bounds_child.py) with
MSDA_DEBUG_BOUNDS=1, so that the binding loads the debug library there while
this process keeps the release one."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_build_checks_gathers_and_scatters():
    env = dict(os.environ, MSDA_DEBUG_BOUNDS="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_child.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-4000:] + "\n" + r.stderr[-4000:])
    assert "debug bounds: ok" in r.stdout
