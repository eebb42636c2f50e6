"""The debug-bounds build (libssmscan_debug.so): every kernel family runs
with its global indices checked, in a process of its own (the binding loads
one library per process), and must record no out-of-range index; the
build's self-test must be reported."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_every_kernel_stays_in_bounds_under_the_debug_build():
    from selective_state_space_25_b200 import build as libbuild
    libbuild.build(debug_bounds=True)
    env = dict(os.environ, SSM_DEBUG_BOUNDS="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "_debug_bounds_run.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "debug-bounds ok" in r.stdout, r.stdout + r.stderr
