"""The bounds-checked debug build of the library (needs a B200).

libssmscan_debug.so is the same source compiled with SSM_DEBUG: every index a scan
kernel computes into a global buffer is checked, and a bad one records
SSM_ERR_BOUNDS in the device status word instead of being used.  A child process
loads that build (SSM_SCAN_LIBRARY) and runs small and odd shapes through both
kernels; every call must report SSM_OK and match the oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_build_reports_no_bounds_error():
    from selective_state_space_30_b200 import build as b
    lib = b.build(debug=True)
    env = dict(os.environ, SSM_SCAN_LIBRARY=lib)
    res = subprocess.run([sys.executable, os.path.join(HERE, "debug_checks.py")], env=env, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-3000:]
    assert "all shapes SSM_OK" in res.stdout
