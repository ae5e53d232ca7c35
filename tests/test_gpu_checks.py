"""The checks library (libdg_checks.so, DG_CHECKS=1) on the GPU: the cases of tests/checks_cases.py
run in a child process with DG_LIB=checks, so that process loads the checks build instead of
libdg.so.  Valid inputs on odd shapes must match the oracle with no device-side check firing; each
wrongly given token id or canvas index must be reported as device error code 2."""
import os
import subprocess
import sys

import pytest

from discrete_diffusion_lm_b200 import build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checks_library_parity_and_bad_inputs():
    build.build(checks=True)
    env = dict(os.environ, DG_LIB="checks")
    r = subprocess.run([sys.executable, "-m", "tests.checks_cases"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-4000:]
    assert "libdg_checks.so" in r.stdout
