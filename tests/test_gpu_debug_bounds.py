"""The bounds-checked build (-DSPEC_DEBUG_BOUNDS, libspecverify_debug.so)
gives the oracle's results on every entry point and finds no index out of
range, on valid inputs and on inputs its validation rejects."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.join(os.path.dirname(HERE), "speculative_decoding_verify_temperature_b200")


@pytest.mark.gpu
def test_bounds_checked_build_matches_the_oracle(cuda_device):
    from speculative_decoding_verify_temperature_b200 import build
    build.build()
    env = dict(os.environ, SPEC_VERIFY_LIB=os.path.join(PKG, "libspecverify_debug.so"))
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_run.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "bounds_hits=0" in r.stdout
