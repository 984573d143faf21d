"""The checked build (-DDIFFQKV_BOUNDS_CHECK: every kernel tests the index of its global accesses
and reports DIFFQKV_ERR_DEVICE_BOUNDS instead of touching memory out of range) on the edge shapes
of every kernel, in a fresh process with DIFFQKV_BOUNDS_CHECK=1: results match the oracle and no
check fires.  (compute-sanitizer is not used on the test machines; this is its stand-in.)"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_checked_build_edge_shapes(cuda_device):
    env = dict(os.environ, DIFFQKV_BOUNDS_CHECK="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_build_cases.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "all cases ok" in r.stdout
