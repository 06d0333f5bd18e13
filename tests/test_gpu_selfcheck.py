"""The installation check runs clean on a GPU."""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def test_selfcheck_passes():
    out = subprocess.run([sys.executable, "-m", "cache_gating_kv_b200.selfcheck"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "selfcheck passed" in out.stdout
