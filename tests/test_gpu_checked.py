"""The bounds-checked build (LBCA_CHECKED=1): the same parity cases pass with
every cache row range the decode kernels derive tested against the cache's
extent, and no check fires on valid inputs (a fired check would set the status
word the tests assert on)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _env():
    env = dict(os.environ)
    env["LBCA_CHECKED"] = "1"
    return env


def test_checked_library_is_the_one_loaded():
    r = subprocess.run([sys.executable, "-c", "from block_compressed_long_b200 import lbca as L; print(L._LIB_PATH)"],
                       cwd=ROOT, env=_env(), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip().endswith("liblbca_checked.so")


def test_decode_parity_under_the_checked_build():
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_step_persistent.py", "tests/test_gpu_step.py", "tests/test_gpu_csa.py",
           "-k", "matches_oracle or sparse"]
    r = subprocess.run(cmd, cwd=ROOT, env=_env(), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
