"""The ATTN_DEBUG build (device-side bounds checks that report instead of
trapping, NaN-filled outputs) on small cases of every entry point, in a child
process that loads it (CSA_ATTN_DEBUG=1)."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_matches_the_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, CSA_ATTN_DEBUG="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_check.py")],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build ok" in r.stdout
