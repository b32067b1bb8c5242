"""The CTA-pair GEMM (M = 256 tiles shared by two SMs, opt-in with
MOE_GEMM_PAIR=1) on the tiny layer: the same oracle bars as the default
path, run in a child process because the switch is read once per process."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_pair_gemm_smoke():
    env = dict(os.environ, MOE_GEMM_PAIR="1")
    r = subprocess.run([sys.executable, "-c", "import __graft_entry__ as g; g.smoke()"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
