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


@pytest.mark.gpu
def test_pair_gemm_bf16_recipe():
    """The BF16 recipe's forward and backward GEMMs on CTA pairs (kind::f16,
    mode-1 weight gradients over 64-token K tiles included)."""
    env = dict(os.environ, MOE_GEMM_PAIR="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        "tests/test_gpu_bf16.py", "tests/test_gpu_bf16_bwd.py"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
