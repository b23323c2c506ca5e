"""The CTA-pair dense kernel (cta_group::2, 256-row tiles), opt-in via DG_PAIR=1.

The switch is read once per process, so each case re-runs the dense NT parity
tests in a child process with the variable set, and checks from the library's
config log that the pair kernel is the one that ran.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("pair_bn", ["256", "128"])
def test_pair_kernel_dense_parity(pair_bn):
    env = dict(os.environ, DG_PAIR="1", DG_PAIR_BN=pair_bn, DG_PRINT_CONFIGS="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-s", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_gemm.py", "tests/test_gpu_failure.py",
           "-k", "dense_nt_vs_oracle or cuda_graph or failure or timeout or drop"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert f"256x{pair_bn} tiles" in out, "pair kernel did not run:\n" + out[-2000:]
