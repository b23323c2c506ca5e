"""Every tile width of the persistent NT kernel against the oracle.

The planner picks BN in {128, 256} from the wave count; DG_FORCE_BN
forces one width for every call. It is read once per process, so each case
re-runs the NT parity tests (dense M > 128, contiguous, masked) in a child
process, and checks the config log for the width that ran.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("bn", ["128", "256"])
def test_nt_tile_width_parity(bn):
    env = dict(os.environ, DG_FORCE_BN=bn, DG_PRINT_CONFIGS="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-s", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_gemm.py", "-k", "dense_nt_vs_oracle or contiguous or masked or graph"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert f"BN={bn} " in out, "forced tile width did not run:\n" + out[-2000:]
