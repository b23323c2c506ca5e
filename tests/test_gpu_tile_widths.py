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


@pytest.mark.parametrize("bn,wide", [("128", None), ("256", "0"), ("256", "1")])
def test_nt_tile_width_parity(bn, wide):
    """256-column tiles run twice: with the 4-stage ring and per-chunk output
    staging, and with the 3-stage ring and whole-tile staging (DG_WIDE_EPI)."""
    env = dict(os.environ, DG_FORCE_BN=bn, DG_PRINT_CONFIGS="1")
    if wide:
        env["DG_WIDE_EPI"] = wide
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-s", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_gemm.py", "-k", "dense_nt_vs_oracle or contiguous or masked or graph"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert f"BN={bn} " in out, "forced tile width did not run:\n" + out[-2000:]
    if wide == "1":
        assert "wide epilogue" in out, "whole-tile staging did not run:\n" + out[-2000:]
