"""Dense split-K tail (see tests/tail_cases.py) in a child process with
DG_FORCE_BN=256, checking from the config log that tails were split 2, 4 and
8 ways."""
import os
import re
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_split_tail_cases():
    env = dict(os.environ, DG_FORCE_BN="256", DG_PRINT_CONFIGS="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-s", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/tail_cases.py"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    splits = set(int(k) for k in re.findall(r"tail split (\d+)x", out))
    assert {2, 4, 8} <= splits, f"expected 2-, 4- and 8-way tails, saw {sorted(splits)}"


def test_split_layout_cases():
    """The NN / TN / TT split-K cases of tests/test_gpu_layouts.py in a child
    process, checking from the config log that every layout split whole
    one-wave launches 8 and 4 ways and capped-grid tails 8 and 4 ways."""
    env = dict(os.environ, DG_PRINT_CONFIGS="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-s", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_layouts.py", "-k", "split_k"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    for name in ("fp8_gemm_nn", "fp8_gemm_tn", "fp8_gemm_tt"):
        seen = set(re.findall(name + r" M=\d+ N=\d+ K=\d+: .* split (\d+x\d+)", out))
        assert {"8x4", "4x9", "4x2", "8x1", "4x4"} <= seen, f"{name}: saw {sorted(seen)}"


def test_masked_tail_split_is_planned():
    """The masked last-wave split test in a child process with the config log:
    the host plans a 4-way tail split for it."""
    env = dict(os.environ, DG_PRINT_CONFIGS="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-s", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_gemm.py", "-k", "masked_last_wave_split"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert re.search(r"masked tail split 4 x up to [1-9]\d* clusters", out), out[-2000:]
