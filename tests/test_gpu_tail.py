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
