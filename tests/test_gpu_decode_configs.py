"""Every configuration of the small-M (decode) kernel against the oracle.

The planner picks CTAs per SM (1 or 2), a split count and the token tile
(one tile of up to 128 tokens); DG_DECODE_MINB, DG_DECODE_SPLITS,
DG_DECODE_BNP=64 (two 64-token tiles for 65..128 tokens) and DG_DECODE_PAIR
(128-token tiles on CTA pairs) force them for every call. Each
case re-runs the decode parity tests in a child process with one forced plan
(split counts that do not divide a tile's tokens evenly included) and checks
the config log.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PLANS = [("1", None, None, None), ("2", None, None, None), ("1", "7", None, None),
         ("2", "3", None, None), ("2", "8", None, None), ("2", None, "64", None),
         ("1", "5", "64", None), ("1", None, None, "1"), ("1", "3", None, "1")]


@pytest.mark.parametrize("minb,splits,bnp,pair", PLANS)
def test_decode_kernel_configs_parity(minb, splits, bnp, pair):
    env = dict(os.environ, DG_DECODE_MINB=minb, DG_PRINT_CONFIGS="1")
    if splits:
        env["DG_DECODE_SPLITS"] = splits
    if bnp:
        env["DG_DECODE_BNP"] = bnp
    if pair:
        env["DG_DECODE_PAIR"] = pair
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-s", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_gemm.py", "tests/test_gpu_failure.py",
           "-k", "decode or graph or dropped_arrive"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert f"({minb} CTA/SM)" in out, "forced configuration did not run:\n" + out[-2000:]
    if splits:
        assert f"split-K {splits} " in out, "forced split count did not run:\n" + out[-2000:]
    if bnp:
        assert f"BNP={bnp} " in out, "forced token tile did not run:\n" + out[-2000:]
    if pair:
        assert "CTA pairs" in out, "CTA-pair configuration did not run:\n" + out[-2000:]


def test_small_m_plan_choice():
    """65..128 tokens: the cost model sends 128x7168x16384 (28 tiles of 256
    weight rows, 4-way split-K) to the tile kernel and 128x4096x7168 to the
    swap-AB decode kernel; the log shows which ran."""
    env = dict(os.environ, DG_PRINT_CONFIGS="1")
    env.pop("DG_SMALL_M_TILES", None)
    cmd = [sys.executable, "bench.py", "--shape", "128,7168,16384;128,4096,7168", "--steps", "1",
           "--warmup", "1", "--quick", "--no-cpu-baseline", "--no-moe"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert "M=128 N=7168 K=16384: BM=128 BN=256 tiles=28 split 4" in out, out[-2000:]
    dec = [ln for ln in out.splitlines() if "M=128 N=4096 K=7168" in ln]
    assert dec and all("CTA/SM" in ln for ln in dec), out[-2000:]
