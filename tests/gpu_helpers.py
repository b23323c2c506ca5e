"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the library's quantiser, and compare results with the CPU oracle under
the stated tolerances (normalised difference <= 1e-4 and per-element
|D - R| <= 1e-2 * max|R|, both in float64 over the elements the oracle
computed)."""
import numpy as np
import torch

import oracle

CALC_DIFF_TOL = 1e-4
ELEM_TOL = 1e-2


def dev():
    return torch.device("cuda:0")


def to_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dev())


def bf16_dev(bits):
    """uint16 bf16 bit patterns (numpy) -> torch.bfloat16 CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev()).view(
        torch.bfloat16)


def as_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def check_close(D, R, what=""):
    """D float64 (GPU result), R float64 (oracle, NaN = not computed)."""
    assert D.shape == R.shape, (D.shape, R.shape)
    ok = ~np.isnan(R)
    assert ok.any(), "nothing to compare"
    d, r = D[ok], R[ok]
    assert np.all(np.isfinite(d)), f"{what}: non-finite GPU output"
    diff = oracle.calc_diff(d, r)
    rmax = np.max(np.abs(r))
    err = np.max(np.abs(d - r))
    assert diff <= CALC_DIFF_TOL, f"{what}: calc_diff {diff:.3e}"
    assert err <= ELEM_TOL * rmax + 1e-30, f"{what}: max err {err:.3e} vs max|R| {rmax:.3e}"
    return diff, err / max(rmax, 1e-30)
