"""Pins for the oracle's E4M3 decode table and encoder (CPU only).

The oracle's decode comes from the OFP8 definition; it is checked exhaustively
against torch's float8_e4m3fn conversion (a library routine) and against the
landmark values the OFP8 spec fixes (tests/golden/e4m3_landmarks.txt). The
encoder (brute-force nearest, ties to even, saturating) is checked against
torch's round-to-nearest-even cast inside the finite range, against exact
rational midpoints, and against the saturation rule outside it.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_landmarks.txt")


def torch_decode_all():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_exhaustive_vs_torch():
    ours = oracle.e4m3_table()
    ref = torch_decode_all()
    for c in range(256):
        if math.isnan(ref[c]):
            assert math.isnan(ours[c]), hex(c)
        else:
            assert ours[c] == ref[c], (hex(c), ours[c], ref[c])
            assert math.copysign(1.0, ours[c]) == math.copysign(1.0, ref[c]), hex(c)


def test_decode_landmarks_from_spec():
    n = 0
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        code, val = line.split()
        c = int(code, 16)
        got = oracle.e4m3_decode(c)
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val), (code, got, val)
            assert math.copysign(1.0, got) == math.copysign(1.0, float(val))
        n += 1
    assert n >= 10


def test_nan_codes_only_two():
    t = oracle.e4m3_table()
    assert [c for c in range(256) if math.isnan(t[c])] == [0x7F, 0xFF]


def test_decode_monotone_and_symmetric():
    t = oracle.e4m3_table()
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)
    for c in range(0x7F):
        assert t[c | 0x80] == -t[c]


def test_encode_roundtrip_all_finite():
    t = oracle.e4m3_table()
    for c in range(256):
        if math.isnan(t[c]):
            continue
        assert oracle.e4m3_encode(t[c]) == c, hex(c)


def _sweep_values():
    """Every finite E4M3 value, every midpoint between neighbours, and the
    float32 values one ulp either side of each midpoint, both signs."""
    t = oracle.e4m3_table()
    pos = sorted(set(float(v) for v in t[:0x7F]))
    vals = set()
    for a, b in zip(pos[:-1], pos[1:]):
        mid = np.float32((a + b) / 2)          # midpoints are exact in float32
        assert float(mid) == (a + b) / 2
        vals.update([float(mid), float(np.nextafter(mid, np.float32(0))),
                     float(np.nextafter(mid, np.float32(1e9))), a, b])
    # dense random float32 sample across the range, log-uniform magnitudes
    rng = np.random.default_rng(1234)
    mags = np.exp(rng.uniform(np.log(1e-5), np.log(448.0), 20000)).astype(np.float32)
    vals.update(float(v) for v in mags)
    vals = np.array(sorted(vals), dtype=np.float32)
    return np.concatenate([vals, -vals])


def test_encode_vs_torch_rne_in_range():
    ys = _sweep_values()
    ys = ys[np.abs(ys) <= 448.0]
    ref = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(y)) for y in ys], dtype=np.uint8)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(ys[i]), int(ours[i]), int(ref[i])) for i in bad[:10]]


def test_encode_ties_go_to_even_exact():
    """At every exact midpoint the result has an even mantissa (checked with
    exact rational arithmetic, independent of the oracle's float search)."""
    t = oracle.e4m3_table()
    pos = [Fraction(float(v)) for v in t[:0x7F]]
    for c in range(0x7E):
        mid = (pos[c] + pos[c + 1]) / 2
        got = oracle.e4m3_encode(float(mid))
        assert got in (c, c + 1)
        assert got % 2 == 0, (c, float(mid), got)


def test_encode_saturates_and_nan():
    for y in [448.0, 448.0001, 463.9, 464.0, 480.0, 1e6, 3.0e38, float("inf")]:
        assert oracle.e4m3_encode(y) == 0x7E, y
        assert oracle.e4m3_encode(-y) == 0xFE, y
    assert oracle.e4m3_encode(float("nan")) == 0x7F


def test_encode_signed_zero():
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-9) == 0x80          # rounds to -0
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00      # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(2.0 ** -10 * 1.0001) == 0x01
