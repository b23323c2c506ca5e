"""Pins for the oracle's FP4 (E2M1) encoding, FP4 quantiser and FP8 x FP4 GEMM.

E2M1 is pinned to the OCP MX v1.0 definition (tests/golden/e2m1_values.txt)
and to an independent library implementation (ml_dtypes.float4_e2m1fn); the
quantiser to the invariants its definition fixes; the GEMM to a numpy matmul
of the decoded, scaled operands.
"""
import os

import ml_dtypes
import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_values.txt")
F4 = ml_dtypes.float4_e2m1fn


def lib_decode(codes):
    """ml_dtypes decode of E2M1 nibbles (uint8 array, low 4 bits)."""
    return (np.asarray(codes, np.uint8) & 0xF).view(np.uint8).astype(np.uint8).view(F4).astype(
        np.float64)


def test_decode_matches_spec_table():
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        code, val = line.split()
        v = oracle.e2m1_decode(int(code, 16))
        assert v == float(val) and np.signbit(v) == np.signbit(float(val)), code


def test_decode_matches_library_all_codes():
    ours = np.array([oracle.e2m1_decode(c) for c in range(16)])
    assert np.array_equal(ours, lib_decode(np.arange(16)))


def test_encode_matches_library_rne():
    rng = np.random.default_rng(5)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    mids = (grid[1:] + grid[:-1]) / 2
    vals = np.concatenate([grid, mids, np.nextafter(mids, 0), np.nextafter(mids, 10),
                           rng.uniform(0, 6, 2000)]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    ours = np.array([oracle.e2m1_encode(v) for v in vals], np.uint8)
    ref = vals.astype(F4).view(np.uint8) & 0xF
    assert np.array_equal(ours, ref)


def test_encode_ties_even_and_saturation():
    # midpoints of the grid go to the code with a zero mantissa bit
    assert [oracle.e2m1_encode(v) for v in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)] == \
        [0, 2, 2, 4, 4, 6, 6]
    assert oracle.e2m1_encode(6.5) == 7 and oracle.e2m1_encode(1e30) == 7
    assert oracle.e2m1_encode(-7.0) == 0xF
    assert oracle.e2m1_encode(-0.0) == 0x8 and oracle.e2m1_encode(-0.1) == 0x8


def _unpack(codes):
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


@pytest.mark.parametrize("rows,cols", [(3, 32), (17, 256), (64, 1024)])
def test_quantiser_invariants(rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    x = (rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-6, 6, (rows, 1)))).astype(
        np.float32)
    x[0, :32] = 0.0  # an all-zero strip
    codes, s = oracle.quantize_fp4(x)
    assert codes.shape == (rows, cols // 2) and s.shape == (rows, cols // 32)
    # scales: powers of two, the smallest with max(amax, 1e-4) / 6 <= s
    m, _ = np.frexp(s)
    assert np.all(m == 0.5)
    amax = np.abs(x).reshape(rows, cols // 32, 32).max(axis=2)
    t = (np.maximum(amax, np.float32(1e-4)) / np.float32(6.0)).astype(np.float32)
    assert np.all(s >= t) and np.all(s / 2 < t)
    assert s[0, 0] == 2.0 ** -15  # ceil(log2(1e-4 / 6)) = -15
    # codes: the library's nearest E2M1 of x / s (exact: s is a power of two)
    y = x / np.repeat(s, 32, axis=1)
    ref = y.astype(F4).view(np.uint8) & 0xF
    assert np.array_equal(_unpack(codes), ref)


def test_quantiser_nibble_order_and_bf16_input():
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 1], x[0, 31] = 6.0, 0.5, -3.0
    codes, s = oracle.quantize_fp4(x)
    assert s[0, 0] == 1.0
    assert codes[0, 0] == 0x17  # element 0 (6.0 -> 0x7) low nibble, element 1 (0.5 -> 0x1) high
    assert codes[0, 15] == 0xD0  # element 31 (-3.0 -> 0xD) high nibble, element 30 zero
    rng = np.random.default_rng(9)
    xb = rng.standard_normal((5, 128)).astype(np.float32)
    bits = (xb.view(np.uint32) >> 16).astype(np.uint16)  # truncate to bf16
    xt = (bits.astype(np.uint32) << 16).view(np.float32)
    c1, s1 = oracle.quantize_fp4(bits, bf16=True)
    c2, s2 = oracle.quantize_fp4(xt)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def _e4m3(a):
    return a.view(ml_dtypes.float8_e4m3fn).astype(np.float64)


@pytest.mark.parametrize("M,N,K,with_c", [(5, 7, 128, False), (9, 33, 384, True), (16, 64, 512, True)])
def test_gemm_reduces_to_matmul(M, N, K, with_c):
    rng = np.random.default_rng(M * N + K)
    A = rng.integers(0, 256, (M, K), dtype=np.uint8)
    A[(A & 0x7F) == 0x7F] = 0x3A  # no NaN codes
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sfa = np.ldexp(1.0, rng.integers(-6, 7, (K // 128, M + 3))).astype(np.float32)
    sfb = np.ldexp(1.0, rng.integers(-6, 7, (N, K // 32))).astype(np.float32)
    C = None
    if with_c:
        C = (rng.standard_normal((M, N)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    R = oracle.gemm_fp8_fp4_nt(A, sfa, B, sfb, C)
    a_eff = _e4m3(A) * np.repeat(sfa[:, :M].T.astype(np.float64), 128, axis=1)
    b_eff = lib_decode(_unpack(B)) * np.repeat(sfb.astype(np.float64), 32, axis=1)
    ref = a_eff @ b_eff.T
    if with_c:
        ref += (C.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    np.testing.assert_allclose(R, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    rows = [M - 1, 0, M // 2]
    assert np.array_equal(oracle.gemm_fp8_fp4_nt(A, sfa, B, sfb, C, rows=rows), R[rows])


def test_gemm_equals_fp8_gemm_when_fp4_values_are_fp8_values():
    """Every E2M1 value is exactly an E4M3 value. With B's four 1x32 scales of
    each 128-block equal (per row, per K-block) and the same across the rows
    of each 128-row block, the FP8 x FP4 GEMM must equal the FP8 x FP8 GEMM
    on the same values with that block scale, element for element."""
    rng = np.random.default_rng(77)
    M, N, K = 7, 130, 256
    A = rng.integers(0, 256, (M, K), dtype=np.uint8)
    A[(A & 0x7F) == 0x7F] = 0x40
    nib = rng.integers(0, 16, (N, K), dtype=np.uint8)
    B4 = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    # the same values as E4M3 codes, via the oracle's own encoder
    vals = lib_decode(nib)
    B8 = np.array([[oracle.e4m3_encode(v) for v in row] for row in vals], dtype=np.uint8)
    assert np.array_equal(_e4m3(B8), vals)
    sfa = np.ldexp(1.0, rng.integers(-4, 5, (K // 128, M + 1))).astype(np.float32)
    sfb8 = np.ldexp(1.0, rng.integers(-4, 5, ((N + 127) // 128, K // 128))).astype(np.float32)
    sfb4 = np.repeat(np.repeat(sfb8, 128, axis=0)[:N], 4, axis=1)  # [N][K/32]
    R4 = oracle.gemm_fp8_fp4_nt(A, sfa, B4, np.ascontiguousarray(sfb4))
    R8 = oracle.gemm_nt(A, sfa, B8, sfb8)
    np.testing.assert_allclose(R4, R8, rtol=1e-13, atol=1e-13 * np.abs(R8).max())
