"""FP8 x FP4: the E2M1 quantiser bit-exact against the oracle (codes, FP32
scales and packed UE8M0 bytes), and the block-scaled FP8 x FP4 GEMM against
the oracle's FP64 result on the same quantised inputs (each side quantises
for itself; the quantisers are shown bit-identical first)."""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_07_b200 as dg
import oracle
import synth
import synth.workloads as wl
from gpu_helpers import as_f64, bf16_dev, check_close, dev, to_dev

pytestmark = pytest.mark.gpu


def expected_packed_fp4(s_rows_strips):
    """Oracle scales [R][S] (powers of two, S = K/32) -> packed UE8M0 bytes
    [S/4][ceil(R/128)][32][4][4] (last axis: strip within the word) and the
    mask of bytes the quantiser writes."""
    R, S = s_rows_strips.shape
    e = np.frexp(s_rows_strips)[1] - 1
    Q, RB = S // 4, (R + 127) // 128
    out = np.zeros((Q, RB, 32, 4, 4), np.uint8)
    mask = np.zeros_like(out, dtype=bool)
    for r in range(R):
        rb, i, j = r // 128, r % 32, (r % 128) // 32
        for c in range(S):
            out[c // 4, rb, i, j, c % 4] = e[r, c] + 127
            mask[c // 4, rb, i, j, c % 4] = True
    return out, mask


def packed_bytes(packed):
    return packed.cpu().numpy().view(np.uint8).reshape(packed.shape + (4,))


@pytest.mark.parametrize("rows,cols,bf16", [(1, 128, False), (77, 384, True), (256, 640, False),
                                            (300, 1024, True)])
def test_fp4_quantiser_bit_exact(rows, cols, bf16):
    x = synth.normal((rows, cols), synth.seed(40, rows, cols)) * np.float32(3.0)
    x[:, :32] *= np.float32(1e-3)  # strips with small scales
    if rows > 1:
        x[1, 32:64] = 0.0  # an all-zero strip
    if bf16:
        bits = synth.to_bf16_bits(x)
        xd = bf16_dev(bits)
        oc, osc = oracle.quantize_fp4(bits, bf16=True)
    else:
        xd = to_dev(x)
        oc, osc = oracle.quantize_fp4(x)
    codes, s, packed = dg.dg_quantize_fp4_e2m1(xd)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), osc.view(np.uint32))
    exp, mask = expected_packed_fp4(osc.astype(np.float64))
    assert np.array_equal(packed_bytes(packed)[mask], exp[mask])


def quantise_both(w):
    """GPU and oracle quantisation of a dense workload's A (FP8, 1x128
    power-of-two) and B (FP4, 1x32 power-of-two)."""
    qa, _, pa = dg.dg_quantize_fp8_ue8m0(to_dev(w.A), dg.DG_QUANT_ROW_1x128, with_scales=False)
    qb, _, pb = dg.dg_quantize_fp4_e2m1(to_dev(w.B), with_scales=False)
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128_POW2)
    oqb, osb = oracle.quantize_fp4(w.B)
    return (qa, pa, qb, pb), (oqa, osa, oqb, osb)


CASES = [
    (128, 256, 512, False),
    (130, 264, 384, True),     # ragged M and N; K-blocks not a multiple of 4
    (256, 512, 1024, True),
    (300, 2112, 640, False),   # ragged last N tile (its second scale unit absent)
    (513, 136, 1152, True),
    (64, 256, 128, False),     # a single K-block
    (1, 8, 256, True),
]




def test_fp4_quantiser_ties_and_signed_zeros():
    """Strips whose amax is 6 (scale 1) holding every E2M1 midpoint, values one
    ulp either side of them, the saturation edge and tiny values of both signs:
    codes (ties to even, -0 keeps its sign bit) and scales match the oracle."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    vals = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(7)),
                           np.array([0.0, 1e-30, 6.0, 5.999999], np.float32)])
    row = np.concatenate([vals, -vals])          # 52 values
    row = np.concatenate([row, np.zeros(128 - row.size, np.float32)])
    row[row.size - 1] = 6.0                      # every 32-strip has amax 6
    row[31] = 6.0
    row[63] = -6.0
    row[95] = 6.0
    x = np.tile(row, (4, 2)).astype(np.float32)  # 4 x 256
    x[1] *= np.float32(0.5)                      # scale 2^-1
    x[2] *= np.float32(8.0)                      # scale 2^3
    x[3] = -x[3]
    oc, osc = oracle.quantize_fp4(x)
    codes, s, packed = dg.dg_quantize_fp4_e2m1(to_dev(x))
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(s.cpu().numpy(), osc)


@pytest.mark.parametrize("M,N,K,with_c", CASES)
def test_fp8_fp4_gemm_vs_oracle(M, N, K, with_c):
    w = wl.dense(M, N, K, cfg=95, shape=M + N + K, with_c=with_c)
    (qa, pa, qb, pb), (oqa, osa, oqb, osb) = quantise_both(w)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    R = oracle.gemm_fp8_fp4_nt(oqa, osa, oqb, osb, Cb)
    C = bf16_dev(Cb) if with_c else None
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, C, D)
    check_close(as_f64(D), R, f"fp8 x fp4 {M}x{N}x{K}")


def test_fp8_fp4_deterministic_and_in_place_c():
    M, N, K = 256, 512, 2048
    w = wl.dense(M, N, K, cfg=96, shape=1, with_c=True)
    (qa, pa, qb, pb), (oqa, osa, oqb, osb) = quantise_both(w)
    Cb = synth.to_bf16_bits(w.C)
    outs = []
    for _ in range(3):
        D = bf16_dev(Cb).clone()
        dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, D, D)  # C aliases D
        outs.append(D)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    check_close(as_f64(outs[0]), oracle.gemm_fp8_fp4_nt(oqa, osa, oqb, osb, Cb), "in-place C")


def test_fp8_fp4_full_size_sampled_rows():
    """4096 x 7168 x 16384 (the dominant dense shape) with FP4 weights; rows
    at the start, middle and end against the oracle on those rows only."""
    M, N, K = 4096, 7168, 16384
    A = synth.normal((M, K), synth.seed(41, 0, 0))
    B = synth.normal((N, K), synth.seed(41, 0, 1))
    qa, _, pa = dg.dg_quantize_fp8_ue8m0(to_dev(A), dg.DG_QUANT_ROW_1x128, with_scales=False)
    qb, _, pb = dg.dg_quantize_fp4_e2m1(to_dev(B), with_scales=False)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, None, D)
    oqb, osb = oracle.quantize_fp4(B)
    assert np.array_equal(qb.cpu().numpy(), oqb)
    for r0 in (0, 2048, M - 32):
        oqa, osa = oracle.quantize(np.ascontiguousarray(A[r0:r0 + 32]), oracle.ROW_1x128_POW2)
        R = oracle.gemm_fp8_fp4_nt(oqa, osa, oqb, osb)
        check_close(as_f64(D[r0:r0 + 32]), R, f"full size rows {r0}..")


def test_fp8_fp4_dropped_arrive_times_out_and_recovers():
    dg.dg_set_wait_timeout_ns(50_000_000)
    try:
        M, N, K = 256, 256, 512
        w = wl.dense(M, N, K, cfg=97, shape=2)
        (qa, pa, qb, pb), (oqa, osa, oqb, osb) = quantise_both(w)
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
        dg.dg_debug_drop_next_arrive(True)
        dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, None, D)
        st, site = dg.dg_get_last_device_error()
        assert st == dg.DG_ERR_TIMEOUT and site > 0
        dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, None, D)
        assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)
        check_close(as_f64(D), oracle.gemm_fp8_fp4_nt(oqa, osa, oqb, osb), "after recovery")
    finally:
        dg.dg_set_wait_timeout_ns(0)


# --------------------------------------------------------------- M <= 128
# The block-scaled decode kernel (swap-AB, cluster split-K): token widths
# 16..128, split counts from the plan, ragged N, C.
DECODE_CASES = [
    (1, 256, 4096, False),
    (16, 2112, 1024, True),
    (30, 384, 640, False),
    (64, 264, 512, True),     # ragged last weight tile
    (100, 1032, 2048, True),
    (128, 7168, 2048, False),
    (128, 19200, 256, False),  # at least one weight tile per SM: one split
]


@pytest.mark.parametrize("M,N,K,with_c", DECODE_CASES)
def test_fp8_fp4_decode_vs_oracle(M, N, K, with_c):
    w = wl.dense(M, N, K, cfg=98, shape=M + N + K, with_c=with_c)
    (qa, pa, qb, pb), (oqa, osa, oqb, osb) = quantise_both(w)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    R = oracle.gemm_fp8_fp4_nt(oqa, osa, oqb, osb, Cb)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, bf16_dev(Cb) if with_c else None, D)
    check_close(as_f64(D), R, f"fp8 x fp4 decode {M}x{N}x{K}")


@pytest.mark.parametrize("minb,splits", [(1, 1), (2, 1), (1, 3), (2, 5), (1, 8), (2, 8)])
def test_fp8_fp4_decode_plans(monkeypatch, minb, splits):
    """Forced plans (CTAs per SM, split count) give the same result, bit for
    bit across repeats, and meet the bar."""
    monkeypatch.setenv("DG_DECODE_MINB", str(minb))
    monkeypatch.setenv("DG_DECODE_SPLITS", str(splits))
    M, N, K = 48, 640, 2048
    w = wl.dense(M, N, K, cfg=99, shape=minb * 10 + splits, with_c=True)
    (qa, pa, qb, pb), (oqa, osa, oqb, osb) = quantise_both(w)
    Cb = synth.to_bf16_bits(w.C)
    outs = []
    for _ in range(2):
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
        dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, bf16_dev(Cb), D)
        outs.append(D)
    assert torch.equal(outs[0], outs[1])
    check_close(as_f64(outs[0]), oracle.gemm_fp8_fp4_nt(oqa, osa, oqb, osb, Cb),
                f"plan minb={minb} splits={splits}")


def test_fp8_fp4_decode_full_size():
    """64 x 7168 x 16384, every row against the oracle."""
    M, N, K = 64, 7168, 16384
    w = wl.dense(M, N, K, cfg=100, shape=0)
    (qa, pa, qb, pb), (oqa, osa, oqb, osb) = quantise_both(w)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, None, D)
    check_close(as_f64(D), oracle.gemm_fp8_fp4_nt(oqa, osa, oqb, osb), "decode full size")


def test_fp8_fp4_decode_dropped_arrive_times_out_and_recovers():
    dg.dg_set_wait_timeout_ns(50_000_000)
    try:
        M, N, K = 32, 512, 1024
        w = wl.dense(M, N, K, cfg=101, shape=3)
        (qa, pa, qb, pb), (oqa, osa, oqb, osb) = quantise_both(w)
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
        dg.dg_debug_drop_next_arrive(True)
        dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, None, D)
        st, site = dg.dg_get_last_device_error()
        assert st == dg.DG_ERR_TIMEOUT and site > 0
        dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, None, D)
        assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)
        check_close(as_f64(D), oracle.gemm_fp8_fp4_nt(oqa, osa, oqb, osb), "after recovery")
    finally:
        dg.dg_set_wait_timeout_ns(0)
