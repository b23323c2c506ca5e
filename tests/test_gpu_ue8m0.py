"""Power-of-two (UE8M0) scales: quantiser bit-exact vs the oracle, and both
GEMM paths vs the oracle on the same inputs.

The two paths compute the same D = C + sum_kb sfa*sfb*P_kb with
power-of-two scales: the explicit promotion kernel (dg_fp8_gemm_nt with the
FP32 copies of the scales) and the tensor core's block-scaled MMA
(dg_fp8_gemm_nt_ue8m0 with the packed bytes), which accumulates across
K-blocks in TMEM. Both must meet the same bar against the FP64 oracle.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_07_b200 as dg
import oracle
import synth
import synth.workloads as wl
from gpu_helpers import as_f64, bf16_dev, check_close, dev, to_dev

pytestmark = pytest.mark.gpu


def expected_packed(s_rows_kb):
    """Oracle scales [R][KB] (powers of two) -> packed UE8M0 bytes
    [ceil(KB/4)][ceil(R/128)][32][4][4] (the last axis: K-block within the
    word), and a mask of the positions a quantiser writes."""
    R, KB = s_rows_kb.shape
    e = np.frexp(s_rows_kb)[1] - 1                 # s = 0.5 * 2^ex -> log2 s = ex - 1
    Q, RB = (KB + 3) // 4, (R + 127) // 128
    out = np.zeros((Q, RB, 32, 4, 4), np.uint8)
    mask = np.zeros_like(out, dtype=bool)
    for r in range(R):
        rb, i, j = r // 128, r % 32, (r % 128) // 32
        for kb in range(KB):
            out[kb // 4, rb, i, j, kb % 4] = e[r, kb] + 127
            mask[kb // 4, rb, i, j, kb % 4] = True
    return out, mask


def gpu_packed_bytes(packed):
    return packed.cpu().numpy().view(np.uint8).reshape(packed.shape + (4,))


@pytest.mark.parametrize("rows,cols", [(1, 128), (77, 384), (256, 640), (300, 1024)])
def test_ue8m0_row_quantiser_bit_exact(rows, cols):
    x = synth.normal((rows, cols), synth.seed(12, rows, 0)) * np.float32(7.0)
    codes, s, packed = dg.dg_quantize_fp8_ue8m0(to_dev(x), dg.DG_QUANT_ROW_1x128)
    oc, osc = oracle.quantize(x, oracle.ROW_1x128_POW2)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(s.cpu().numpy()[:, :rows].view(np.uint32), osc[:, :rows].view(np.uint32))
    exp, mask = expected_packed(osc[:, :rows].T.astype(np.float64))
    got = gpu_packed_bytes(packed)
    assert np.array_equal(got[mask], exp[mask])


@pytest.mark.parametrize("rows,cols", [(128, 128), (200, 512), (2112, 640)])
def test_ue8m0_block_quantiser_bit_exact(rows, cols):
    x = synth.normal((rows, cols), synth.seed(13, rows, 0))
    codes, s, packed = dg.dg_quantize_fp8_ue8m0(to_dev(x), dg.DG_QUANT_BLOCK_128x128)
    oc, osc = oracle.quantize(x, oracle.BLOCK_128x128_POW2)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), osc.view(np.uint32))
    per_row = np.repeat(osc, 128, axis=0)[:rows].astype(np.float64)  # [rows][KB]
    exp, mask = expected_packed(per_row)
    got = gpu_packed_bytes(packed)
    assert np.array_equal(got[mask], exp[mask])


CASES = [
    (128, 256, 512, False),
    (130, 264, 384, True),     # ragged M and N, K-blocks not a multiple of 4
    (256, 512, 1024, True),
    (300, 2112, 640, False),   # ragged last N tile (second scale unit absent)
    (513, 136, 1152, True),
    (64, 256, 256, False),
]


@pytest.mark.parametrize("M,N,K,with_c", CASES)
def test_ue8m0_both_paths_vs_oracle(M, N, K, with_c):
    w = wl.dense(M, N, K, cfg=92, shape=M + N + K, with_c=with_c)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    qa, sa, pa = dg.dg_quantize_fp8_ue8m0(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb, pb = dg.dg_quantize_fp8_ue8m0(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128_POW2)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128_POW2)
    R = oracle.gemm_nt(oqa, osa, oqb, osb, Cb)
    C = bf16_dev(Cb) if with_c else None
    D_hw = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, C, D_hw)
    check_close(as_f64(D_hw), R, f"block-scaled MMA {M}x{N}x{K}")
    D_pr = torch.empty_like(D_hw)
    dg.dg_fp8_gemm_nt(qa, sa, qb, sb, C, D_pr)
    check_close(as_f64(D_pr), R, f"promotion, power-of-two scales {M}x{N}x{K}")


def test_ue8m0_gemm_deterministic_and_in_place_c():
    M, N, K = 256, 512, 2048
    w = wl.dense(M, N, K, cfg=93, shape=1, with_c=True)
    qa, _, pa = dg.dg_quantize_fp8_ue8m0(to_dev(w.A), dg.DG_QUANT_ROW_1x128, with_scales=False)
    qb, _, pb = dg.dg_quantize_fp8_ue8m0(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128, with_scales=False)
    Cb = synth.to_bf16_bits(w.C)
    outs = []
    for _ in range(3):
        D = bf16_dev(Cb).clone()
        dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, D, D)  # C aliases D
        outs.append(D)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128_POW2)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128_POW2)
    check_close(as_f64(outs[0]), oracle.gemm_nt(oqa, osa, oqb, osb, Cb), "in-place C")


def test_ue8m0_full_size_sampled_rows():
    """4096 x 7168 x 16384 (the dominant benchmark shape) through the
    block-scaled path; 128-row stripes (first, middle, last) against the
    oracle computed on those rows only."""
    M, N, K = 4096, 7168, 16384
    A = synth.normal((M, K), synth.seed(14, 0, 0))
    B = synth.normal((N, K), synth.seed(14, 0, 1))
    qa, _, pa = dg.dg_quantize_fp8_ue8m0(to_dev(A), dg.DG_QUANT_ROW_1x128, with_scales=False)
    qb, _, pb = dg.dg_quantize_fp8_ue8m0(to_dev(B), dg.DG_QUANT_BLOCK_128x128, with_scales=False)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, D)
    oqb, osb = oracle.quantize(B, oracle.BLOCK_128x128_POW2)
    for r0 in (0, 2048, M - 128):
        oqa, osa = oracle.quantize(np.ascontiguousarray(A[r0:r0 + 128]), oracle.ROW_1x128_POW2)
        R = oracle.gemm_nt(oqa, osa, oqb, osb)
        check_close(as_f64(D[r0:r0 + 128]), R, f"full size rows {r0}..")


def test_ue8m0_dropped_arrive_times_out_and_recovers():
    dg.dg_set_wait_timeout_ns(50_000_000)
    try:
        M, N, K = 256, 256, 512
        w = wl.dense(M, N, K, cfg=94, shape=2)
        qa, _, pa = dg.dg_quantize_fp8_ue8m0(to_dev(w.A), dg.DG_QUANT_ROW_1x128, with_scales=False)
        qb, _, pb = dg.dg_quantize_fp8_ue8m0(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128,
                                             with_scales=False)
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
        dg.dg_debug_drop_next_arrive(True)
        dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, D)
        st, site = dg.dg_get_last_device_error()
        assert st == dg.DG_ERR_TIMEOUT and site > 0
        dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, D)
        assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)
        oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128_POW2)
        oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128_POW2)
        check_close(as_f64(D), oracle.gemm_nt(oqa, osa, oqb, osb), "after recovery")
    finally:
        dg.dg_set_wait_timeout_ns(0)


# --------------------------------------------------------------- M <= 128
# dg_fp8_gemm_nt_ue8m0 routes M <= 128 to the block-scaled decode kernel
# (swap-AB, cluster split-K).
@pytest.mark.parametrize("M,N,K,with_c", [(1, 256, 4096, False), (30, 384, 640, True),
                                          (64, 264, 1536, True), (128, 7168, 2048, False)])
def test_ue8m0_decode_vs_oracle(M, N, K, with_c):
    w = wl.dense(M, N, K, cfg=102, shape=M + N + K, with_c=with_c)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    qa, _, pa = dg.dg_quantize_fp8_ue8m0(to_dev(w.A), dg.DG_QUANT_ROW_1x128, with_scales=False)
    qb, _, pb = dg.dg_quantize_fp8_ue8m0(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128,
                                         with_scales=False)
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128_POW2)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128_POW2)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, bf16_dev(Cb) if with_c else None, D)
    check_close(as_f64(D), oracle.gemm_nt(oqa, osa, oqb, osb, Cb), f"ue8m0 decode {M}x{N}x{K}")


@pytest.mark.parametrize("minb,splits", [(1, 2), (2, 4), (1, 7)])
def test_ue8m0_decode_plans(monkeypatch, minb, splits):
    monkeypatch.setenv("DG_DECODE_MINB", str(minb))
    monkeypatch.setenv("DG_DECODE_SPLITS", str(splits))
    M, N, K = 100, 512, 3072
    w = wl.dense(M, N, K, cfg=103, shape=minb * 10 + splits)
    qa, _, pa = dg.dg_quantize_fp8_ue8m0(to_dev(w.A), dg.DG_QUANT_ROW_1x128, with_scales=False)
    qb, _, pb = dg.dg_quantize_fp8_ue8m0(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128,
                                         with_scales=False)
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128_POW2)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128_POW2)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, D)
    check_close(as_f64(D), oracle.gemm_nt(oqa, osa, oqb, osb), f"plan {minb}/{splits}")
