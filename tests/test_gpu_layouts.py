"""Dense NN / TN / TT layouts vs the oracle.

The operands are stored in the layout under test and quantised there by the
GPU (ROW / COL for A, BLOCK for B); the oracle quantises the same stored
arrays, and its codes and scales are transposed into the NT form its GEMM
takes (plain numpy re-layout). Quantising a [K][M] array in 128x1 column
strips groups exactly the elements a 1x128 row strip of the [M][K] array
does, so the NT-form codes also equal those of NT quantisation (checked).
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

FN = {"nn": dg.dg_fp8_gemm_nn, "tn": dg.dg_fp8_gemm_tn, "tt": dg.dg_fp8_gemm_tt}
CASES = [(256, 256, 512, True), (144, 384, 640, False), (64, 512, 1024, True),
         (1024, 2048, 2048, False), (128, 128, 128, True),
         (256, 2112, 1024, True)]   # N % 128 == 64: ragged last 128x128 block of B


def run_layout_case(layout, M, N, K, with_c, cfg, sms=0, reps=1):
    """Quantise the stored operands on the GPU, run the layout `reps` times
    (grid capped at `sms` CTAs when nonzero) and return the outputs and the
    oracle's result in NT form."""
    w = wl.dense(M, N, K, cfg=cfg, shape=M + N + K + sms, with_c=with_c)
    a_mn, b_mn = layout[0] == "t", layout[1] == "n"
    A = np.ascontiguousarray(w.A.T) if a_mn else w.A          # [K][M] or [M][K]
    B = np.ascontiguousarray(w.B.T) if b_mn else w.B          # [K][N] or [N][K]
    qa, sa = dg.dg_quantize_fp8(to_dev(A), dg.DG_QUANT_COL_128x1 if a_mn else dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(B), dg.DG_QUANT_BLOCK_128x128)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    outs = []
    dg.dg_set_num_sms(sms)
    try:
        for _ in range(reps):
            D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev())
            FN[layout](qa, sa, qb, sb, bf16_dev(Cb) if with_c else None, D)
            outs.append(D)
        assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)
    finally:
        dg.dg_set_num_sms(0)

    # oracle in NT form
    if a_mn:
        oqa, osa = oracle.quantize(A, oracle.COL_128x1)        # [K][M], [K/128][M]
        oqa = np.ascontiguousarray(oqa.T)
        sa_nt = np.zeros((K // 128, oracle.sf_rows_ld(M)), np.float32)
        sa_nt[:, :M] = osa
    else:
        oqa, sa_nt = oracle.quantize(A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(B, oracle.BLOCK_128x128)
    if b_mn:
        oqb = np.ascontiguousarray(oqb.T)                       # [N][K]
        osb = np.ascontiguousarray(osb.T)                       # [N/128][K/128]
    ref_qa, _ = oracle.quantize(w.A, oracle.ROW_1x128)
    assert np.array_equal(oqa, ref_qa)
    return outs, oracle.gemm_nt(oqa, sa_nt, oqb, osb, Cb)


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("M,N,K,with_c", CASES)
def test_dense_layouts_vs_oracle(layout, M, N, K, with_c):
    outs, R = run_layout_case(layout, M, N, K, with_c, cfg=95)
    check_close(as_f64(outs[0]), R, f"{layout} {M}x{N}x{K}")


# Split-K over a cluster: with one wave of tiles (few rows and long K) every
# tile is split; with a capped grid a partial last wave runs as a split launch.
# Results repeat bit for bit (the parts are summed in a fixed order).
SPLIT_CASES = [
    (64, 1024, 4096, True, 0),      # 4 tiles, 8 parts each
    (128, 2176, 2048, False, 0),    # 9 tiles (ragged N), 4 parts each
    (128, 2112, 2048, False, 0),    # 9 tiles, the last B block 64 wide
    (48, 512, 2048, True, 0),       # 2 tiles of 48 rows
    (384, 768, 8192, True, 8),      # 9 tiles on 8 CTAs: 1 tail tile x 8 parts
    (608, 1024, 12288, False, 16),  # 20 tiles on 16: 4 tail tiles x 4 parts
]


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("M,N,K,with_c,sms", SPLIT_CASES)
def test_dense_layouts_split_k_vs_oracle(layout, M, N, K, with_c, sms):
    outs, R = run_layout_case(layout, M, N, K, with_c, cfg=97, sms=sms, reps=2)
    assert torch.equal(outs[0], outs[1])
    check_close(as_f64(outs[0]), R, f"{layout} split {M}x{N}x{K} on {sms or 'all'} SMs")
