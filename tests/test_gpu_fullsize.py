"""Parity at the full benchmark sizes, through the same entry points the
benchmark times, on sampled output rows the oracle computes one by one.

Sampled rows always include each operand's first and last row and the rows on
both sides of a 128-row tile boundary; every column of a sampled row is
checked (so ragged N tails are covered). Rows the method must leave alone
(masked rows, padding rows) are checked in full against a sentinel fill.
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_07_b200 as dg
import oracle
import synth
import synth.workloads as wl
from gpu_helpers import as_f64, check_close, dev, to_dev

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FBF


def sample_rows(M, extra, seed):
    base = {0, M - 1, min(127, M - 1), min(128, M - 1)}
    rnd = synth.randint(0, M - 1, extra, seed)
    return np.array(sorted(base | set(int(r) for r in rnd)), dtype=np.int64)


def stripe(M, seed):
    """One whole 128-row tile of an M-row output at a seeded tile position."""
    t = int(synth.u64(1, seed)[0] % np.uint64((M + 127) // 128))
    return np.arange(128 * t, min(M, 128 * t + 128), dtype=np.int64)


@pytest.mark.parametrize("NK", wl.DENSE_NK)
def test_dense_sweep_full_size(NK):
    """Workload 2: every M of the sweep for one (N, K) weight."""
    N, K = NK
    nki = wl.DENSE_NK.index(NK)
    B = synth.normal((N, K), synth.seed(2, nki, 1))
    qb, sb = dg.dg_quantize_fp8(to_dev(B), dg.DG_QUANT_BLOCK_128x128)
    oqb, osb = oracle.quantize(B, oracle.BLOCK_128x128)
    assert np.array_equal(qb.cpu().numpy(), oqb)
    del B
    for M in wl.DENSE_M:
        i = wl.dense_shapes().index((M, N, K))
        A = synth.normal((M, K), synth.seed(2, i, 0))
        qa, sa = dg.dg_quantize_fp8(to_dev(A), dg.DG_QUANT_ROW_1x128)
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
        dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, D)
        rows = sample_rows(M, 6, synth.seed(60, i))
        oqa, osa = oracle.quantize(np.ascontiguousarray(A[rows]), oracle.ROW_1x128)
        assert np.array_equal(qa.cpu().numpy()[rows], oqa)
        R = oracle.gemm_nt(oqa, osa, oqb, osb)
        check_close(as_f64(D)[rows], R, f"dense {M}x{N}x{K}")


def test_contiguous_full_size():
    """Workload 3: 8 experts, N=4096, K=7168, rows/expert ~ U[2048, 6144]."""
    w = wl.contiguous()
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    D = torch.full((w.Mt, w.N), SENTINEL, dtype=torch.int16, device=dev()).view(torch.bfloat16)
    dg.dg_m_grouped_fp8_gemm_nt_contiguous(qa, sa, qb, sb, to_dev(w.m_indices), None, D)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    # per expert: its first, middle and last row, plus one whole 128-row tile
    # (every row a tile holds) at a seeded tile position inside the expert
    rows = []
    off = 0
    pick = synth.u64(w.G, synth.seed(62, 0))
    for g, r in enumerate(w.rows):
        rows += [off, off + r - 1, off + r // 2]
        t = int(pick[g] % np.uint64((r + 127) // 128))
        rows += [x for x in range(off + 128 * t, off + 128 * t + 128) if x < off + r]
        off += wl.align(r)
    rows = np.array(sorted(set(rows)), dtype=np.int64)
    oqa, osa = oracle.quantize(np.ascontiguousarray(w.A[rows]), oracle.ROW_1x128)
    mi_rows = w.m_indices[rows]
    R = np.empty((rows.size, w.N))
    for g in range(w.G):
        sel = np.nonzero(mi_rows == g)[0]
        R[sel] = oracle.gemm_nt(np.ascontiguousarray(oqa[sel]), np.ascontiguousarray(osa[:, sel]),
                                oqb[g], osb[g])
    check_close(as_f64(D)[rows], R, "contiguous full")
    raw = D.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(raw[w.m_indices < 0] == SENTINEL)


@pytest.mark.parametrize("NK", wl.MASKED_NK)
def test_masked_full_size(NK):
    """Workload 4: 16 groups, max_m=256, masked_m ~ U[64, 256]."""
    N, K = NK
    w = wl.masked(N=N, K=K, shape=wl.MASKED_NK.index(NK))
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    D = torch.full((w.G, w.max_m, N), SENTINEL, dtype=torch.int16,
                   device=dev()).view(torch.bfloat16)
    dg.dg_m_grouped_fp8_gemm_nt_masked(qa, sa, qb, sb, to_dev(w.masked_m), D)
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    R = oracle.m_grouped_masked(oqa, osa, oqb, osb, w.masked_m, row_stride=23)
    check_close(as_f64(D), R, f"masked {N}x{K}")
    raw = D.view(torch.int16).cpu().numpy().view(np.uint16)
    for g in range(w.G):
        assert np.all(raw[g, w.masked_m[g]:] == SENTINEL)
        assert not np.any(raw[g, :w.masked_m[g]] == SENTINEL)


def test_k_grouped_full_size():
    """Workload 5: 8 groups, M=4096, N=7168, K_g ~ U[1024, 8192] padded to 128,
    D accumulated onto C ~ N(0,1) (in place)."""
    w = wl.k_grouped()
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_COL_128x1)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_COL_128x1)
    D = to_dev(w.C)
    dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa, sa, qb, sb, w.ks, D, D)
    rows = np.union1d(sample_rows(w.M, 4, synth.seed(61, 0)), stripe(w.M, synth.seed(61, 1)))
    # the oracle quantises the sampled columns of A (COL mode is per column)
    oqa_s, osa_s = oracle.quantize(np.ascontiguousarray(w.A[:, rows]), oracle.COL_128x1)
    oqb, osb = oracle.quantize(w.B, oracle.COL_128x1)
    Cs = np.ascontiguousarray(w.C[:, rows, :])
    R = oracle.k_grouped_tn(oqa_s, osa_s, oqb, osb, w.ks, Cs)
    Dn = D.cpu().numpy()[:, rows, :].astype(np.float64)
    check_close(Dn, R, "k-grouped full")


def test_dense_weight_gradient_full_size():
    """The dense weight gradient dW = C + dY^T X (both operands stored
    K-outer, FP32 accumulated onto C) is the K-grouped TN entry point with a
    single group: M=4096, N=7168, K=4096, in place on C."""
    w = wl.k_grouped(G=1, M=4096, N=7168, ks=[4096], cfg=5, shape=1)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_COL_128x1)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_COL_128x1)
    D = to_dev(w.C)
    dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa, sa, qb, sb, w.ks, D, D)
    rows = np.union1d(sample_rows(w.M, 4, synth.seed(61, 2)), stripe(w.M, synth.seed(61, 3)))
    oqa_s, osa_s = oracle.quantize(np.ascontiguousarray(w.A[:, rows]), oracle.COL_128x1)
    oqb, osb = oracle.quantize(w.B, oracle.COL_128x1)
    Cs = np.ascontiguousarray(w.C[:, rows, :])
    R = oracle.k_grouped_tn(oqa_s, osa_s, oqb, osb, w.ks, Cs)
    Dn = D.cpu().numpy()[:, rows, :].astype(np.float64)
    check_close(Dn, R, "dense weight gradient (G = 1)")
