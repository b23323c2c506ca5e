"""Pins for the oracle's GEMMs (CPU only).

Independent checks, none of which re-types the oracle's per-K-block formula:
  * dequantise each operand elementwise (decode x scale, expanded to the
    element grid) and multiply with torch.matmul in float64 (library routine);
    the two agree to ~1e-12 relative because every 128-term E4M3 product sum
    is exact in double;
  * identity B reproduces sfa * dec(A) exactly;
  * A = 0 gives C exactly; R(C) == C + R(0) bit for bit (C added once);
  * grouped results equal per-group dense results; padding/masked rows are
    not computed;
  * a K-grouped group with K_g = 128 is one scaled outer product; K_g = 0
    gives C_g exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import synth.workloads  # noqa: F401

F32 = np.float32


def deq_rows(codes, sf_rows):
    """codes [M,K], row scales [K/128, ld] -> float64 [M,K]."""
    tab = oracle.e4m3_table()
    M, K = codes.shape
    s = np.repeat(sf_rows[:, :M].T.astype(np.float64), 128, axis=1)
    return tab[codes] * s


def deq_blocks(codes, sf_blk):
    tab = oracle.e4m3_table()
    N, K = codes.shape
    s = np.repeat(np.repeat(sf_blk.astype(np.float64), 128, axis=0), 128, axis=1)[:N, :K]
    return tab[codes] * s


def mm64(a, b):
    return (torch.from_numpy(a) @ torch.from_numpy(b).T).numpy()


def make_nt(M, N, K, seed, with_c=True):
    w = synth.workloads.dense(M, N, K, cfg=90, shape=seed, with_c=with_c)
    qa, sa = oracle.quantize(w.A, oracle.ROW_1x128)
    qb, sb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    return qa, sa, qb, sb, Cb


@pytest.mark.parametrize("M,N,K", [(1, 8, 128), (5, 200, 384), (130, 264, 512), (64, 128, 1024)])
def test_nt_vs_dequantised_torch_matmul(M, N, K):
    qa, sa, qb, sb, Cb = make_nt(M, N, K, seed=M + N + K)
    R = oracle.gemm_nt(qa, sa, qb, sb, Cb)
    ref = synth.bf16_bits_to_f32(Cb).astype(np.float64) + mm64(deq_rows(qa, sa), deq_blocks(qb, sb))
    scale = np.abs(ref).max()
    assert np.max(np.abs(R - ref)) <= 1e-12 * scale


def test_nt_row_subset_equals_full():
    qa, sa, qb, sb, Cb = make_nt(96, 136, 256, seed=3)
    full = oracle.gemm_nt(qa, sa, qb, sb, Cb)
    rows = [0, 17, 95, 42]
    sub = oracle.gemm_nt(qa, sa, qb, sb, Cb, rows=rows)
    assert np.array_equal(sub, full[rows])


def test_nt_identity_b_reproduces_dequantised_a():
    M, K = 40, 256
    N = K
    qa, sa, _, _, _ = make_nt(M, 8, K, seed=5, with_c=False)
    qb = np.zeros((N, K), dtype=np.uint8)
    qb[np.arange(N), np.arange(N)] = 0x38            # 1.0
    sb = np.ones(((N + 127) // 128, K // 128), dtype=F32)
    R = oracle.gemm_nt(qa, sa, qb, sb)
    assert np.array_equal(R, deq_rows(qa, sa))


def test_nt_zero_a_gives_c_and_c_added_once():
    M, N, K = 33, 72, 256
    qa, sa, qb, sb, Cb = make_nt(M, N, K, seed=6)
    Cf = synth.bf16_bits_to_f32(Cb).astype(np.float64)
    R0 = oracle.gemm_nt(np.zeros_like(qa), sa, qb, sb, Cb)
    assert np.array_equal(R0, Cf)
    Rc = oracle.gemm_nt(qa, sa, qb, sb, Cb)
    Rn = oracle.gemm_nt(qa, sa, qb, sb, None)
    assert np.array_equal(Rc, Cf + Rn)
    # an fp32 C goes through the same path
    C32 = synth.normal((M, N), 77)
    assert np.array_equal(oracle.gemm_nt(qa, sa, qb, sb, C32), C32.astype(np.float64) + Rn)


def test_nt_scale_linearity():
    """Doubling every A scale doubles the product exactly (powers of two)."""
    qa, sa, qb, sb, _ = make_nt(16, 64, 384, seed=8, with_c=False)
    R1 = oracle.gemm_nt(qa, sa, qb, sb)
    R2 = oracle.gemm_nt(qa, (sa * 2).astype(F32), qb, sb)
    assert np.array_equal(R2, 2 * R1)


def test_contiguous_equals_per_group_dense():
    w = synth.workloads.contiguous(G=3, N=136, K=256, lo=100, hi=300, cfg=91)
    qa, sa = oracle.quantize(w.A, oracle.ROW_1x128)
    qb, sb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    C = synth.to_bf16_bits(synth.normal((w.Mt, w.N), 92))
    R = oracle.m_grouped_contiguous(qa, sa, qb, sb, w.m_indices, C)
    for g in range(w.G):
        rows = np.nonzero(w.m_indices == g)[0]
        ref = oracle.gemm_nt(qa, sa, qb[g], sb[g], C, rows=rows)
        assert np.array_equal(R[rows], ref)
    pad = np.nonzero(w.m_indices < 0)[0]
    assert pad.size > 0 and np.all(np.isnan(R[pad]))
    # segments are 128-aligned and every expert's rows are contiguous
    off = 0
    for g, r in enumerate(w.rows):
        assert np.all(w.m_indices[off:off + r] == g)
        off += synth.workloads.align(r)
    assert off == w.Mt


def test_masked_equals_per_group_dense_and_skips_rows():
    w = synth.workloads.masked(G=4, max_m=96, N=72, K=256, lo=0, hi=96, cfg=93)
    w.masked_m[0] = 0
    w.masked_m[1] = 96
    qa, sa = oracle.quantize(w.A, oracle.ROW_1x128)        # batched: [G][K/128][ld]
    qb, sb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    R = oracle.m_grouped_masked(qa, sa, qb, sb, w.masked_m)
    for g in range(w.G):
        mm = int(w.masked_m[g])
        if mm:
            ref = oracle.gemm_nt(qa[g], sa[g], qb[g], sb[g], rows=list(range(mm)))
            assert np.array_equal(R[g, :mm], ref)
        assert np.all(np.isnan(R[g, mm:]))
    Rs = oracle.m_grouped_masked(qa, sa, qb, sb, w.masked_m, row_stride=5)
    ok = ~np.isnan(Rs)
    assert np.array_equal(Rs[ok], R[ok])


def deq_cols(codes, sf_cols):
    """codes [K, X] with per-(128-row strip, column) scales [K/128, X]."""
    tab = oracle.e4m3_table()
    return tab[codes] * np.repeat(sf_cols.astype(np.float64), 128, axis=0)


def test_k_grouped_vs_torch_matmul_per_group():
    w = synth.workloads.k_grouped(G=3, M=48, N=80, ks=[256, 0, 384], cfg=94)
    qa, sa = oracle.quantize(w.A, oracle.COL_128x1)
    qb, sb = oracle.quantize(w.B, oracle.COL_128x1)
    R = oracle.k_grouped_tn(qa, sa, qb, sb, w.ks, w.C)
    off = 0
    for g, k in enumerate(w.ks):
        a = deq_cols(qa[off:off + k], sa[off // 128:(off + k) // 128])   # [k, M]
        b = deq_cols(qb[off:off + k], sb[off // 128:(off + k) // 128])   # [k, N]
        ref = w.C[g].astype(np.float64) + (torch.from_numpy(a).T @ torch.from_numpy(b)).numpy()
        if k == 0:
            assert np.array_equal(R[g], w.C[g].astype(np.float64))
        else:
            assert np.max(np.abs(R[g] - ref)) <= 1e-12 * np.abs(ref).max()
        off += k


def test_k_grouped_single_block_is_scaled_outer_product_sum():
    w = synth.workloads.k_grouped(G=1, M=16, N=32, ks=[128], cfg=95)
    qa, sa = oracle.quantize(w.A, oracle.COL_128x1)
    qb, sb = oracle.quantize(w.B, oracle.COL_128x1)
    R = oracle.k_grouped_tn(qa, sa, qb, sb, w.ks, None, rows=[3, 7])
    tab = oracle.e4m3_table()
    for i, m in enumerate([3, 7]):
        for n in range(32):
            inner = sum(tab[qa[k, m]] * tab[qb[k, n]] for k in range(128))  # exact in double
            assert R[0, i, n] == pytest.approx(float(sa[0, m]) * float(sb[0, n]) * inner,
                                               rel=1e-15, abs=0)


def test_calc_diff_closed_forms():
    R = synth.normal((50,), 3).astype(np.float64)
    assert oracle.calc_diff(R, R) == pytest.approx(0.0, abs=1e-15)
    assert oracle.calc_diff(-R, R) == pytest.approx(2.0)
    assert oracle.calc_diff(np.zeros_like(R), R) == pytest.approx(1.0)
    assert oracle.calc_diff(np.zeros(4), np.zeros(4)) == 0.0
    Rn = R.copy()
    Rn[::2] = np.nan                                 # NaN entries are excluded
    assert oracle.calc_diff(R, Rn) == pytest.approx(0.0, abs=1e-15)
    # D = (1+e) R  ->  1 - 2(1+e)/(1+(1+e)^2) = e^2 / (2 + 2e + e^2)
    e = 1e-3
    assert oracle.calc_diff((1 + e) * R, R) == pytest.approx(e * e / (2 + 2 * e + e * e), rel=1e-6)
