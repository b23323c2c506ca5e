"""GPU GEMMs vs the CPU oracle on seeded inputs, element by element.

Each case quantises the same float32 inputs on both sides (GPU kernels vs
oracle), runs the GPU GEMM through the C ABI and the FP64 oracle GEMM, and
checks calc_diff <= 1e-4 and |D - R| <= 1e-2 max|R|. Shapes span several tiles
and ragged M/N tails; rows the method leaves alone (masked rows, padding rows)
are checked bit-exactly against a sentinel fill.
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

SENTINEL = 0x7FBF  # a bf16 NaN pattern no computed value can produce


def quant_nt_gpu(A, B):
    qa, sa = dg.dg_quantize_fp8(to_dev(A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(B), dg.DG_QUANT_BLOCK_128x128)
    return qa, sa, qb, sb


def quant_nt_cpu(A, B):
    oqa, osa = oracle.quantize(A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(B, oracle.BLOCK_128x128)
    return oqa, osa, oqb, osb


def sentinel_bf16(shape):
    t = torch.full(shape, SENTINEL, dtype=torch.int16, device=dev())
    return t.view(torch.bfloat16)


# ------------------------------------------------------------------ dense NT
DENSE_CASES = [
    (128, 256, 512, False),     # the correctness configuration (C = 0)
    (1, 8, 128, False),
    (77, 200, 384, True),
    (130, 264, 512, True),
    (256, 512, 1024, True),
    (300, 2112, 256, False),    # ragged last N tile (2112 = 8.25 x 256)
    (513, 136, 640, True),
]


@pytest.mark.parametrize("M,N,K,with_c", DENSE_CASES)
def test_dense_nt_vs_oracle(M, N, K, with_c):
    w = wl.dense(M, N, K, cfg=80, shape=M + N + K, with_c=with_c)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    qa, sa, qb, sb = quant_nt_gpu(w.A, w.B)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_gemm_nt(qa, sa, qb, sb, bf16_dev(Cb) if with_c else None, D)
    R = oracle.gemm_nt(*quant_nt_cpu(w.A, w.B), Cb)
    check_close(as_f64(D), R, f"dense {M}x{N}x{K}")


# M <= 128 runs the swap-AB split-K cluster kernel (token widths 16/32/64/128)
# or, for 65..128 tokens where a cost model expects it to be faster, 128 x 256
# tiles split along K over a cluster; DG_SMALL_M_TILES=0|1 forces either, and
# every case runs on both
DECODE_CASES = [
    (1, 256, 7168, False),
    (16, 2112, 7168, True),
    (17, 200, 1024, False),
    (33, 1024, 2048, True),
    (64, 384, 512, False),
    (100, 2112, 3072, True),
    (128, 4096, 1408, False),   # 11 K-blocks: uneven split
    (128, 136, 128, True),      # a single K-block
    # more tile counts for the split planner (42, 48 and 98 tiles of 128 rows)
    (48, 5376, 2048, True),
    (80, 6144, 2048, False),
    (24, 12544, 768, True),
]


@pytest.mark.parametrize("path", ["0", "1"])
@pytest.mark.parametrize("M,N,K,with_c", DECODE_CASES)
def test_dense_decode_path_vs_oracle(M, N, K, with_c, path, monkeypatch):
    monkeypatch.setenv("DG_SMALL_M_TILES", path)
    w = wl.dense(M, N, K, cfg=88, shape=M + N + K, with_c=with_c)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    qa, sa, qb, sb = quant_nt_gpu(w.A, w.B)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_gemm_nt(qa, sa, qb, sb, bf16_dev(Cb) if with_c else None, D)
    R = oracle.gemm_nt(*quant_nt_cpu(w.A, w.B), Cb)
    check_close(as_f64(D), R, f"decode {M}x{N}x{K}")


def test_decode_deterministic_and_c_alias():
    M, N, K = 128, 2112, 7168
    w = wl.dense(M, N, K, cfg=89, with_c=True)
    Cb = synth.to_bf16_bits(w.C)
    qa, sa, qb, sb = quant_nt_gpu(w.A, w.B)
    outs = []
    for _ in range(3):
        D = bf16_dev(Cb).clone()
        dg.dg_fp8_gemm_nt(qa, sa, qb, sb, D, D)
        outs.append(D.view(torch.int16).cpu().numpy())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
    R = oracle.gemm_nt(*quant_nt_cpu(w.A, w.B), Cb)
    check_close(synth.bf16_bits_to_f32(outs[0].view(np.uint16)).astype(np.float64), R,
                "decode C alias")


def test_dense_c_aliases_d_and_is_added_once():
    M, N, K = 200, 384, 512
    w = wl.dense(M, N, K, cfg=81, with_c=True)
    Cb = synth.to_bf16_bits(w.C)
    qa, sa, qb, sb = quant_nt_gpu(w.A, w.B)
    D = bf16_dev(Cb).clone()
    dg.dg_fp8_gemm_nt(qa, sa, qb, sb, D, D)
    R = oracle.gemm_nt(*quant_nt_cpu(w.A, w.B), Cb)
    check_close(as_f64(D), R, "C aliases D")


def test_dense_deterministic():
    M, N, K = 384, 768, 1024
    w = wl.dense(M, N, K, cfg=82)
    qa, sa, qb, sb = quant_nt_gpu(w.A, w.B)
    outs = []
    for _ in range(3):
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
        dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, D)
        outs.append(D.view(torch.int16).cpu().numpy())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_dense_k_zero_copies_c_and_empty_is_noop():
    M, N = 64, 128
    C = torch.randn(M, N, device=dev()).to(torch.bfloat16)
    D = torch.zeros(M, N, device=dev(), dtype=torch.bfloat16)
    e = torch.empty(0, device=dev(), dtype=torch.uint8)
    s = torch.zeros(1, device=dev(), dtype=torch.float32)
    dg._check("k0", dg._lib.dg_fp8_gemm_nt(None, None, None, None, dg._ptr(C), dg._ptr(D), M, N, 0,
                                           dg._stream()))
    torch.cuda.synchronize()
    assert torch.equal(D.view(torch.int16), C.view(torch.int16))
    assert dg._lib.dg_fp8_gemm_nt(None, None, None, None, None, None, 0, N, 128,
                                  dg._stream()) == dg.DG_OK
    del e, s


def test_dense_rejects_bad_args():
    z = torch.zeros(16, device=dev(), dtype=torch.uint8)
    p = dg._ptr(z)
    st = dg._stream()
    assert dg._lib.dg_fp8_gemm_nt(p, p, p, p, None, p, 8, 8, 100, st) == dg.DG_ERR_UNSUPPORTED_SHAPE
    assert dg._lib.dg_fp8_gemm_nt(p, p, p, p, None, p, 8, 12, 128, st) == dg.DG_ERR_UNSUPPORTED_SHAPE
    assert dg._lib.dg_fp8_gemm_nt(p, p, p, p, None, p, -1, 8, 128, st) == dg.DG_ERR_INVALID_ARG
    bad = dg._vp(z.data_ptr() + 4)
    assert dg._lib.dg_fp8_gemm_nt(bad, p, p, p, None, p, 8, 8, 128, st) == dg.DG_ERR_MISALIGNED
    assert dg._lib.dg_fp8_gemm_nt(None, p, p, p, None, p, 8, 8, 128, st) == dg.DG_ERR_INVALID_ARG


# ------------------------------------------------------------------ contiguous
@pytest.mark.parametrize("G,N,K,lo,hi", [(3, 264, 256, 100, 300), (4, 512, 384, 1, 200)])
def test_contiguous_vs_oracle(G, N, K, lo, hi):
    w = wl.contiguous(G=G, N=N, K=K, lo=lo, hi=hi, cfg=83, shape=G)
    Cb = synth.to_bf16_bits(synth.normal((w.Mt, N), synth.seed(83, G, 2)))
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    D = sentinel_bf16((w.Mt, N))
    mi = to_dev(w.m_indices)
    dg.dg_m_grouped_fp8_gemm_nt_contiguous(qa, sa, qb, sb, mi, bf16_dev(Cb), D)
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    R = oracle.m_grouped_contiguous(oqa, osa, oqb, osb, w.m_indices, Cb)
    check_close(as_f64(D), R, "contiguous")
    raw = D.view(torch.int16).cpu().numpy().view(np.uint16)
    pad = w.m_indices < 0
    assert np.all(raw[pad] == SENTINEL), "padding rows were written"


# ------------------------------------------------------------------ masked
@pytest.mark.parametrize("G,max_m,N,K", [(4, 192, 200, 384), (3, 256, 512, 256)])
def test_masked_vs_oracle(G, max_m, N, K):
    w = wl.masked(G=G, max_m=max_m, N=N, K=K, lo=0, hi=max_m, cfg=84, shape=G)
    w.masked_m[0] = max_m
    w.masked_m[-1] = 0
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    D = sentinel_bf16((G, max_m, N))
    dg.dg_m_grouped_fp8_gemm_nt_masked(qa, sa, qb, sb, to_dev(w.masked_m), D)
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    R = oracle.m_grouped_masked(oqa, osa, oqb, osb, w.masked_m)
    check_close(as_f64(D), R, "masked")
    raw = D.view(torch.int16).cpu().numpy().view(np.uint16)
    for g in range(G):
        assert np.all(raw[g, w.masked_m[g]:] == SENTINEL), f"group {g}: masked rows written"


def test_masked_last_wave_split():
    """Masked GEMM on a capped grid: 60 tiles of 128 x 256 on 28 CTAs leave a
    last wave of 4 tiles, which a second launch splits 4 ways along K over
    clusters (the count is known only on the device). Results match the
    oracle, repeat bit for bit, and rows past each count stay untouched."""
    G, max_m, N, K = 3, 256, 3072, 4096
    w = wl.masked(G=G, max_m=max_m, N=N, K=K, lo=0, hi=max_m, cfg=99, shape=G)
    w.masked_m[:] = np.array([200, 100, 256], dtype=w.masked_m.dtype)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    outs = []
    dg.dg_set_num_sms(28)
    try:
        for _ in range(2):
            D = sentinel_bf16((G, max_m, N))
            dg.dg_m_grouped_fp8_gemm_nt_masked(qa, sa, qb, sb, to_dev(w.masked_m), D)
            outs.append(D)
        assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)
    finally:
        dg.dg_set_num_sms(0)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    R = oracle.m_grouped_masked(oqa, osa, oqb, osb, w.masked_m)
    check_close(as_f64(outs[0]), R, "masked, split last wave")
    raw = outs[0].view(torch.int16).cpu().numpy().view(np.uint16)
    for g in range(G):
        assert np.all(raw[g, w.masked_m[g]:] == SENTINEL), f"group {g}: masked rows written"


def test_masked_expected_m_hint_changes_plan_not_results():
    """expected_m only steers the host's tile-width plan. For 8 groups of up
    to 1024 rows, N=1024, the bound (64 row blocks) plans 128x256 tiles and
    the hint expected_m=128 (8 row blocks) plans 128x128 tiles; the results
    must be bit-identical and meet the bar."""
    G, max_m, N, K = 8, 1024, 1024, 256
    w = wl.masked(G=G, max_m=max_m, N=N, K=K, lo=1, hi=128, cfg=86)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    mm = to_dev(w.masked_m)
    outs = []
    for hint in (None, 128, 1, 5000):
        D = sentinel_bf16((G, max_m, N))
        dg.dg_m_grouped_fp8_gemm_nt_masked(qa, sa, qb, sb, mm, D, expected_m=hint)
        outs.append(D)
    for D in outs[1:]:
        assert torch.equal(D.view(torch.int16), outs[0].view(torch.int16))
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    check_close(as_f64(outs[1]), oracle.m_grouped_masked(oqa, osa, oqb, osb, w.masked_m),
                "masked with hint")


def test_masked_counts_above_max_are_clamped():
    G, max_m, N, K = 2, 128, 128, 128
    w = wl.masked(G=G, max_m=max_m, N=N, K=K, cfg=85)
    mm = np.array([1000, -5], dtype=np.int32)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    D = sentinel_bf16((G, max_m, N))
    dg.dg_m_grouped_fp8_gemm_nt_masked(qa, sa, qb, sb, to_dev(mm), D)
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    R = oracle.m_grouped_masked(oqa, osa, oqb, osb, np.array([max_m, 0], dtype=np.int32))
    check_close(as_f64(D), R, "masked clamp")
    raw = D.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(raw[1] == SENTINEL)


# ------------------------------------------------------------------ K-grouped
@pytest.mark.parametrize("G,M,N,ks,with_c", [
    (3, 144, 272, [256, 0, 384], True),
    (2, 128, 256, [128, 640], False),
    (4, 256, 512, [384, 128, 256, 512], True),
])
def test_k_grouped_vs_oracle(G, M, N, ks, with_c):
    w = wl.k_grouped(G=G, M=M, N=N, ks=ks, cfg=86, shape=G)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_COL_128x1)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_COL_128x1)
    C = to_dev(w.C) if with_c else None
    D = torch.full((G, M, N), float("nan"), device=dev())
    dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa, sa, qb, sb, w.ks, C, D)
    oqa, osa = oracle.quantize(w.A, oracle.COL_128x1)
    oqb, osb = oracle.quantize(w.B, oracle.COL_128x1)
    R = oracle.k_grouped_tn(oqa, osa, oqb, osb, w.ks, w.C if with_c else None)
    check_close(D.cpu().numpy().astype(np.float64), R, "k-grouped")
    for g, k in enumerate(ks):
        if k == 0:
            expect = w.C[g] if with_c else np.zeros((M, N), np.float32)
            assert np.array_equal(D[g].cpu().numpy(), expect)


@pytest.mark.parametrize("ks,extra", [([256, 0, 384, 128], 0), ([128, 640], 256), ([0, 0, 128], 128)])
def test_k_grouped_device_sizes(ks, extra):
    """Sizes in device memory (capacity may exceed their sum): same result as
    the host-size call bit for bit, and the oracle's within tolerance."""
    G, M, N = len(ks), 256, 384
    w = wl.k_grouped(G=G, M=M, N=N, ks=ks, cfg=89, shape=G + extra)
    A = np.concatenate([w.A, np.zeros((extra, M), np.float32)])
    B = np.concatenate([w.B, np.zeros((extra, N), np.float32)])
    qa, sa = dg.dg_quantize_fp8(to_dev(A), dg.DG_QUANT_COL_128x1)
    qb, sb = dg.dg_quantize_fp8(to_dev(B), dg.DG_QUANT_COL_128x1)
    C = to_dev(w.C)
    D1 = torch.empty((G, M, N), dtype=torch.float32, device=dev())
    D2 = torch.empty_like(D1)
    ks_dev = torch.tensor(ks, dtype=torch.int32, device=dev())
    dg.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(qa, sa, qb, sb, ks_dev, C, D1)
    assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)
    s = sum(ks)
    dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa[:s], sa[: s // 128], qb[:s], sb[: s // 128], ks, C, D2)
    assert torch.equal(D1, D2)
    oqa, osa = oracle.quantize(w.A, oracle.COL_128x1)
    oqb, osb = oracle.quantize(w.B, oracle.COL_128x1)
    R = oracle.k_grouped_tn(oqa, osa, oqb, osb, ks, w.C)
    check_close(D1.cpu().numpy().astype(np.float64), R, "k-grouped, device sizes")


def test_k_grouped_device_sizes_invalid_are_reported():
    """A size that is not a multiple of 128, or a sum beyond the capacity,
    counts as empty / is clamped and is reported as DG_ERR_INVALID_ARG."""
    G, M, N = 3, 128, 256
    w = wl.k_grouped(G=G, M=M, N=N, ks=[128, 256, 128], cfg=90)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_COL_128x1)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_COL_128x1)
    C = to_dev(w.C)
    D = torch.empty((G, M, N), dtype=torch.float32, device=dev())
    bad = torch.tensor([128, 100, 256], dtype=torch.int32, device=dev())  # 100: not a multiple
    dg.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(qa, sa, qb, sb, bad, C, D)
    st, site = dg.dg_get_last_device_error()
    assert st == dg.DG_ERR_INVALID_ARG and site == 9
    # group 1 counted as empty: D_1 = C_1 exactly; groups 0 and 2 use rows [0,128), [128,384)
    assert torch.equal(D[1], C[1])
    over = torch.tensor([256, 256, 256], dtype=torch.int32, device=dev())  # sum 768 > 512
    dg.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(qa, sa, qb, sb, over, C, D)
    st, site = dg.dg_get_last_device_error()
    assert st == dg.DG_ERR_INVALID_ARG and site == 9
    assert torch.equal(D[2], C[2])  # clamped to the 512 rows: group 2 gets none
    good = torch.tensor([128, 256, 128], dtype=torch.int32, device=dev())
    dg.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(qa, sa, qb, sb, good, C, D)
    assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)


def test_k_grouped_device_sizes_graph_replay():
    """Captured once, replayed with new sizes written into the same device
    array: every replay matches a fresh host-size call."""
    G, M, N, cap = 3, 128, 256, 768
    w = wl.k_grouped(G=G, M=M, N=N, ks=[256, 256, 256], cfg=91)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_COL_128x1)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_COL_128x1)
    D = torch.empty((G, M, N), dtype=torch.float32, device=dev())
    ks_dev = torch.tensor([256, 256, 256], dtype=torch.int32, device=dev())
    dg.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(qa, sa, qb, sb, ks_dev, None, D)  # set-up call
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            dg.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(qa, sa, qb, sb, ks_dev, None, D)
    for ks in ([256, 256, 256], [0, 640, 128], [384, 0, 0]):
        ks_dev.copy_(torch.tensor(ks, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        ref = torch.empty_like(D)
        n = sum(ks)
        dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa[:n], sa[: n // 128], qb[:n], sb[: n // 128], ks,
                                               None, ref)
        torch.cuda.synchronize()
        assert torch.equal(D, ref), ks


def test_k_grouped_accumulates_in_place():
    G, M, N, ks = 2, 128, 256, [256, 384]
    w = wl.k_grouped(G=G, M=M, N=N, ks=ks, cfg=87)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_COL_128x1)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_COL_128x1)
    D = to_dev(w.C).clone()
    dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa, sa, qb, sb, ks, D, D)
    oqa, osa = oracle.quantize(w.A, oracle.COL_128x1)
    oqb, osb = oracle.quantize(w.B, oracle.COL_128x1)
    R = oracle.k_grouped_tn(oqa, osa, oqb, osb, ks, w.C)
    check_close(D.cpu().numpy().astype(np.float64), R, "k-grouped in place")


def test_cuda_graph_capture_and_replay():
    """The calls do no host synchronisation or allocation, so quantise + GEMM
    (decode path, persistent path, masked) can be captured in a CUDA graph and
    replayed on new inputs. The first calls (one-time per-device set-up) are
    made before capture."""
    Ms, N, K = (64, 256), 512, 1024
    dense = {M: wl.dense(M, N, K, cfg=79, shape=M) for M in Ms}
    B = dense[Ms[0]].B
    qb, sb = dg.dg_quantize_fp8(to_dev(B), dg.DG_QUANT_BLOCK_128x128)
    bufs = {}
    for M in Ms:
        A = to_dev(dense[M].A)
        qa = torch.empty((M, K), dtype=torch.uint8, device=dev())
        sa = torch.zeros((K // 128, (M + 3) // 4 * 4), dtype=torch.float32, device=dev())
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
        bufs[M] = (A, qa, sa, D)
    mw = wl.masked(G=3, max_m=128, N=N, K=K, lo=1, hi=128, cfg=79, shape=9)
    mA, mmm = to_dev(mw.A), to_dev(mw.masked_m)
    mqa = torch.empty(mw.A.shape, dtype=torch.uint8, device=dev())
    msa = torch.zeros((3, K // 128, 128), dtype=torch.float32, device=dev())
    mqb, msb = dg.dg_quantize_fp8(to_dev(mw.B), dg.DG_QUANT_BLOCK_128x128)
    mD = torch.zeros((3, 128, N), dtype=torch.bfloat16, device=dev())

    def work():
        for M in Ms:
            A, qa, sa, D = bufs[M]
            dg.dg_quantize_fp8(A, dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa)
            dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, D)
        dg.dg_quantize_fp8(mA, dg.DG_QUANT_ROW_1x128, codes=mqa, scales=msa)
        dg.dg_m_grouped_fp8_gemm_nt_masked(mqa, msa, mqb, msb, mmm, mD)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        work()  # warm-up: one-time set-up happens outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        work()
    oqb, osb = oracle.quantize(B, oracle.BLOCK_128x128)
    for rep in range(2):
        new = {M: synth.normal((M, K), synth.seed(79, 50 + rep, M)) for M in Ms}
        for M in Ms:
            bufs[M][0].copy_(to_dev(new[M]))
        g.replay()
        torch.cuda.synchronize()
        for M in Ms:
            oqa, osa = oracle.quantize(new[M], oracle.ROW_1x128)
            check_close(as_f64(bufs[M][3]), oracle.gemm_nt(oqa, osa, oqb, osb), f"graph M={M}")
    oqa, osa = oracle.quantize(mw.A, oracle.ROW_1x128)
    oqb2, osb2 = oracle.quantize(mw.B, oracle.BLOCK_128x128)
    check_close(as_f64(mD), oracle.m_grouped_masked(oqa, osa, oqb2, osb2, mw.masked_m), "graph masked")
