"""Failure detection without a GPU fault.

The library's test hook makes the next GEMM launch skip arming its first
pipeline stage (a dropped arrive). Every consumer wait in the kernels is
bounded, so the launch must end on its own within the (shortened) timeout,
report DG_ERR_TIMEOUT with the site of the wait that gave up, free its TMEM,
and leave the context usable: the next launch on the same stream is correct.
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

SITES = {1, 2, 3, 4, 5, 6, 7, 8}


@pytest.fixture
def short_timeout():
    dg.dg_set_wait_timeout_ns(20_000_000)  # 20 ms
    st, _ = dg.dg_get_last_device_error()
    assert st == dg.DG_OK
    yield
    dg.dg_debug_drop_next_arrive(False)
    dg.dg_set_wait_timeout_ns(0)


def run_dense(M, N, K, cfg):
    w = wl.dense(M, N, K, cfg=cfg)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    return w, (qa, sa, qb, sb)


@pytest.mark.parametrize("M", [256, 64])  # persistent kernel, then the decode cluster kernel
def test_dropped_arrive_times_out_and_recovers(short_timeout, M):
    N, K = 512, 1024
    w, (qa, sa, qb, sb) = run_dense(M, N, K, cfg=75)
    D = torch.zeros((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_debug_drop_next_arrive(True)
    dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, D)
    st, site = dg.dg_get_last_device_error()
    assert st == dg.DG_ERR_TIMEOUT
    assert site in SITES
    # the error word was cleared, and the context still computes correctly
    dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, D)
    st2, _ = dg.dg_get_last_device_error()
    assert st2 == dg.DG_OK
    oqa, osa = oracle.quantize(w.A, oracle.ROW_1x128)
    oqb, osb = oracle.quantize(w.B, oracle.BLOCK_128x128)
    check_close(as_f64(D), oracle.gemm_nt(oqa, osa, oqb, osb), "after recovery")


def test_dropped_arrive_k_grouped(short_timeout):
    ks = [256, 384]
    w = wl.k_grouped(G=2, M=128, N=256, ks=ks, cfg=76)
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_COL_128x1)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_COL_128x1)
    D = torch.zeros((2, 128, 256), device=dev())
    dg.dg_debug_drop_next_arrive(True)
    dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa, sa, qb, sb, ks, None, D)
    st, site = dg.dg_get_last_device_error()
    assert st == dg.DG_ERR_TIMEOUT and site in SITES
    dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa, sa, qb, sb, ks, None, D)
    assert dg.dg_get_last_device_error()[0] == dg.DG_OK
    oqa, osa = oracle.quantize(w.A, oracle.COL_128x1)
    oqb, osb = oracle.quantize(w.B, oracle.COL_128x1)
    check_close(D.cpu().numpy().astype(np.float64),
                oracle.k_grouped_tn(oqa, osa, oqb, osb, ks), "k-grouped after recovery")


def test_no_error_on_normal_launch():
    w, (qa, sa, qb, sb) = run_dense(256, 256, 512, cfg=77)
    D = torch.empty((256, 256), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, D)
    assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)
