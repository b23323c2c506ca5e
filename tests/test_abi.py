"""The C-ABI library loads without a GPU and exports every entry point that
include/dg.h declares; host-side validation rejects bad arguments before any
CUDA call (these paths never touch a device)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")
LIB = os.path.join(ROOT, "moe_grouped_gemm_07_b200", "libdg.so")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_gemms_and_quantiser():
    names = declared_functions()
    for n in ["dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous",
              "dg_m_grouped_fp8_gemm_nt_masked", "dg_k_grouped_fp8_gemm_tn_contiguous",
              "dg_quantize_fp8"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    assert os.path.exists(LIB), "build libdg.so first (python moe_grouped_gemm_07_b200/build.py)"
    out = subprocess.check_output(["nm", "-D", "--defined-only", LIB], text=True)
    exported = set(l.split()[-1] for l in out.splitlines() if l.strip())
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(LIB)
    for n in declared_functions():
        assert getattr(lib, n) is not None


def test_binding_exports_same_names():
    import moe_grouped_gemm_07_b200 as dg
    for n in declared_functions():
        assert hasattr(dg, n), n
        assert n in dg.EXPORTED


def test_host_utilities_without_gpu():
    import moe_grouped_gemm_07_b200 as dg
    assert dg.dg_get_mk_alignment_for_contiguous_layout() == 128
    assert dg.dg_get_tma_aligned_size(37, 4) == 40
    assert dg.dg_get_tma_aligned_size(37, 2) == 40
    assert dg.dg_get_tma_aligned_size(37, 1) == 48
    assert dg.dg_get_tma_aligned_size(64, 4) == 64
    assert dg.dg_get_tma_aligned_size(3, 3) == -1
    assert dg.dg_status_string(dg.DG_ERR_TIMEOUT) == "DG_ERR_TIMEOUT"
    assert dg.dg_status_string(99) == "DG_ERR_UNKNOWN"


def test_host_validation_before_any_cuda_call():
    import moe_grouped_gemm_07_b200 as dg
    L, vp = dg._lib, ctypes.c_void_p
    fake = vp(0x1000)
    # shape errors are reported before pointers are touched or a device queried
    assert L.dg_fp8_gemm_nt(fake, fake, fake, fake, None, fake, 8, 8, 100, None) == \
        dg.DG_ERR_UNSUPPORTED_SHAPE
    assert L.dg_fp8_gemm_nt(fake, fake, fake, fake, None, fake, 8, 12, 128, None) == \
        dg.DG_ERR_UNSUPPORTED_SHAPE
    assert L.dg_fp8_gemm_nt(fake, fake, fake, fake, None, fake, -1, 8, 128, None) == \
        dg.DG_ERR_INVALID_ARG
    assert L.dg_fp8_gemm_nt(None, None, None, None, None, None, 0, 8, 128, None) == dg.DG_OK
    assert L.dg_m_grouped_fp8_gemm_nt_contiguous(fake, fake, fake, fake, fake, None, fake, 100,
                                                 8, 128, 2, None) == dg.DG_ERR_UNSUPPORTED_SHAPE
    assert L.dg_m_grouped_fp8_gemm_nt_contiguous(fake, fake, fake, fake, fake, None, fake, 128,
                                                 8, 128, 0, None) == dg.DG_ERR_INVALID_ARG
    assert L.dg_m_grouped_fp8_gemm_nt_masked(fake, fake, fake, fake, fake, fake, 2000, 64, 0, 8,
                                             128, None) == dg.DG_ERR_UNSUPPORTED_SHAPE
    assert L.dg_m_grouped_fp8_gemm_nt_masked(fake, fake, fake, fake, fake, fake, 0, 64, 0, 8,
                                             128, None) == dg.DG_ERR_INVALID_ARG
    # expected_m is a hint only: any value passes validation
    assert L.dg_m_grouped_fp8_gemm_nt_masked(fake, fake, fake, fake, fake, fake, 2, 0, -5, 8,
                                             128, None) == dg.DG_OK
    ks = (ctypes.c_int * 2)(128, 100)
    assert L.dg_k_grouped_fp8_gemm_tn_contiguous(fake, fake, fake, fake, ks, None, fake, 2, 16,
                                                 16, None) == dg.DG_ERR_UNSUPPORTED_SHAPE
    ks = (ctypes.c_int * 2)(128, -128)
    assert L.dg_k_grouped_fp8_gemm_tn_contiguous(fake, fake, fake, fake, ks, None, fake, 2, 16,
                                                 16, None) == dg.DG_ERR_INVALID_ARG
    ks = (ctypes.c_int * 1)(128)
    assert L.dg_k_grouped_fp8_gemm_tn_contiguous(fake, fake, fake, fake, ks, None, fake, 1, 24,
                                                 16, None) == dg.DG_ERR_UNSUPPORTED_SHAPE
    # device-side K sizes: capacity and group checks happen on the host
    dk = L.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks
    assert dk(fake, fake, fake, fake, fake, 100, None, fake, 2, 16, 16, None) == \
        dg.DG_ERR_UNSUPPORTED_SHAPE
    assert dk(fake, fake, fake, fake, None, 128, None, fake, 2, 16, 16, None) == \
        dg.DG_ERR_INVALID_ARG
    assert dk(fake, fake, fake, fake, fake, 128, None, fake, 0, 16, 16, None) == \
        dg.DG_ERR_INVALID_ARG
    assert dk(fake, fake, fake, fake, fake, 128, None, fake, 300, 16, 16, None) == \
        dg.DG_ERR_UNSUPPORTED_SHAPE
    assert dk(fake, fake, fake, fake, vp(0x1002), 128, None, fake, 2, 16, 16, None) == \
        dg.DG_ERR_MISALIGNED
    assert dk(fake, fake, fake, fake, fake, 128, None, fake, 2, 0, 16, None) == dg.DG_OK
    assert L.dg_quantize_fp8(fake, 0, 1, 128, 100, 0, fake, fake, 128, None) == \
        dg.DG_ERR_UNSUPPORTED_SHAPE
    assert L.dg_quantize_fp8(fake, 0, 1, 100, 128, 2, fake, fake, 0, None) == \
        dg.DG_ERR_UNSUPPORTED_SHAPE
    # BLOCK mode takes ragged columns in whole groups of four
    assert L.dg_quantize_fp8(fake, 0, 1, 128, 130, 1, fake, fake, 0, None) == \
        dg.DG_ERR_UNSUPPORTED_SHAPE
    assert L.dg_quantize_fp8(fake, 0, 1, 128, 132, 1, vp(0x1002), fake, 0, None) == \
        dg.DG_ERR_MISALIGNED
    assert L.dg_quantize_fp8(fake, 7, 1, 128, 128, 0, fake, fake, 128, None) == \
        dg.DG_ERR_INVALID_ARG
    assert L.dg_quantize_fp8(fake, 0, 1, 128, 128, 0, fake, fake, 126, None) == \
        dg.DG_ERR_INVALID_ARG


def test_fp4_entry_validation_before_any_cuda_call():
    import moe_grouped_gemm_07_b200 as dg
    L, vp = dg._lib, ctypes.c_void_p
    fake = vp(0x1000)
    q = L.dg_quantize_fp4_e2m1
    assert q(fake, 0, 8, 100, fake, None, fake, None) == dg.DG_ERR_UNSUPPORTED_SHAPE
    assert q(fake, 7, 8, 128, fake, None, fake, None) == dg.DG_ERR_INVALID_ARG
    assert q(fake, 0, -1, 128, fake, None, fake, None) == dg.DG_ERR_INVALID_ARG
    assert q(None, 0, 0, 128, None, None, None, None) == dg.DG_OK
    assert q(fake, 0, 8, 128, vp(0x1008), None, fake, None) == dg.DG_ERR_MISALIGNED
    g = L.dg_fp8_fp4_gemm_nt
    assert g(fake, fake, fake, fake, None, fake, 8, 8, 100, None) == dg.DG_ERR_UNSUPPORTED_SHAPE
    assert g(fake, fake, fake, fake, None, fake, 8, 12, 128, None) == dg.DG_ERR_UNSUPPORTED_SHAPE
    assert g(fake, fake, fake, fake, None, fake, -1, 8, 128, None) == dg.DG_ERR_INVALID_ARG
    assert g(None, None, None, None, None, None, 0, 8, 128, None) == dg.DG_OK
    # the packed E2M1 operand must be 32-byte aligned (4-bit TMA loads)
    assert g(fake, fake, vp(0x1010), fake, None, fake, 8, 8, 128, None) == dg.DG_ERR_MISALIGNED


def test_every_environment_variable_read_is_documented():
    import re as _re
    src = os.path.join(ROOT, "moe_grouped_gemm_07_b200", "csrc", "dg_api.cu")
    read = set(_re.findall(r'getenv\("(DG_[A-Z_]+)"\)', open(src).read()))
    assert read, "no environment variables found"
    header = open(HEADER).read()
    missing = sorted(v for v in read if v not in header)
    assert not missing, missing
