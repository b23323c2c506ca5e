"""CPU oracle for the FP8 fine-grained-scaled GEMM family -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It wraps ``liboracle.so`` (built from
``dg_oracle.c``) with numpy arrays in and out; it shares no code with the CUDA
library. What each function computes, and the passages it follows, is stated in
``dg_oracle.h``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

ROW_1x128, BLOCK_128x128, COL_128x1 = 0, 1, 2
ROW_1x128_POW2, BLOCK_128x128_POW2 = 3, 4  # power-of-two (UE8M0) scales
C_NONE, C_BF16, C_F32 = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        vp, i32, f64 = C.c_void_p, C.c_int, C.c_double
        L.dgo_e4m3_decode.argtypes = [C.c_uint8]
        L.dgo_e4m3_decode.restype = f64
        L.dgo_e4m3_encode.argtypes = [C.c_float]
        L.dgo_e4m3_encode.restype = C.c_uint8
        L.dgo_quantize.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, i32]
        L.dgo_quantize.restype = i32
        L.dgo_gemm_nt.argtypes = [vp, vp, i32, vp, vp, vp, i32, vp, i32, i32, i32, vp, i32]
        L.dgo_gemm_nt.restype = i32
        L.dgo_m_grouped_contiguous.argtypes = [vp, vp, i32, vp, vp, vp, vp, i32, vp,
                                               i32, i32, i32, i32, vp, i32]
        L.dgo_m_grouped_contiguous.restype = i32
        L.dgo_m_grouped_masked.argtypes = [vp, vp, i32, vp, vp, vp, vp, i32, i32, i32, i32, i32]
        L.dgo_m_grouped_masked.restype = i32
        L.dgo_k_grouped_tn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, i32]
        L.dgo_k_grouped_tn.restype = i32
        L.dgo_e2m1_decode.argtypes = [C.c_uint8]
        L.dgo_e2m1_decode.restype = f64
        L.dgo_e2m1_encode.argtypes = [C.c_float]
        L.dgo_e2m1_encode.restype = C.c_uint8
        L.dgo_quantize_fp4.argtypes = [vp, i32, i32, i32, vp, vp]
        L.dgo_quantize_fp4.restype = i32
        L.dgo_gemm_fp8_fp4_nt.argtypes = [vp, vp, i32, vp, vp, vp, i32, vp, i32, i32, i32, vp,
                                          i32]
        L.dgo_gemm_fp8_fp4_nt.restype = i32
        L.dgo_calc_diff.argtypes = [vp, vp, C.c_size_t]
        L.dgo_calc_diff.restype = f64
        L.dgo_num_threads.argtypes = []
        L.dgo_num_threads.restype = i32
        _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "need C-contiguous numpy"
    return a.ctypes.data_as(C.c_void_p)


def _rows(rows):
    if rows is None:
        return None, None
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    return r, r.size


def num_threads() -> int:
    return lib().dgo_num_threads()


def e4m3_decode(code: int) -> float:
    return lib().dgo_e4m3_decode(int(code) & 0xFF)


def e4m3_table() -> np.ndarray:
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(y: float) -> int:
    return int(lib().dgo_e4m3_encode(float(y)))


def sf_rows_ld(rows: int) -> int:
    """Leading dimension of a transposed (MN-major) row-scale tensor: rows
    rounded up to a multiple of 4 floats (16 bytes)."""
    return (rows + 3) // 4 * 4


def quantize(x: np.ndarray, mode: int, ld_scales: int | None = None, bf16: bool = False):
    """x: float32 [batch?, rows, cols] (or uint16 bf16 bits with bf16=True).
    Returns (codes uint8 same shape, scales float32) in the layouts of
    dg_oracle.h."""
    x = np.ascontiguousarray(x)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[None]
    batch, rows, cols = x.shape
    if mode in (ROW_1x128, ROW_1x128_POW2):
        ld = ld_scales if ld_scales is not None else sf_rows_ld(rows)
        scales = np.zeros((batch, cols // 128, ld), dtype=np.float32)
    elif mode in (BLOCK_128x128, BLOCK_128x128_POW2):
        ld = 0
        scales = np.zeros((batch, (rows + 127) // 128, (cols + 127) // 128), dtype=np.float32)
    elif mode == COL_128x1:
        ld = 0
        scales = np.zeros((batch, rows // 128, cols), dtype=np.float32)
    else:
        raise ValueError(mode)
    codes = np.zeros(x.shape, dtype=np.uint8)
    rc = lib().dgo_quantize(_p(x), int(bf16), batch, rows, cols, mode, _p(codes), _p(scales), ld)
    if rc != 0:
        raise ValueError("oracle quantize: invalid arguments")
    if squeeze:
        return codes[0], scales[0]
    return codes, scales


def _c_kind(c):
    if c is None:
        return C_NONE
    if c.dtype == np.uint16:
        return C_BF16
    if c.dtype == np.float32:
        return C_F32
    raise TypeError(c.dtype)


def gemm_nt(A, sfa, B, sfb, C=None, rows=None):
    """Dense NT. A uint8 [M,K], sfa float32 [K/128, ld], B uint8 [N,K],
    sfb float32 [ceil(N/128), K/128], C bf16-bits uint16 or float32 [M,N].
    Returns float64 [len(rows) or M, N]."""
    M, K = A.shape
    N = B.shape[0]
    r, nr = _rows(rows)
    nr = M if r is None else nr
    R = np.empty((nr, N), dtype=np.float64)
    rc = lib().dgo_gemm_nt(_p(A), _p(sfa), sfa.shape[-1], _p(B), _p(sfb), _p(C), _c_kind(C),
                           _p(R), M, N, K, _p(r), nr)
    if rc != 0:
        raise ValueError("oracle gemm_nt: invalid arguments")
    return R


def m_grouped_contiguous(A, sfa, B, sfb, m_indices, C=None, rows=None):
    Mt, K = A.shape
    G, N, _ = B.shape
    r, nr = _rows(rows)
    nr = Mt if r is None else nr
    R = np.empty((nr, N), dtype=np.float64)
    mi = np.ascontiguousarray(m_indices, dtype=np.int32)
    rc = lib().dgo_m_grouped_contiguous(_p(A), _p(sfa), sfa.shape[-1], _p(B), _p(sfb), _p(mi),
                                        _p(C), _c_kind(C), _p(R), Mt, N, K, G, _p(r), nr)
    if rc != 0:
        raise ValueError("oracle m_grouped_contiguous: invalid arguments")
    return R


def m_grouped_masked(A, sfa, B, sfb, masked_m, row_stride=1):
    G, max_m, K = A.shape
    N = B.shape[1]
    R = np.empty((G, max_m, N), dtype=np.float64)
    mm = np.ascontiguousarray(masked_m, dtype=np.int32)
    rc = lib().dgo_m_grouped_masked(_p(A), _p(sfa), sfa.shape[-1], _p(B), _p(sfb), _p(mm), _p(R),
                                    G, max_m, N, K, row_stride)
    if rc != 0:
        raise ValueError("oracle m_grouped_masked: invalid arguments")
    return R


def k_grouped_tn(A, sfa, B, sfb, ks, C=None, rows=None):
    """A uint8 [sumK, M], B uint8 [sumK, N], sfa [sumK/128, M], sfb [sumK/128, N],
    ks list of per-group K, C float32 [G, M, N]. Returns float64 [G, rows, N]."""
    M = A.shape[1]
    N = B.shape[1]
    G = len(ks)
    k = np.ascontiguousarray(np.asarray(ks, dtype=np.int32))
    r, nr = _rows(rows)
    nr = M if r is None else nr
    R = np.empty((G, nr, N), dtype=np.float64)
    if C is not None:
        assert C.dtype == np.float32
    rc = lib().dgo_k_grouped_tn(_p(A), _p(sfa), _p(B), _p(sfb), _p(k), _p(C), _p(R), G, M, N,
                                _p(r), nr)
    if rc != 0:
        raise ValueError("oracle k_grouped_tn: invalid arguments")
    return R


def e2m1_decode(code: int) -> float:
    return lib().dgo_e2m1_decode(int(code) & 0xF)


def e2m1_encode(y: float) -> int:
    return int(lib().dgo_e2m1_encode(float(y)))


def quantize_fp4(x: np.ndarray, bf16: bool = False):
    """x: float32 [rows, cols] (or uint16 bf16 bits with bf16=True), cols % 32 == 0.
    Returns (codes uint8 [rows, cols/2], element 2j in the low nibble of byte j;
    scales float32 [rows, cols/32], powers of two)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.float32)
    if lib().dgo_quantize_fp4(_p(x), int(bf16), rows, cols, _p(codes), _p(scales)) != 0:
        raise ValueError("oracle quantize_fp4: invalid arguments")
    return codes, scales


def gemm_fp8_fp4_nt(A, sfa, B, sfb, C=None, rows=None):
    """FP8 x FP4 NT. A uint8 [M,K] E4M3, sfa float32 [K/128, ld]; B uint8
    [N,K/2] packed E2M1, sfb float32 [N, K/32]; C as gemm_nt.
    Returns float64 [len(rows) or M, N]."""
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] * 2 == K and sfb.shape == (N, K // 32)
    r, nr = _rows(rows)
    nr = M if r is None else nr
    R = np.empty((nr, N), dtype=np.float64)
    rc = lib().dgo_gemm_fp8_fp4_nt(_p(A), _p(sfa), sfa.shape[-1], _p(B), _p(sfb), _p(C),
                                   _c_kind(C), _p(R), M, N, K, _p(r), nr)
    if rc != 0:
        raise ValueError("oracle gemm_fp8_fp4_nt: invalid arguments")
    return R


def calc_diff(D, R) -> float:
    D = np.ascontiguousarray(D, dtype=np.float64)
    R = np.ascontiguousarray(R, dtype=np.float64)
    assert D.shape == R.shape
    return lib().dgo_calc_diff(_p(D), _p(R), D.size)
