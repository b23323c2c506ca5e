"""Python binding for libdg.so -- FP8 fine-grained-scaled GEMMs on B200.

Argument marshalling only: every function takes torch CUDA tensors, checks
their shapes/dtypes against the C ABI in ``include/dg.h``, and passes raw device
pointers plus the current CUDA stream to the library. All arithmetic runs in
the library's sm_100a kernels. If ``libdg.so`` is missing or cannot be loaded,
importing this package raises: there is no fallback path.

Functions keep the C names:
  dg_quantize_fp8, dg_fp8_gemm_nt, dg_m_grouped_fp8_gemm_nt_contiguous,
  dg_m_grouped_fp8_gemm_nt_masked, dg_k_grouped_fp8_gemm_tn_contiguous,
  dg_get_mk_alignment_for_contiguous_layout, dg_get_tma_aligned_size,
  dg_set_num_sms, dg_get_num_sms, dg_set_wait_timeout_ns,
  dg_get_last_device_error, dg_debug_drop_next_arrive, dg_get_launch_count,
  dg_set_pdl, dg_get_pdl.
"""
from __future__ import annotations

import ctypes as _C
import math
import os as _os

import torch

LIB_PATH = _os.path.join(_os.path.dirname(_os.path.abspath(__file__)), "libdg.so")

if not _os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python moe_grouped_gemm_07_b200/build.py` "
        "(there is no non-CUDA fallback)")

_lib = _C.CDLL(LIB_PATH)

DG_OK, DG_ERR_INVALID_ARG, DG_ERR_UNSUPPORTED_SHAPE, DG_ERR_MISALIGNED, DG_ERR_CUDA, \
    DG_ERR_TIMEOUT = range(6)
DG_IN_F32, DG_IN_BF16 = 0, 1
DG_QUANT_ROW_1x128, DG_QUANT_BLOCK_128x128, DG_QUANT_COL_128x1 = 0, 1, 2

EXPORTED = (
    "dg_status_string", "dg_quantize_fp8", "dg_fp8_gemm_nt",
    "dg_m_grouped_fp8_gemm_nt_contiguous", "dg_m_grouped_fp8_gemm_nt_masked",
    "dg_k_grouped_fp8_gemm_tn_contiguous", "dg_get_mk_alignment_for_contiguous_layout",
    "dg_get_tma_aligned_size", "dg_set_num_sms", "dg_get_num_sms", "dg_set_wait_timeout_ns",
    "dg_get_last_device_error", "dg_debug_drop_next_arrive", "dg_get_launch_count",
    "dg_set_pdl", "dg_get_pdl", "dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks",
    "dg_quantize_fp8_ue8m0", "dg_fp8_gemm_nt_ue8m0", "dg_fp8_gemm_nn", "dg_fp8_gemm_tn",
    "dg_fp8_gemm_tt", "dg_quantize_fp4_e2m1", "dg_fp8_fp4_gemm_nt",
)

_vp, _i32 = _C.c_void_p, _C.c_int
_lib.dg_status_string.argtypes = [_i32]
_lib.dg_status_string.restype = _C.c_char_p
_lib.dg_quantize_fp8.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp]
_lib.dg_fp8_gemm_nt.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp]
_lib.dg_m_grouped_fp8_gemm_nt_contiguous.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                                     _i32, _i32, _i32, _vp]
_lib.dg_m_grouped_fp8_gemm_nt_masked.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                                 _i32, _i32, _vp]
_lib.dg_k_grouped_fp8_gemm_tn_contiguous.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                                     _i32, _i32, _vp]
_lib.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                                            _vp, _i32, _i32, _i32, _vp]
_lib.dg_quantize_fp8_ue8m0.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _vp]
_lib.dg_fp8_gemm_nt_ue8m0.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp]
_lib.dg_quantize_fp4_e2m1.argtypes = [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp]
_lib.dg_fp8_fp4_gemm_nt.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp]
for _f in ("dg_fp8_gemm_nn", "dg_fp8_gemm_tn", "dg_fp8_gemm_tt"):
    getattr(_lib, _f).argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp]
    getattr(_lib, _f).restype = _i32
for _f in ("dg_quantize_fp8", "dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous",
           "dg_m_grouped_fp8_gemm_nt_masked", "dg_k_grouped_fp8_gemm_tn_contiguous",
           "dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks", "dg_quantize_fp8_ue8m0",
           "dg_fp8_gemm_nt_ue8m0"):
    getattr(_lib, _f).restype = _i32
_lib.dg_get_mk_alignment_for_contiguous_layout.restype = _i32
_lib.dg_get_tma_aligned_size.argtypes = [_i32, _i32]
_lib.dg_get_tma_aligned_size.restype = _i32
_lib.dg_set_num_sms.argtypes = [_i32]
_lib.dg_get_num_sms.restype = _i32
_lib.dg_set_wait_timeout_ns.argtypes = [_C.c_uint64]
_lib.dg_get_last_device_error.argtypes = [_vp, _C.POINTER(_C.c_int)]
_lib.dg_get_last_device_error.restype = _i32
_lib.dg_debug_drop_next_arrive.argtypes = [_i32]
_lib.dg_get_launch_count.restype = _C.c_uint64
_lib.dg_set_pdl.argtypes = [_i32]
_lib.dg_get_pdl.restype = _i32


class DGError(RuntimeError):
    def __init__(self, name: str, status: int):
        self.status = status
        super().__init__(f"{name}: {dg_status_string(status)}")


def dg_status_string(status: int) -> str:
    return _lib.dg_status_string(int(status)).decode()


def _check(name, status):
    if status != DG_OK:
        raise DGError(name, status)


def _ptr(t):
    if t is None:
        return None
    return _vp(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return _vp(s.cuda_stream)


def _need(cond, msg):
    if not cond:
        raise ValueError(msg)


def _is_fp8(t):
    return t.dtype in (torch.uint8, torch.float8_e4m3fn)


def _cuda_contig(*ts):
    for t in ts:
        if t is not None:
            _need(t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors")


def align4(x: int) -> int:
    return (x + 3) // 4 * 4


# ----------------------------------------------------------------- quantiser
def dg_quantize_fp8(x, mode, codes=None, scales=None, ld_scales=None, stream=None):
    """x: [rows, cols] or [batch, rows, cols], float32 or bfloat16 (CUDA).
    Returns (codes uint8 like x, scales float32) in the layout of ``mode``."""
    _cuda_contig(x)
    _need(x.dtype in (torch.float32, torch.bfloat16), "x must be float32 or bfloat16")
    squeeze = x.dim() == 2
    batch, rows, cols = (1, *x.shape) if squeeze else tuple(x.shape)
    if mode == DG_QUANT_ROW_1x128:
        ld = align4(rows) if ld_scales is None else int(ld_scales)
        sshape = (batch, cols // 128, ld)
    elif mode == DG_QUANT_BLOCK_128x128:
        ld = 0
        sshape = (batch, (rows + 127) // 128, (cols + 127) // 128)
    elif mode == DG_QUANT_COL_128x1:
        ld = 0
        sshape = (batch, rows // 128, cols)
    else:
        raise ValueError(f"bad mode {mode}")
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.zeros(sshape[1:] if squeeze else sshape, dtype=torch.float32,
                             device=x.device)
    _cuda_contig(codes, scales)
    _need(_is_fp8(codes) and codes.shape == x.shape, "codes shape/dtype")
    _need(scales.dtype == torch.float32 and scales.numel() >= batch * sshape[1] * sshape[2],
          "scales too small")
    dt = DG_IN_BF16 if x.dtype == torch.bfloat16 else DG_IN_F32
    _check("dg_quantize_fp8", _lib.dg_quantize_fp8(_ptr(x), dt, batch, rows, cols, int(mode),
                                                   _ptr(codes), _ptr(scales), ld, _stream(stream)))
    return codes, scales


# ----------------------------------------------------------------- GEMMs
def dg_fp8_gemm_nt(A, sfa, B, sfb, C, D, stream=None):
    """D = C + A @ B.T. A [M,K] e4m3, sfa [K/128, align4(M)] f32, B [N,K] e4m3,
    sfb [ceil(N/128), K/128] f32, C [M,N] bf16 or None, D [M,N] bf16."""
    _cuda_contig(A, sfa, B, sfb, C, D)
    M, K = A.shape
    N = B.shape[0]
    _need(_is_fp8(A) and _is_fp8(B) and B.shape[1] == K, "A/B")
    _need(D.dtype == torch.bfloat16 and tuple(D.shape) == (M, N), "D")
    _need(C is None or (C.dtype == torch.bfloat16 and tuple(C.shape) == (M, N)), "C")
    _need(sfa.dtype == torch.float32 and sfa.numel() >= (K // 128) * align4(M), "sfa")
    _need(sfb.dtype == torch.float32 and sfb.numel() >= ((N + 127) // 128) * (K // 128), "sfb")
    _check("dg_fp8_gemm_nt", _lib.dg_fp8_gemm_nt(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(C),
                                                 _ptr(D), M, N, K, _stream(stream)))
    return D


def dg_m_grouped_fp8_gemm_nt_contiguous(A, sfa, B, sfb, m_indices, C, D, stream=None):
    """A [Mt,K], sfa [K/128, align4(Mt)], B [G,N,K], sfb [G, ceil(N/128), K/128],
    m_indices [Mt] int32 (-1 = padding), C [Mt,N] bf16 or None, D [Mt,N] bf16."""
    _cuda_contig(A, sfa, B, sfb, m_indices, C, D)
    Mt, K = A.shape
    G, N, K2 = B.shape
    _need(_is_fp8(A) and _is_fp8(B) and K2 == K, "A/B")
    _need(m_indices.dtype == torch.int32 and m_indices.numel() == Mt, "m_indices")
    _need(D.dtype == torch.bfloat16 and tuple(D.shape) == (Mt, N), "D")
    _need(C is None or (C.dtype == torch.bfloat16 and tuple(C.shape) == (Mt, N)), "C")
    _need(sfa.dtype == torch.float32 and sfa.numel() >= (K // 128) * align4(Mt), "sfa")
    _need(sfb.dtype == torch.float32 and sfb.numel() >= G * ((N + 127) // 128) * (K // 128),
          "sfb")
    _check("dg_m_grouped_fp8_gemm_nt_contiguous",
           _lib.dg_m_grouped_fp8_gemm_nt_contiguous(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb),
                                                    _ptr(m_indices), _ptr(C), _ptr(D), Mt, N, K,
                                                    G, _stream(stream)))
    return D


def dg_m_grouped_fp8_gemm_nt_masked(A, sfa, B, sfb, masked_m, D, expected_m=None, stream=None):
    """A [G,max_m,K], sfa [G, K/128, align4(max_m)], B [G,N,K],
    sfb [G, ceil(N/128), K/128], masked_m [G] int32, D [G,max_m,N] bf16.
    expected_m: optional host hint of the typical valid rows per group (plans
    the tile width only; None = plan for max_m)."""
    _cuda_contig(A, sfa, B, sfb, masked_m, D)
    G, max_m, K = A.shape
    G2, N, K2 = B.shape
    _need(_is_fp8(A) and _is_fp8(B) and K2 == K and G2 == G, "A/B")
    _need(masked_m.dtype == torch.int32 and masked_m.numel() == G, "masked_m")
    _need(D.dtype == torch.bfloat16 and tuple(D.shape) == (G, max_m, N), "D")
    _need(sfa.dtype == torch.float32 and sfa.numel() >= G * (K // 128) * align4(max_m), "sfa")
    _need(sfb.dtype == torch.float32 and sfb.numel() >= G * ((N + 127) // 128) * (K // 128),
          "sfb")
    _check("dg_m_grouped_fp8_gemm_nt_masked",
           _lib.dg_m_grouped_fp8_gemm_nt_masked(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb),
                                                _ptr(masked_m), _ptr(D), G, max_m,
                                                int(expected_m or 0), N, K, _stream(stream)))
    return D


def dg_k_grouped_fp8_gemm_tn_contiguous(A, sfa, B, sfb, ks, C, D, stream=None):
    """A [sumK, M], sfa [sumK/128, M], B [sumK, N], sfb [sumK/128, N] (all CUDA),
    ks: host list of per-group K, C [G,M,N] f32 or None, D [G,M,N] f32."""
    _cuda_contig(A, sfa, B, sfb, C, D)
    ks = [int(k) for k in ks]
    G = len(ks)
    sumK, M = A.shape
    N = B.shape[1]
    _need(_is_fp8(A) and _is_fp8(B) and B.shape[0] == sumK and sum(ks) == sumK, "A/B/ks")
    _need(D.dtype == torch.float32 and tuple(D.shape) == (G, M, N), "D")
    _need(C is None or (C.dtype == torch.float32 and tuple(C.shape) == (G, M, N)), "C")
    _need(sfa.dtype == torch.float32 and sfa.numel() >= (sumK // 128) * M, "sfa")
    _need(sfb.dtype == torch.float32 and sfb.numel() >= (sumK // 128) * N, "sfb")
    ks_arr = (_C.c_int * max(G, 1))(*ks)
    _check("dg_k_grouped_fp8_gemm_tn_contiguous",
           _lib.dg_k_grouped_fp8_gemm_tn_contiguous(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), ks_arr,
                                                    _ptr(C), _ptr(D), G, M, N, _stream(stream)))
    return D


def _dense_layout(name, a_mn, b_mn, A, sfa, B, sfb, C, D, stream):
    _cuda_contig(A, sfa, B, sfb, C, D)
    _need(_is_fp8(A) and _is_fp8(B), "A/B must be E4M3 bytes")
    K, M = A.shape if a_mn else A.shape[::-1]
    N = B.shape[1] if b_mn else B.shape[0]
    _need((B.shape[0] if b_mn else B.shape[1]) == K, "A/B K mismatch")
    _need(D.dtype == torch.bfloat16 and tuple(D.shape) == (M, N), "D must be bf16 [M, N]")
    _need(C is None or (C.dtype == torch.bfloat16 and tuple(C.shape) == (M, N)), "C")
    _need(sfa.dtype == torch.float32 and sfa.numel() >= (K // 128) * (M if a_mn else align4(M)),
          "sfa")
    _need(sfb.dtype == torch.float32 and sfb.numel() >= (K // 128) * ((N + 127) // 128), "sfb")
    _check(name, getattr(_lib, name)(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(C), _ptr(D),
                                     M, N, K, _stream(stream)))
    return D


def dg_fp8_gemm_nn(A, sfa, B, sfb, C, D, stream=None):
    """A [M, K], sfa [K/128, align4(M)]; B [K, N], sfb [K/128, ceil(N/128)]."""
    return _dense_layout("dg_fp8_gemm_nn", False, True, A, sfa, B, sfb, C, D, stream)


def dg_fp8_gemm_tn(A, sfa, B, sfb, C, D, stream=None):
    """A [K, M], sfa [K/128, M]; B [K, N], sfb [K/128, ceil(N/128)]."""
    return _dense_layout("dg_fp8_gemm_tn", True, True, A, sfa, B, sfb, C, D, stream)


def dg_fp8_gemm_tt(A, sfa, B, sfb, C, D, stream=None):
    """A [K, M], sfa [K/128, M]; B [N, K], sfb [ceil(N/128), K/128]."""
    return _dense_layout("dg_fp8_gemm_tt", True, False, A, sfa, B, sfb, C, D, stream)


def ue8m0_packed_shape(rows: int, cols: int):
    """Shape of the packed UE8M0 scale tensor (int32) of a [rows, cols] operand."""
    return ((cols + 511) // 512, (rows + 127) // 128, 32, 4)


def dg_quantize_fp8_ue8m0(x, mode, codes=None, scales=None, packed=None, with_scales=True,
                          stream=None):
    """x [rows, cols] f32/bf16 CUDA; mode DG_QUANT_ROW_1x128 or DG_QUANT_BLOCK_128x128.
    Power-of-two scales. Returns (codes, FP32 scales or None, packed UE8M0 int32)."""
    _cuda_contig(x, codes, scales, packed)
    _need(x.dim() == 2, "x must be 2-D")
    rows, cols = x.shape
    _need(mode in (DG_QUANT_ROW_1x128, DG_QUANT_BLOCK_128x128), "mode")
    dt = DG_IN_BF16 if x.dtype == torch.bfloat16 else DG_IN_F32
    _need(x.dtype in (torch.float32, torch.bfloat16), "x dtype")
    if codes is None:
        codes = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    ld = 0
    if with_scales and scales is None:
        if mode == DG_QUANT_ROW_1x128:
            scales = torch.zeros((cols // 128, align4(rows)), dtype=torch.float32, device=x.device)
        else:
            scales = torch.zeros(((rows + 127) // 128, cols // 128), dtype=torch.float32,
                                 device=x.device)
    if scales is not None and mode == DG_QUANT_ROW_1x128:
        ld = scales.shape[-1]
    if packed is None:
        packed = torch.zeros(ue8m0_packed_shape(rows, cols), dtype=torch.int32, device=x.device)
    _need(packed.dtype == torch.int32 and packed.numel() >= math.prod(ue8m0_packed_shape(rows, cols)),
          "packed")
    _check("dg_quantize_fp8_ue8m0",
           _lib.dg_quantize_fp8_ue8m0(_ptr(x), dt, rows, cols, mode, _ptr(codes), _ptr(scales), ld,
                                      _ptr(packed), _stream(stream)))
    return codes, scales, packed


def dg_fp8_gemm_nt_ue8m0(A, sfa_packed, B, sfb_packed, C, D, stream=None):
    """D = C + A @ B.T on the block-scaled MMA with packed UE8M0 scales."""
    _cuda_contig(A, sfa_packed, B, sfb_packed, C, D)
    M, K = A.shape
    N = B.shape[0]
    _need(_is_fp8(A) and _is_fp8(B) and B.shape[1] == K, "A/B")
    _need(D.dtype == torch.bfloat16 and tuple(D.shape) == (M, N), "D")
    _need(C is None or (C.dtype == torch.bfloat16 and tuple(C.shape) == (M, N)), "C")
    _need(sfa_packed.dtype == torch.int32 and
          sfa_packed.numel() >= math.prod(ue8m0_packed_shape(M, K)), "sfa_packed")
    _need(sfb_packed.dtype == torch.int32 and
          sfb_packed.numel() >= math.prod(ue8m0_packed_shape(N, K)), "sfb_packed")
    _check("dg_fp8_gemm_nt_ue8m0",
           _lib.dg_fp8_gemm_nt_ue8m0(_ptr(A), _ptr(sfa_packed), _ptr(B), _ptr(sfb_packed), _ptr(C),
                                     _ptr(D), M, N, K, _stream(stream)))
    return D


def fp4_packed_shape(rows: int, cols: int):
    """Shape of the packed UE8M0 scale tensor (int32) of a [rows, cols] FP4
    operand: one byte per (row, 32-column strip), four strips per word."""
    return ((cols + 127) // 128, (rows + 127) // 128, 32, 4)


def dg_quantize_fp4_e2m1(x, codes=None, scales=None, packed=None, with_scales=True, stream=None):
    """x [rows, cols] f32/bf16 CUDA, cols % 128 == 0. Returns (codes uint8
    [rows, cols/2] packed E2M1, FP32 scales [rows, cols/32] or None, packed
    UE8M0 int32 [cols/128, ceil(rows/128), 32, 4])."""
    _cuda_contig(x, codes, scales, packed)
    _need(x.dim() == 2, "x must be 2-D")
    rows, cols = x.shape
    _need(x.dtype in (torch.float32, torch.bfloat16), "x dtype")
    dt = DG_IN_BF16 if x.dtype == torch.bfloat16 else DG_IN_F32
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    _need(codes.dtype == torch.uint8 and codes.numel() >= rows * (cols // 2), "codes")
    if with_scales and scales is None:
        scales = torch.zeros((rows, cols // 32), dtype=torch.float32, device=x.device)
    if packed is None:
        packed = torch.zeros(fp4_packed_shape(rows, cols), dtype=torch.int32, device=x.device)
    _need(packed.dtype == torch.int32 and packed.numel() >= math.prod(fp4_packed_shape(rows, cols)),
          "packed")
    _check("dg_quantize_fp4_e2m1",
           _lib.dg_quantize_fp4_e2m1(_ptr(x), dt, rows, cols, _ptr(codes), _ptr(scales),
                                     _ptr(packed), _stream(stream)))
    return codes, scales, packed


def dg_fp8_fp4_gemm_nt(A, sfa_packed, B, sfb_packed, C, D, stream=None):
    """D = C + A @ B.T, A E4M3 [M, K] with packed UE8M0 1x128 scales (from
    dg_quantize_fp8_ue8m0, ROW mode), B packed E2M1 uint8 [N, K/2] with packed
    1x32 scales (from dg_quantize_fp4_e2m1)."""
    _cuda_contig(A, sfa_packed, B, sfb_packed, C, D)
    M, K = A.shape
    N = B.shape[0]
    _need(_is_fp8(A) and B.dtype == torch.uint8 and B.shape[1] * 2 == K, "A/B")
    _need(D.dtype == torch.bfloat16 and tuple(D.shape) == (M, N), "D")
    _need(C is None or (C.dtype == torch.bfloat16 and tuple(C.shape) == (M, N)), "C")
    _need(sfa_packed.dtype == torch.int32 and
          sfa_packed.numel() >= math.prod(ue8m0_packed_shape(M, K)), "sfa_packed")
    _need(sfb_packed.dtype == torch.int32 and
          sfb_packed.numel() >= math.prod(fp4_packed_shape(N, K)), "sfb_packed")
    _check("dg_fp8_fp4_gemm_nt",
           _lib.dg_fp8_fp4_gemm_nt(_ptr(A), _ptr(sfa_packed), _ptr(B), _ptr(sfb_packed), _ptr(C),
                                   _ptr(D), M, N, K, _stream(stream)))
    return D


def dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(A, sfa, B, sfb, ks_dev, C, D, stream=None):
    """As dg_k_grouped_fp8_gemm_tn_contiguous, with the per-group K sizes in a
    CUDA int32 tensor ks_dev [G] (read on the device); A/B hold k_capacity =
    A.shape[0] rows."""
    _cuda_contig(A, sfa, B, sfb, ks_dev, C, D)
    G = ks_dev.numel()
    kcap, M = A.shape
    N = B.shape[1]
    _need(ks_dev.dtype == torch.int32, "ks_dev must be int32")
    _need(_is_fp8(A) and _is_fp8(B) and B.shape[0] == kcap, "A/B")
    _need(D.dtype == torch.float32 and tuple(D.shape) == (G, M, N), "D")
    _need(C is None or (C.dtype == torch.float32 and tuple(C.shape) == (G, M, N)), "C")
    _need(sfa.dtype == torch.float32 and sfa.numel() >= (kcap // 128) * M, "sfa")
    _need(sfb.dtype == torch.float32 and sfb.numel() >= (kcap // 128) * N, "sfb")
    _check("dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks",
           _lib.dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(
               _ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(ks_dev), kcap, _ptr(C), _ptr(D), G, M, N,
               _stream(stream)))
    return D


# ----------------------------------------------------------------- utilities
def dg_get_mk_alignment_for_contiguous_layout() -> int:
    return _lib.dg_get_mk_alignment_for_contiguous_layout()


def dg_get_tma_aligned_size(mn: int, elem_bytes: int) -> int:
    return _lib.dg_get_tma_aligned_size(int(mn), int(elem_bytes))


def dg_set_num_sms(n: int) -> None:
    _lib.dg_set_num_sms(int(n))


def dg_get_num_sms() -> int:
    return _lib.dg_get_num_sms()


def dg_set_wait_timeout_ns(ns: int) -> None:
    _lib.dg_set_wait_timeout_ns(int(ns))


def dg_get_last_device_error(stream=None):
    """Synchronises the stream; returns (status, site) and clears the word."""
    site = _C.c_int(0)
    st = _lib.dg_get_last_device_error(_stream(stream), _C.byref(site))
    return st, site.value


def dg_debug_drop_next_arrive(enable: bool = True) -> None:
    _lib.dg_debug_drop_next_arrive(1 if enable else 0)


def dg_get_launch_count() -> int:
    return int(_lib.dg_get_launch_count())


def dg_set_pdl(enable: bool) -> None:
    _lib.dg_set_pdl(1 if enable else 0)


def dg_get_pdl() -> bool:
    return bool(_lib.dg_get_pdl())
