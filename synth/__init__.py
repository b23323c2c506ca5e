"""Seeded synthetic inputs for tests and the benchmark.

Holds no GEMM or quantiser arithmetic: a counter-based SplitMix64 stream plus
the Box-Muller transform, compiled from ``synth.c``. The same arrays feed both
the CUDA library and the CPU oracle. Seeds follow one rule: workload ``c``,
shape ``i``, tensor ``t`` uses ``seed(c, i, t) = 1_000_000 * c + 1000 * i + t``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(HERE, "synth.c")
_OUT = os.path.join(HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_OUT) or os.path.getmtime(_OUT) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-march=x86-64-v2", "-fPIC", "-shared", "-fopenmp",
                               "-ffp-contract=off", "-std=c11", _SRC, "-o", _OUT + ".tmp", "-lm"])
        os.replace(_OUT + ".tmp", _OUT)
    return _OUT


def _L():
    global _lib
    if _lib is None:
        L = C.CDLL(build())
        L.synth_u64.argtypes = [C.c_uint64, C.c_uint64, C.c_void_p, C.c_size_t]
        L.synth_normal_f32.argtypes = [C.c_uint64, C.c_uint64, C.c_void_p, C.c_size_t]
        L.synth_randint.argtypes = [C.c_uint64, C.c_uint64, C.c_int64, C.c_int64, C.c_void_p,
                                    C.c_size_t]
        _lib = L
    return _lib


def seed(config: int, shape: int = 0, tensor: int = 0) -> int:
    return 1_000_000 * config + 1000 * shape + tensor


def normal(shape, seed: int, offset: int = 0) -> np.ndarray:
    """float32 N(0,1) array of the given shape."""
    out = np.empty(shape, dtype=np.float32)
    _L().synth_normal_f32(seed, offset, out.ctypes.data_as(C.c_void_p), out.size)
    return out


def u64(n: int, seed: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _L().synth_u64(seed, offset, out.ctypes.data_as(C.c_void_p), n)
    return out


def randint(lo: int, hi: int, n: int, seed: int, offset: int = 0) -> np.ndarray:
    """int64 array of n integers uniform in [lo, hi]."""
    out = np.empty(n, dtype=np.int64)
    _L().synth_randint(seed, offset, lo, hi, out.ctypes.data_as(C.c_void_p), n)
    return out


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round-to-nearest-even, via torch) and return
    the raw uint16 bit patterns. Used to give both sides the same bf16 C."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
