"""Synthetic workload recipes (shapes, value distributions, group structure).

Holds no GEMM or quantiser arithmetic. Each recipe returns plain numpy inputs
(float32 operands, int32 index/count arrays) drawn from the seeded streams in
``synth``; both the CUDA path and the CPU oracle quantise and multiply them
themselves.

Workloads (sizes from the benchmark configuration of the FP8 GEMM pages):
  1 dense NT      M=128 N=256 K=512, C = 0
  2 dense sweep   M in {64,128,4096} x (N,K) in DENSE_NK (18 shapes)
  3 contiguous    G=8 experts, N=4096, K=7168, rows_g ~ U[2048,6144] padded to 128
  4 masked        G=16, max_m=256, masked_m ~ U[64,256], (N,K) in MASKED_NK
  5 K-grouped TN  G=8, M=4096, N=7168, K_g ~ U[1024,8192] padded to 128, C ~ N(0,1)
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import normal, randint, seed

DENSE_M = (64, 128, 4096)
DENSE_NK = ((2112, 7168), (24576, 1536), (32768, 512), (7168, 16384), (4096, 7168), (7168, 2048))
MASKED_NK = ((4096, 7168), (7168, 2048))
ALIGN = 128


def align(x: int, a: int = ALIGN) -> int:
    return (x + a - 1) // a * a


def dense_shapes():
    """The 18 (M, N, K) shapes of the dense sweep, M fastest."""
    return [(m, n, k) for (n, k) in DENSE_NK for m in DENSE_M]


@dataclass
class Dense:
    M: int
    N: int
    K: int
    A: np.ndarray            # float32 [M, K]
    B: np.ndarray            # float32 [N, K]
    C: np.ndarray | None     # float32 [M, N] (rounded to bf16 by the caller) or None


def dense(M, N, K, cfg=1, shape=0, with_c=False) -> Dense:
    A = normal((M, K), seed(cfg, shape, 0))
    B = normal((N, K), seed(cfg, shape, 1))
    C = normal((M, N), seed(cfg, shape, 2)) if with_c else None
    return Dense(M, N, K, A, B, C)


@dataclass
class Contiguous:
    G: int
    N: int
    K: int
    rows: list                # real rows per expert
    m_indices: np.ndarray     # int32 [Mt], expert id or -1 on padding
    A: np.ndarray             # float32 [Mt, K]; padding rows are zero
    B: np.ndarray             # float32 [G, N, K]

    @property
    def Mt(self):
        return self.m_indices.size


def contiguous(G=8, N=4096, K=7168, lo=2048, hi=6144, cfg=3, shape=0, zero_pad=True) -> Contiguous:
    rows = [int(r) for r in randint(lo, hi, G, seed(cfg, shape, 3))]
    segs = [align(r) for r in rows]
    Mt = sum(segs)
    mi = np.full(Mt, -1, dtype=np.int32)
    off = 0
    for g, (r, s) in enumerate(zip(rows, segs)):
        mi[off:off + r] = g
        off += s
    A = normal((Mt, K), seed(cfg, shape, 0))
    if zero_pad:
        A[mi < 0] = 0.0
    B = normal((G, N, K), seed(cfg, shape, 1))
    return Contiguous(G, N, K, rows, mi, A, B)


@dataclass
class Masked:
    G: int
    max_m: int
    N: int
    K: int
    masked_m: np.ndarray      # int32 [G]
    A: np.ndarray             # float32 [G, max_m, K]
    B: np.ndarray             # float32 [G, N, K]


def masked(G=16, max_m=256, N=4096, K=7168, lo=64, hi=256, cfg=4, shape=0) -> Masked:
    mm = randint(lo, hi, G, seed(cfg, shape, 3)).astype(np.int32)
    A = normal((G, max_m, K), seed(cfg, shape, 0))
    B = normal((G, N, K), seed(cfg, shape, 1))
    return Masked(G, max_m, N, K, mm, A, B)


@dataclass
class KGrouped:
    G: int
    M: int
    N: int
    ks: list                  # per-group K (multiples of 128)
    A: np.ndarray             # float32 [sumK, M]; pad rows zero
    B: np.ndarray             # float32 [sumK, N]; pad rows zero
    C: np.ndarray             # float32 [G, M, N]

    @property
    def sumK(self):
        return sum(self.ks)


def k_grouped(G=8, M=4096, N=7168, lo=1024, hi=8192, cfg=5, shape=0, ks=None) -> KGrouped:
    if ks is None:
        raw = [int(k) for k in randint(lo, hi, G, seed(cfg, shape, 3))]
        ks = [align(k) for k in raw]
    else:
        raw = list(ks)
    sumK = sum(ks)
    A = normal((sumK, M), seed(cfg, shape, 0))
    B = normal((sumK, N), seed(cfg, shape, 1))
    off = 0
    for r, k in zip(raw, ks):
        A[off + r:off + k] = 0.0
        B[off + r:off + k] = 0.0
        off += k
    C = normal((G, M, N), seed(cfg, shape, 2))
    return KGrouped(G, M, N, list(ks), A, B, C)
