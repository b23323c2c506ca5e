"""The seeded input generators (synth/) and the workload recipes built on
them, on the CPU: the SplitMix64 stream against its published outputs, the
counter-based sub-ranges, the Box-Muller pairing, the integer range, and the
group structure of the five benchmark configurations (at small N and K: the
counts come from their own streams, so they are the full-size counts)."""
import math

import numpy as np

import synth
import synth.workloads as wl

M64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15


def splitmix64(seed, n):
    """The generator as published (Steele, Lea & Flood, OOPSLA 2014; Vigna's
    constants): state += golden gamma, then the variant-13 finaliser."""
    out, x = [], seed & M64
    for _ in range(n):
        x = (x + GOLDEN) & M64
        z = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_published_outputs():
    # the first outputs of SplitMix64 seeded with 0, as its reference code prints them
    assert [int(v) for v in synth.u64(3, 0)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                                0x06C45D188009454F]
    for s in (1, 12345, synth.seed(5, 2, 1)):
        assert [int(v) for v in synth.u64(64, s)] == splitmix64(s, 64)


def test_streams_are_counter_based():
    s = synth.seed(3, 0, 0)
    full = synth.u64(1000, s)
    assert np.array_equal(synth.u64(100, s, offset=450), full[450:550])
    z = synth.normal((1000,), s)
    assert np.array_equal(synth.normal((37,), s, offset=500), z[500:537])
    assert np.array_equal(synth.normal((3, 4), 7), synth.normal((12,), 7).reshape(3, 4))


def test_box_muller_pairs():
    """Elements 2p and 2p+1 are r cos(2 pi u2) and r sin(2 pi u2) of one pair
    of counters: their squares sum to -2 ln(1 - u1)."""
    s = 99
    z = synth.normal((2000,), s).astype(np.float64)
    u = synth.u64(2000, s)
    u1 = (u[0::2] >> np.uint64(11)).astype(np.float64) / 2.0 ** 53
    r2 = -2.0 * np.log(1.0 - u1)
    assert np.allclose(z[0::2] ** 2 + z[1::2] ** 2, r2, rtol=1e-6, atol=1e-6)


def test_normal_moments():
    z = synth.normal((1 << 20,), synth.seed(1, 0, 0)).astype(np.float64)
    n = z.size
    assert abs(z.mean()) < 5 / math.sqrt(n)
    assert abs(z.std() - 1.0) < 5 / math.sqrt(2 * n)
    assert abs(np.mean(np.abs(z) > 1.959964) - 0.05) < 0.002     # two-sided 5% tail


def test_randint_inclusive_range_and_uniformity():
    v = synth.randint(64, 256, 200000, 5)
    assert v.min() == 64 and v.max() == 256
    counts = np.bincount(v - 64, minlength=193)
    exp = v.size / 193
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    assert chi2 < 192 + 6 * math.sqrt(2 * 192)                   # 192 degrees of freedom


def test_dense_sweep_shapes():
    sh = wl.dense_shapes()
    assert len(sh) == 18 and len(set(sh)) == 18
    assert {m for m, _, _ in sh} == {64, 128, 4096}
    assert {(n, k) for _, n, k in sh} == set(wl.DENSE_NK)
    assert all(k % 128 == 0 and n % 8 == 0 for _, n, k in sh)


def test_contiguous_recipe():
    """8 experts, rows ~ U[2048, 6144] (0.5x to 1.5x of 4096), each segment
    padded to a multiple of 128 with m_indices -1 and zero rows of A."""
    w = wl.contiguous(N=16, K=128)
    assert w.G == 8 and len(w.rows) == 8
    assert all(2048 <= r <= 6144 for r in w.rows)
    off = 0
    for g, r in enumerate(w.rows):
        seg = wl.align(r)
        assert np.all(w.m_indices[off:off + r] == g)
        assert np.all(w.m_indices[off + r:off + seg] == -1)
        assert not np.any(w.A[off + r:off + seg])
        off += seg
    assert off == w.Mt and w.Mt % 128 == 0
    # the counts do not depend on N and K: these are the full-size workload's
    assert wl.contiguous(N=32, K=256).rows == w.rows


def test_masked_recipe():
    for i, (N, K) in enumerate(wl.MASKED_NK):
        w = wl.masked(N=16, K=128, shape=i)
        assert w.G == 16 and w.max_m == 256
        assert w.masked_m.dtype == np.int32
        assert np.all((w.masked_m >= 64) & (w.masked_m <= 256))
        assert np.array_equal(wl.masked(N=N // 64, K=256, shape=i).masked_m, w.masked_m)


def test_k_grouped_recipe():
    """8 groups, K_g ~ U[1024, 8192] rounded up to 128 with zero pad rows in
    both operands, C ~ N(0, 1)."""
    w = wl.k_grouped(M=16, N=32)
    assert w.G == 8 and len(w.ks) == 8
    assert all(k % 128 == 0 and 1024 <= k <= 8192 for k in w.ks)
    raw = [int(k) for k in synth.randint(1024, 8192, 8, synth.seed(5, 0, 3))]
    assert w.ks == [wl.align(k) for k in raw]
    off = 0
    for r, k in zip(raw, w.ks):
        assert not np.any(w.A[off + r:off + k]) and not np.any(w.B[off + r:off + k])
        assert np.all(np.any(w.A[off:off + r] != 0, axis=1))
        off += k
    assert off == w.sumK and w.C.shape == (8, 16, 32)
