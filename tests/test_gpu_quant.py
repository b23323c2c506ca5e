"""GPU quantiser vs the CPU oracle: codes and scales must match bit for bit."""
import zlib

import numpy as np
import pytest
import torch

import moe_grouped_gemm_07_b200 as dg
import oracle
import synth
from gpu_helpers import to_dev

pytestmark = pytest.mark.gpu

MODES = {
    "row": (dg.DG_QUANT_ROW_1x128, oracle.ROW_1x128),
    "block": (dg.DG_QUANT_BLOCK_128x128, oracle.BLOCK_128x128),
    "col": (dg.DG_QUANT_COL_128x1, oracle.COL_128x1),
}


def run_both(x, mode_name, bf16=False):
    gmode, omode = MODES[mode_name]
    if bf16:
        bits = synth.to_bf16_bits(x)
        xg = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        oc, osf = oracle.quantize(bits, omode, bf16=True)
    else:
        xg = to_dev(x)
        oc, osf = oracle.quantize(x, omode)
    gc, gsf = dg.dg_quantize_fp8(xg, gmode)
    torch.cuda.synchronize()
    return gc.cpu().numpy(), gsf.cpu().numpy(), oc, osf


def assert_bit_exact(gc, gsf, oc, osf):
    assert gc.shape == oc.shape and gsf.shape == osf.shape
    bad = np.nonzero(gc != oc)
    assert bad[0].size == 0, f"{bad[0].size} code mismatches, first at {[b[0] for b in bad]}"
    assert np.array_equal(gsf.view(np.uint32), osf.view(np.uint32)), "scale bits differ"


@pytest.mark.parametrize("mode", ["row", "block", "col"])
@pytest.mark.parametrize("shape", [(128, 128), (200, 384), (256, 1024), (3, 256, 512)])
def test_quant_random_bit_exact(mode, shape):
    if mode == "col" and shape[-2] % 128 != 0:
        pytest.skip("COL mode needs rows % 128 == 0")
    x = synth.normal(shape, synth.seed(70, zlib.crc32(repr((mode, shape)).encode()) % 997))
    assert_bit_exact(*run_both(x, mode))


@pytest.mark.parametrize("shape", [(200, 328), (7168, 2112), (3, 130, 196), (64, 4)])
@pytest.mark.parametrize("bf16", [False, True])
def test_quant_block_ragged_columns_bit_exact(shape, bf16):
    """BLOCK mode with cols % 128 != 0 (B stored [K][N] for NN / TN, e.g.
    N = 2112): the right-edge blocks cover only the existing columns."""
    x = synth.normal(shape, synth.seed(70, zlib.crc32(repr(("ragged", shape)).encode()) % 997))
    x[..., : min(128, shape[-1])] *= np.float32(50.0)   # an amax past a row's end would show
    assert_bit_exact(*run_both(x, "block", bf16=bf16))


@pytest.mark.parametrize("mode", ["row", "block", "col"])
def test_quant_bf16_bit_exact(mode):
    x = synth.normal((256, 512), synth.seed(71, 1))
    assert_bit_exact(*run_both(x, mode, bf16=True))


def test_quant_heavy_tails_and_zeros():
    """Mixed magnitudes (subnormal codes, exact ties, zero strips, -0)."""
    x = synth.normal((256, 512), synth.seed(72, 0))
    x[:, :128] *= 1e-3
    x[7] = 0.0
    x[9, 5] = -0.0
    x[11, 130:140] = np.float32(1e-30)
    x[3, ::3] *= 1e4
    for mode in ("row", "block", "col"):
        assert_bit_exact(*run_both(x, mode))


def test_encoder_exhaustive_via_unit_scale():
    """Strips whose amax is 448 have scale exactly 1, so the codes are the E4M3
    encoding of the inputs themselves: sweep every E4M3 midpoint and its float32
    neighbours (both signs) through the GPU encoder and compare with the oracle."""
    t = oracle.e4m3_table()
    pos = sorted(set(float(v) for v in t[:0x7F]))
    vals = []
    for a, b in zip(pos[:-1], pos[1:]):
        m = np.float32((a + b) / 2)
        vals += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9)), a, b]
    vals = np.array(vals, dtype=np.float32)
    vals = np.concatenate([vals, -vals, np.float32([0.0, -0.0, 1e-30, -1e-30])])
    n_per = 127
    strips = (vals.size + n_per - 1) // n_per
    x = np.zeros((strips, 128), dtype=np.float32)
    x[:, 0] = 448.0
    flat = np.zeros(strips * n_per, dtype=np.float32)
    flat[:vals.size] = vals
    x[:, 1:] = flat.reshape(strips, n_per)
    gc, gsf, oc, osf = run_both(x, "row")
    assert np.all(osf[0, :strips] == 1.0)
    assert_bit_exact(gc, gsf, oc, osf)


def test_quant_large_row_mode():
    """One full-size activation (M=4096, K=7168) on sampled rows."""
    x = synth.normal((4096, 7168), synth.seed(2, 12, 0))
    xg = to_dev(x)
    gc, gsf = dg.dg_quantize_fp8(xg, dg.DG_QUANT_ROW_1x128)
    rows = np.arange(0, 4096, 97)
    oc, osf = oracle.quantize(x[rows], oracle.ROW_1x128)
    gcn = gc.cpu().numpy()[rows]
    gsn = gsf.cpu().numpy()[:, rows]
    assert np.array_equal(gcn, oc)
    assert np.array_equal(gsn.view(np.uint32), osf[:, :rows.size].view(np.uint32))


def test_quant_rejects_bad_shapes():
    x = torch.zeros((128, 100), device="cuda")
    with pytest.raises(dg.DGError) as e:
        dg.dg_quantize_fp8(x, dg.DG_QUANT_ROW_1x128)
    assert e.value.status == dg.DG_ERR_UNSUPPORTED_SHAPE


def test_quotient_near_rounding_boundaries():
    """Every strip gets a random amax (so a random scale s), and its other 127
    values sit within a few float32 ulps of s times an E4M3 rounding boundary
    (a midpoint between neighbouring codes), either sign. The codes must match
    the oracle, which divides with IEEE float division."""
    t = oracle.e4m3_table()
    pos = np.array(sorted(set(float(v) for v in t[:0x7F])))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    strips = 8192
    u = synth.u64(strips * 130, synth.seed(73, 1))
    amax = np.ldexp(0.5 + (u[:strips] >> np.uint64(11)).astype(np.float64) / 2.0 ** 53,
                    (u[strips:2 * strips] % np.uint64(50)).astype(np.int64) - 30).astype(np.float32)
    amax[::97] = np.float32(3e-5)              # below the 1e-4 floor
    s = (np.maximum(amax, np.float32(1e-4)) / np.float32(448.0)).astype(np.float32)
    pick = (u[2 * strips:2 * strips + strips * 127] % np.uint64(mids.size)).astype(np.int64)
    base = (mids[pick].reshape(strips, 127) * s[:, None]).astype(np.float32)
    nudge = (u[:strips * 127] % np.uint64(9)).astype(np.int64).reshape(strips, 127) - 4
    bits = base.view(np.int32) + nudge.astype(np.int32)
    vals = bits.view(np.float32)
    vals = np.minimum(vals, amax[:, None])      # keep amax the strip maximum
    sign = np.where((u[:strips * 127] >> np.uint64(7)) & np.uint64(1), -1.0, 1.0).astype(np.float32)
    x = np.empty((strips, 128), dtype=np.float32)
    x[:, 0] = amax
    x[:, 1:] = vals * sign.reshape(strips, 127)
    gc, gsf, oc, osf = run_both(x, "row")
    assert_bit_exact(gc, gsf, oc, osf)
