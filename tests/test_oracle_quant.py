"""Pins for the oracle's quantiser (CPU only).

What is pinned and by what:
  * scale placement per mode: inputs whose every strip/block has a distinct,
    known amax, so the expected scale at each position is a closed form;
  * codes: strips that contain 448 give scale == 1 exactly, so the codes must
    equal torch's float8_e4m3fn cast of the inputs (library routine);
  * the E4M3 rounding error bound on random data (half a unit in the last place
    of 3 mantissa bits, or half the subnormal step);
  * the amax element always lands on +-448;
  * all-zero strips (scale floor 1e-4/448, codes zero), ragged 128x128 blocks,
    bf16 inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

F32 = np.float32


def torch_e4m3(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=F32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def dequant_err_ok(x, codes, s):
    """|dec(code)*s - x| <= max(2^-4 |x|, 2^-10 s) (+ tiny slack for the fp32
    division x/s)."""
    tab = oracle.e4m3_table()
    deq = tab[codes] * s
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6) + 1e-30
    return np.all(np.abs(deq - x.astype(np.float64)) <= bound)


def test_row_scale_positions_closed_form():
    rows, cols = 37, 384
    x = np.zeros((rows, cols), dtype=F32)
    for r in range(rows):
        for kb in range(3):
            x[r, kb * 128 + (r * 7 + kb) % 128] = F32(1.0 + r + 1000 * kb)
    codes, sf = oracle.quantize(x, oracle.ROW_1x128)
    assert sf.shape == (3, 40)                     # ld rounded up to 4 floats
    for r in range(rows):
        for kb in range(3):
            assert sf[kb, r] == F32(F32(1.0 + r + 1000 * kb) / F32(448.0))
    assert np.all(sf[:, rows:] == 0)               # padding entries untouched


def test_block_scale_positions_ragged():
    rows, cols = 200, 256                          # second 128-row block has 72 rows
    x = np.zeros((rows, cols), dtype=F32)
    x[5, 3] = -3.0
    x[100, 200] = 7.0
    x[199, 10] = 11.0                              # last existing row of block 1
    x[150, 255] = -13.0
    codes, sf = oracle.quantize(x, oracle.BLOCK_128x128)
    assert sf.shape == (2, 2)
    assert sf[0, 0] == F32(F32(3.0) / F32(448.0))
    assert sf[0, 1] == F32(F32(7.0) / F32(448.0))
    assert sf[1, 0] == F32(F32(11.0) / F32(448.0))
    assert sf[1, 1] == F32(F32(13.0) / F32(448.0))


def test_col_scale_positions_closed_form():
    rows, cols = 256, 48
    x = np.zeros((rows, cols), dtype=F32)
    for rb in range(2):
        for c in range(cols):
            x[rb * 128 + (c * 5 + rb) % 128, c] = F32(2.0 + c + 100 * rb)
    codes, sf = oracle.quantize(x, oracle.COL_128x1)
    assert sf.shape == (2, cols)
    for rb in range(2):
        for c in range(cols):
            assert sf[rb, c] == F32(F32(2.0 + c + 100 * rb) / F32(448.0))


@pytest.mark.parametrize("mode", [oracle.ROW_1x128, oracle.BLOCK_128x128, oracle.COL_128x1])
def test_unit_scale_codes_match_torch_cast(mode):
    """Every strip/block holds 448 somewhere, so scale == 1 and code == cast(x)."""
    x = synth.normal((256, 256), 11) * F32(60.0)
    x = np.clip(x, -440, 440).astype(F32)
    if mode == oracle.ROW_1x128:
        x[:, 0] = 448.0
        x[:, 128] = -448.0
    elif mode == oracle.BLOCK_128x128:
        x[0, 0] = 448.0
        x[0, 128] = 448.0
        x[128, 0] = -448.0
        x[128, 128] = 448.0
    else:
        x[0, :] = 448.0
        x[128, :] = -448.0
    codes, sf = oracle.quantize(x, mode)
    used = sf[sf != 0]
    assert np.all(used == 1.0)
    assert np.array_equal(codes, torch_e4m3(x))


@pytest.mark.parametrize("mode", [oracle.ROW_1x128, oracle.BLOCK_128x128, oracle.COL_128x1])
def test_error_bound_random(mode):
    x = synth.normal((256, 384), 12)
    codes, sf = oracle.quantize(x, mode)
    if mode == oracle.ROW_1x128:
        s = np.repeat(sf[:, :256].T, 128, axis=1)          # [rows, cols]
    elif mode == oracle.BLOCK_128x128:
        s = np.repeat(np.repeat(sf, 128, axis=0), 128, axis=1)[:256, :384]
    else:
        s = np.repeat(sf, 128, axis=0)
    assert s.shape == x.shape
    assert dequant_err_ok(x, codes, s.astype(np.float64))


def test_amax_element_maps_to_448():
    x = synth.normal((64, 512), 13)
    codes, sf = oracle.quantize(x, oracle.ROW_1x128)
    tab = oracle.e4m3_table()
    for r in range(64):
        for kb in range(4):
            strip = x[r, kb * 128:(kb + 1) * 128]
            j = int(np.argmax(np.abs(strip)))
            assert abs(tab[codes[r, kb * 128 + j]]) == 448.0


def test_zero_strip_floor():
    x = np.zeros((4, 256), dtype=F32)
    x[1, 130] = 5e-5                                # below the 1e-4 floor
    codes, sf = oracle.quantize(x, oracle.ROW_1x128)
    floor = F32(F32(1e-4) / F32(448.0))
    assert np.all(sf[:, :4] == floor)
    assert np.all(codes[0] == 0)
    # 5e-5 / (1e-4/448) = 224 -> exactly representable
    assert oracle.e4m3_table()[codes[1, 130]] == pytest.approx(224.0, rel=2 ** -4)


def test_bf16_input_matches_rounded_f32():
    x = synth.normal((128, 256), 14)
    xb = synth.to_bf16_bits(x)
    xr = synth.bf16_bits_to_f32(xb)
    c1, s1 = oracle.quantize(xb, oracle.ROW_1x128, bf16=True)
    c2, s2 = oracle.quantize(xr, oracle.ROW_1x128)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_batched_layout_equals_per_batch():
    x = synth.normal((3, 64, 256), 15)
    c, s = oracle.quantize(x, oracle.ROW_1x128)
    for b in range(3):
        cb, sb = oracle.quantize(x[b], oracle.ROW_1x128)
        assert np.array_equal(c[b], cb) and np.array_equal(s[b], sb)


# ------------------------------------------------------------ power-of-two (UE8M0) scales
def _strip_amax_rows(x):
    rows, cols = x.shape
    return np.abs(x).reshape(rows, cols // 128, 128).max(axis=2)


def test_pow2_row_scales_are_the_next_power_of_two():
    """s is a power of two with s/2 < t <= s for t = max(amax, 1e-4)/448 in
    float32 (closed form, checked with numpy's frexp, independent of the
    oracle's own rounding step)."""
    x = synth.normal((70, 512), synth.seed(9, 1, 0)) * F32(3.0)
    x[5, 128:256] = 0.0                        # floor strip
    x[6, :128] = 0.0
    x[6, 7] = 448.0                            # t == 1 exactly -> s == 1
    x[7, :128] = 0.0
    x[7, 3] = -449.0                           # t just above 1 -> s == 2
    codes, s = oracle.quantize(x, oracle.ROW_1x128_POW2)
    s = s[:, :70].T                            # [rows, kbs]
    t = np.maximum(_strip_amax_rows(x), F32(1e-4)).astype(F32) / F32(448.0)
    m, _ = np.frexp(s)
    assert np.all(m == 0.5)
    assert np.all(s >= t) and np.all(s / 2 < t)
    assert s[6, 0] == 1.0 and s[7, 0] == 2.0


def test_pow2_codes_equal_torch_cast_of_exact_quotient():
    """With s a power of two, x / s is exact, and |x / s| <= 448: the codes
    must equal torch's float8_e4m3fn cast (library routine) of x / s."""
    x = synth.normal((33, 384), synth.seed(9, 2, 0)) * F32(50.0)
    codes, s = oracle.quantize(x, oracle.ROW_1x128_POW2)
    sf = np.repeat(s[:, :33].T, 128, axis=1)   # [rows, cols]
    y = (x / sf).astype(F32)
    assert np.all(np.abs(y) <= 448.0)
    assert np.array_equal(codes, torch_e4m3(y))


def test_pow2_block_scales_ragged():
    rows, cols = 200, 256                      # 2 row blocks, the second has 72 rows
    x = synth.normal((rows, cols), synth.seed(9, 3, 0))
    codes, s = oracle.quantize(x, oracle.BLOCK_128x128_POW2)
    for nb in range(2):
        for kb in range(2):
            blk = x[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            t = F32(max(np.abs(blk).max(), F32(1e-4))) / F32(448.0)
            v = s[nb, kb]
            assert np.frexp(v)[0] == 0.5 and v >= t and v / 2 < t
            y = (blk / v).astype(F32)
            assert np.array_equal(codes[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128],
                                  torch_e4m3(y))


def test_pow2_scales_dequantise_within_bound():
    x = synth.normal((64, 256), synth.seed(9, 4, 0))
    codes, s = oracle.quantize(x, oracle.ROW_1x128_POW2)
    sf = np.repeat(s[:, :64].T, 128, axis=1)
    assert dequant_err_ok(x, codes, sf)
