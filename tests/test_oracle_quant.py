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
    bf16 inputs;
  * the quotient itself, in all three modes: scales recomputed with numpy's
    float32 division and codes equal to torch's cast of numpy's float32 x / s
    (clipped to +-448), on N(0,1) data, heavy tails and zeros, and values on
    s x midpoint rounding boundaries where multiplying by 1 / s instead would
    change codes (the case set checks that it does).
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


def test_block_scale_positions_ragged_columns():
    """Blocks at the right edge (cols % 128 != 0) take their amax over the
    columns that exist, as blocks at the bottom edge do over their rows."""
    rows, cols = 200, 328                          # last column block has 72 columns
    x = np.zeros((rows, cols), dtype=F32)
    x[5, 300] = -3.0                               # block (0, 2)
    x[127, 327] = 5.0                              # block (0, 2), its last column: the amax
    x[150, 256] = -13.0                            # block (1, 2), its first column: the amax
    x[199, 327] = 11.0                             # block (1, 2), its last row and column
    x[64, 100] = 2.0                               # block (0, 0)
    codes, sf = oracle.quantize(x, oracle.BLOCK_128x128)
    assert sf.shape == (2, 3)
    assert sf[0, 0] == F32(F32(2.0) / F32(448.0))
    assert sf[0, 2] == F32(F32(5.0) / F32(448.0))
    assert sf[1, 2] == F32(F32(13.0) / F32(448.0))
    floor = F32(F32(1e-4) / F32(448.0))            # all-zero blocks
    assert sf[0, 1] == floor and sf[1, 0] == floor and sf[1, 1] == floor
    for (r, c), (br, bc) in {(5, 300): (0, 2), (127, 327): (0, 2), (150, 256): (1, 2),
                             (199, 327): (1, 2), (64, 100): (0, 0)}.items():
        assert codes[r, c] == torch_e4m3(np.array([x[r, c] / sf[br, bc]], dtype=F32))[0]


def test_block_quantisation_commutes_with_transpose():
    """A 128x128 block of x holds the same elements as the transposed block of
    x.T, so BLOCK quantisation of x.T is the transpose of that of x: ragged
    columns of one are ragged rows of the other."""
    x = synth.normal((200, 328), synth.seed(9, 13, 0))
    codes, sf = oracle.quantize(x, oracle.BLOCK_128x128)
    codes_t, sf_t = oracle.quantize(np.ascontiguousarray(x.T), oracle.BLOCK_128x128)
    assert sf.shape == (2, 3) and sf_t.shape == (3, 2)
    assert np.array_equal(sf.view(np.uint32), sf_t.T.view(np.uint32))
    assert np.array_equal(codes, codes_t.T)


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


# ------------------------------------------------------------ the quotient x / s
# The scale rule fixes s = max(amax, 1e-4) / 448 and code = E4M3_RN_sat(x / s),
# both IEEE float32 divisions. These pins recompute s and the quotient with
# numpy's float32 division (IEEE round-to-nearest) and encode with torch's
# float8_e4m3fn cast (a library routine), after clipping to +-448 as the
# saturating encoder does; neither side shares code with the oracle.
def _groups_to_layout(g, mode, n_groups):
    """g [n_groups, 128 * 128 or 128]: one quantisation group per row, element
    0 first. Returns x laid out so that every group is one strip (ROW), one
    128x128 block (BLOCK) or one 128-row column strip (COL)."""
    if mode == oracle.ROW_1x128:
        return g.reshape(n_groups, 128)
    if mode == oracle.COL_128x1:
        return np.ascontiguousarray(g.reshape(n_groups, 128).T)
    # BLOCK: n_groups blocks side by side along the columns
    return np.ascontiguousarray(g.reshape(n_groups, 128, 128).transpose(1, 0, 2).reshape(128, -1))


def _numpy_scales(x, mode):
    """Element-wise float32 scale of x under `mode`, computed in numpy."""
    rows, cols = x.shape
    a = np.abs(x)
    if mode == oracle.ROW_1x128:
        amax = a.reshape(rows, cols // 128, 128).max(axis=2)
        s = (np.maximum(amax, F32(1e-4)).astype(F32) / F32(448.0)).astype(F32)
        return np.repeat(s, 128, axis=1)
    if mode == oracle.COL_128x1:
        amax = a.reshape(rows // 128, 128, cols).max(axis=1)
        s = (np.maximum(amax, F32(1e-4)).astype(F32) / F32(448.0)).astype(F32)
        return np.repeat(s, 128, axis=0)
    nb, kb = (rows + 127) // 128, (cols + 127) // 128
    pad = np.zeros((nb * 128, kb * 128), dtype=F32)   # zeros never raise an amax
    pad[:rows, :cols] = a
    amax = pad.reshape(nb, 128, kb, 128).max(axis=(1, 3))
    s = (np.maximum(amax, F32(1e-4)).astype(F32) / F32(448.0)).astype(F32)
    return np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)[:rows, :cols]


def _expected_codes(x, s):
    y = (x.astype(F32) / s).astype(F32)              # IEEE float32 quotient
    return torch_e4m3(np.clip(y, F32(-448.0), F32(448.0)))


def _check_quotient(x, mode):
    codes, sf = oracle.quantize(x, mode)
    s = _numpy_scales(x, mode)
    if mode == oracle.ROW_1x128:
        got_s = np.repeat(sf[:, :x.shape[0]].T, 128, axis=1)
    elif mode == oracle.COL_128x1:
        got_s = np.repeat(sf, 128, axis=0)
    else:
        got_s = np.repeat(np.repeat(sf, 128, axis=0), 128, axis=1)[:x.shape[0], :x.shape[1]]
    assert np.array_equal(got_s.view(np.uint32), s.view(np.uint32))
    assert np.array_equal(codes, _expected_codes(x, s))


MODES3 = [oracle.ROW_1x128, oracle.BLOCK_128x128, oracle.COL_128x1]


@pytest.mark.parametrize("mode", MODES3)
def test_quotient_codes_random(mode):
    """N(0,1) data, a ragged 128x128 block in BLOCK mode (200 rows)."""
    rows = 200 if mode == oracle.BLOCK_128x128 else 256
    x = synth.normal((rows, 512), synth.seed(9, 10, mode))
    _check_quotient(x, mode)


def test_quotient_codes_ragged_block_columns():
    """BLOCK mode on 200 x 328: ragged blocks at both edges. The first column
    block is 50x larger, so an amax that strayed past the end of a row (into
    the next row's first columns) would change the edge blocks' scales."""
    x = synth.normal((200, 328), synth.seed(9, 14, 0))
    x[:, :128] *= F32(50.0)
    _check_quotient(x, oracle.BLOCK_128x128)


@pytest.mark.parametrize("mode", MODES3)
def test_quotient_codes_heavy_tails(mode):
    """Heavy tails and zeros: scales spread over many binades, strips under
    the 1e-4 floor, float32 subnormals, exact zeros and negative zeros."""
    u = (synth.u64(256 * 512, synth.seed(9, 11, mode)) >> np.uint64(11)).astype(np.float64)
    e = (np.floor(u / 2.0 ** 53 * 80.0) - 60.0).reshape(256, 512)   # binades 2^-60 .. 2^19
    x = (synth.normal((256, 512), synth.seed(9, 12, mode)) * np.ldexp(1.0, e.astype(np.int64))
         ).astype(F32)
    x[:, 0:128:3] = F32(0.0)
    x[:, 1:128:5] = F32(-0.0)
    x[7] = F32(0.0)                                     # all-zero row / strips
    x[9, :] = np.float32(1e-40)                         # float32 subnormals, under the floor
    x[11, 128:256] = F32(3e30)
    x[11, 130] = F32(1e-30)                             # underflows to a zero code
    _check_quotient(x, mode)


def _boundary_groups(n_groups, gsize, seed):
    """Groups whose element 0 is a random amax (so s is not a power of two)
    and whose other elements sit within four float32 ulps of s times an E4M3
    rounding boundary (a midpoint between neighbouring codes), either sign."""
    t = oracle.e4m3_table()
    pos = np.array(sorted(set(float(v) for v in t[:0x7F])))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(F32)
    n = n_groups * gsize
    u = synth.u64(3 * n + 2 * n_groups, seed)
    amax = np.ldexp(0.5 + (u[:n_groups] >> np.uint64(11)).astype(np.float64) / 2.0 ** 53,
                    (u[n_groups:2 * n_groups] % np.uint64(40)).astype(np.int64) - 20).astype(F32)
    s = (np.maximum(amax, F32(1e-4)) / F32(448.0)).astype(F32)
    r = u[2 * n_groups:]
    pick = (r[:n] % np.uint64(mids.size)).astype(np.int64).reshape(n_groups, gsize)
    base = (mids[pick] * s[:, None]).astype(F32)
    nudge = ((r[n:2 * n] % np.uint64(9)).astype(np.int64) - 4).reshape(n_groups, gsize)
    vals = (base.view(np.int32) + nudge.astype(np.int32)).view(F32)
    vals = np.minimum(vals, amax[:, None])
    sign = np.where((r[2 * n:3 * n] >> np.uint64(7)) & np.uint64(1), -1.0, 1.0).astype(F32)
    g = vals * sign.reshape(n_groups, gsize)
    g[:, 0] = amax
    return g.astype(F32)


@pytest.mark.parametrize("mode", MODES3)
def test_quotient_codes_on_rounding_boundaries(mode):
    """Values placed on s x (E4M3 midpoint) boundaries. The case set is
    checked to contain quotients whose code changes when x / s is replaced
    by x * (1 / s), so a reciprocal-multiply quantiser fails it."""
    gsize = 128 * 128 if mode == oracle.BLOCK_128x128 else 128
    n_groups = 8 if mode == oracle.BLOCK_128x128 else 1024
    g = _boundary_groups(n_groups, gsize, synth.seed(9, 13, mode))
    x = _groups_to_layout(g, mode, n_groups)
    s = _numpy_scales(x, mode)
    recip = (F32(1.0) / s).astype(F32)
    by_recip = torch_e4m3(np.clip((x * recip).astype(F32), F32(-448.0), F32(448.0)))
    assert np.count_nonzero(by_recip != _expected_codes(x, s)) > 10
    _check_quotient(x, mode)
