"""Pins of the oracle's tensor quantizer: nibble packing, the two-level scale closed form,
exact round trips, 2D weight-block consistency, stochastic-rounding unbiasedness, the
non-finite and degenerate cases, and a per-element error bound."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def unpack(codes):
    lo = codes & 0xF
    hi = codes >> 4
    out = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def bf16(values):
    return synth.f32_to_bf16_bits(np.asarray(values, dtype=np.float32))


def test_nibble_packing_and_codes_by_construction():
    # one block holds every grid value (and negatives); amax = 6 * 2^-3 makes S_enc / sf
    # = 2^3 exactly, so each element maps exactly onto its grid point
    c = 2.0 ** -3
    vals = [GRID[i % 8] * c * (-1 if i >= 8 else 1) for i in range(16)]
    x = bf16([vals, vals[::-1]])
    q = oracle.quantize(x)
    assert q.amax == 6 * c
    want = [(i % 8) | (8 if i >= 8 else 0) for i in range(16)]
    got = unpack(q.codes)
    assert list(got[0]) == want
    assert list(got[1]) == want[::-1]
    # low nibble of byte k is column 2k
    assert q.codes[0, 0] == (want[1] << 4) | want[0]
    assert np.all(q.scales == 0x7E)


def test_block_holding_the_amax_gets_scale_448_and_code_6():
    x = synth.activations((64, 256), seed=0)
    xf = synth.bf16_bits_to_f32(x)
    for kw in ({}, {"sr": True, "seed": 3}, {"transpose": True}, {"block2d": True}):
        q = oracle.quantize(x, **kw)
        xl = xf.T if kw.get("transpose") else xf
        assert q.amax == np.abs(xf).max()
        r, c = np.unravel_index(np.argmax(np.abs(xl)), xl.shape)
        assert q.scales[r, c // 16] == 0x7E
        assert unpack(q.codes)[r, c] & 7 == 7


def _round_trip_tensor(rng, rows, cols, k, block2d):
    """Elements e2m1(code) * sf / 2^k with one +-6 per block and S_enc = 2^k exactly."""
    nb = cols // 16
    e4_vals = np.array([oracle.e4m3_decode(b) for b in range(1, 0x7E)])
    codes = rng.integers(0, 16, (rows, cols))
    if block2d:
        sf_tile = rng.choice(e4_vals, (rows // 16, nb))
        sf = np.repeat(sf_tile, 16, axis=0)
        for tr in range(rows // 16):
            for kb in range(nb):
                codes[16 * tr + rng.integers(0, 16), 16 * kb + rng.integers(0, 16)] = 7
    else:
        sf = rng.choice(e4_vals, (rows, nb))
        for r in range(rows):
            for kb in range(nb):
                codes[r, 16 * kb + rng.integers(0, 16)] = 7 | (8 * rng.integers(0, 2))
    sf[0, 0] = 448.0
    if block2d:
        sf[:16, 0] = 448.0
    mag = np.array(GRID)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    x = mag * np.repeat(sf, 16, axis=1) * 2.0 ** -k
    return x, codes, sf


@pytest.mark.parametrize("block2d", [False, True])
def test_round_trip_of_exactly_representable_inputs(block2d):
    rng = np.random.default_rng(21)
    for k in (0, 10, 20):
        x, codes, sf = _round_trip_tensor(rng, 32, 128, k, block2d)
        xb = bf16(x)
        assert np.array_equal(synth.bf16_bits_to_f32(xb).astype(np.float64), x)
        q = oracle.quantize(xb, block2d=block2d)
        assert q.amax == np.float32(2688 * 2.0 ** -k)
        assert oracle.tensor_scale(q.amax) == 2.0 ** k
        got = unpack(q.codes)
        assert np.array_equal(got, codes), np.argwhere(got != codes)[:3]
        dec = np.vectorize(oracle.e4m3_decode)(q.scales)
        assert np.array_equal(dec, sf)
        assert np.array_equal(q.dequantize(), x)


def test_2d_weight_blocks_are_the_same_in_both_directions():
    W = synth.weights((64, 96), seed=1)
    qr = oracle.quantize(W, block2d=True)
    qc = oracle.quantize(W, transpose=True, block2d=True)
    assert qr.amax == qc.amax
    assert np.array_equal(unpack(qr.codes), unpack(qc.codes).T)
    assert np.array_equal(qr.dequantize(), qc.dequantize().T)
    # one scale per 16 x 16 tile, identical in the two layouts
    sr_ = qr.scales.reshape(4, 16, 6)
    assert np.all(sr_ == sr_[:, :1, :])
    sc_ = qc.scales.reshape(6, 16, 4)
    assert np.array_equal(sr_[:, 0, :], sc_[:, 0, :].T)


def test_1x16_scales_differ_from_2d():
    W = synth.weights((64, 96), seed=1)
    assert not np.array_equal(oracle.quantize(W).scales, oracle.quantize(W, block2d=True).scales)


def test_stochastic_rounding_is_unbiased_over_1e5_draws():
    # S_enc = 448 * 2^3 with amax = 6 * 2^-3 gives r = S_enc / 448 = 2^3 exactly, so the
    # scaled values are exactly the chosen off-grid points
    j = 3
    targets = [0.3, 0.7, 1.1, 1.3, 1.9, 2.2, 2.75, 3.9, 4.6, 5.5, 0.01, 5.99, 1.0, 4.0]
    row = [6.0] + targets + [0.0]
    reps = 100_000 // 16 * 16 + 16 * 16
    x = bf16(np.tile(np.array(row) * 2.0 ** -j, (reps, 1)))
    q = oracle.quantize(x, sr=True, seed=12345, offset=7)
    assert np.all(q.scales == 0x7E)
    deq = q.dequantize() * 2.0 ** j   # back to the scaled units
    vals = synth.bf16_bits_to_f32(x[0]).astype(np.float64) * 2.0 ** j
    for i, v in enumerate(vals):
        col = deq[:, i]
        if v in GRID:
            assert np.all(col == v)  # on-grid values never move
            continue
        lo = max(g for g in GRID if g <= v)
        hi = min(g for g in GRID if g > v)
        p = (v - lo) / (hi - lo)
        sigma = (hi - lo) * np.sqrt(p * (1 - p) / col.size)
        bias_bound = (hi - lo) * 2.0 ** -16
        assert abs(col.mean() - v) <= 4 * sigma + bias_bound, (v, col.mean())
        assert set(np.unique(col)) <= {lo, hi}


def test_stochastic_rounding_up_probability_is_exact():
    # over all 2^16 values of r16, the magnitude rounds up exactly ceil(p * 2^16) times
    r = np.arange(65536, dtype=np.uint32)
    for v in (0.3, 0.7000001, 1.1, 1.9, 2.2, 2.75, 3.9, 4.6, 5.5, 0.0001, 5.9999, 1e-30):
        v32 = np.float32(v)
        fv = Fraction(float(v32))
        lo = max(Fraction(g) for g in GRID if Fraction(g) <= fv)
        hi = min(Fraction(g) for g in GRID if Fraction(g) > fv)
        p = (fv - lo) / (hi - lo)
        want = -((-p * 65536) // 1)  # ceil
        codes = oracle.e2m1_sr_many(np.full(65536, v32), r)
        lo_code = GRID.index(float(lo))
        ups = int((codes == lo_code + 1).sum())
        assert ups == want, (v, ups, want)
        assert int((codes == lo_code).sum()) == 65536 - want
        neg = oracle.e2m1_sr_many(np.full(65536, -v32), r)
        assert np.array_equal(neg, codes | 8)


def test_sr_codes_depend_on_seed_offset_and_position():
    x = synth.gradients((32, 64), seed=2)
    a = oracle.quantize(x, sr=True, seed=1, offset=0).codes
    assert np.array_equal(a, oracle.quantize(x, sr=True, seed=1, offset=0).codes)
    assert not np.array_equal(a, oracle.quantize(x, sr=True, seed=1, offset=1).codes)
    assert not np.array_equal(a, oracle.quantize(x, sr=True, seed=2, offset=0).codes)


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
@pytest.mark.parametrize("mode", [{}, {"transpose": True, "rht": True, "sign_mask": 0x1234},
                                  {"block2d": True}, {"sr": True}])
def test_non_finite_input_zeroes_everything(bad, mode):
    x = synth.activations((32, 64), seed=0)
    xf = synth.bf16_bits_to_f32(x).copy()
    xf[5, 17] = bad
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)
    q = oracle.quantize(xb, **mode)
    assert q.status == oracle.NVO_ERR_NONFINITE
    assert q.amax == np.inf
    assert not q.codes.any() and not q.scales.any()


def test_rht_overflow_is_non_finite():
    big = np.full((16, 16), 3.0e38, dtype=np.float32)
    q = oracle.quantize(synth.f32_to_bf16_bits(big), transpose=True, rht=True)
    assert q.status == oracle.NVO_ERR_NONFINITE


def test_all_zero_tensor_and_signed_zeros():
    x = np.zeros((16, 32), dtype=np.uint16)
    x[3, 5] = 0x8000  # -0.0
    q = oracle.quantize(x)
    assert q.status == oracle.NVO_OK and q.amax == 0.0
    assert oracle.tensor_scale(0.0) == 1.0
    assert not q.scales.any()
    got = unpack(q.codes)
    assert got[3, 5] == 8 and got.sum() == 8


def test_tiny_amax_clamps_the_tensor_scale():
    x = bf16(np.full((16, 32), 1e-38))
    q = oracle.quantize(x)
    assert oracle.tensor_scale(q.amax) == np.float32(3.4028234663852886e38)
    d = q.dequantize()
    assert np.all(np.isfinite(d))


def test_underflowing_block_scale_gives_zero_codes():
    # a block 1e-7 times smaller than the amax: (b/6) * S_enc < 2^-10, so sf = 0
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = 1.0
    x[0, 16:] = -1e-7
    q = oracle.quantize(bf16(x))
    assert q.scales[0, 1] == 0
    assert np.all(unpack(q.codes)[0, 16:] == 8)


def _step(v):
    return np.where(v < 2, 0.5, np.where(v < 4, 1.0, 2.0))


@pytest.mark.parametrize("sr", [False, True])
def test_per_element_error_bound(sr):
    x = synth.activations((64, 512), seed=4)
    q = oracle.quantize(x, sr=sr, seed=9)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    s_enc = float(oracle.tensor_scale(q.amax))
    sf = np.repeat(np.vectorize(oracle.e4m3_decode)(q.scales), 16, axis=1)
    unit = sf / s_enc                     # value of one grid unit in this block
    v = np.abs(xf) / np.where(unit > 0, unit, 1)
    sat = np.maximum(0.0, np.abs(xf) - 6 * unit)
    allowed = (1.0 if sr else 0.5) * _step(np.minimum(v, 5.999)) * unit + sat
    err = np.abs(q.dequantize() - xf)
    assert np.all(err <= allowed * (1 + 1e-6) + 1e-30)
    # e4m3 block scales keep every block max within one E4M3 rounding of 6 units
    assert np.all(sat <= np.abs(xf) * 2.0 ** -4 + 1e-30)


_SPLIT_MODES = [
    dict(),
    dict(sr=True, seed=3, offset=2),
    dict(block2d=True),
    dict(transpose=True, block2d=True),
    dict(transpose=True, rht=True, sign_mask=0x1234, sr=True, seed=9, offset=1),
    dict(transpose=True, rht=True, sign_mask=0xBEEF),
]


@pytest.mark.parametrize("kw", _SPLIT_MODES)
@pytest.mark.parametrize("shape", [(512, 768), (48, 320)])
def test_row_ranges_and_threads_give_the_whole_call(kw, shape):
    """The element index of stochastic rounding is the absolute row's (e = r * C' + c), and a
    16 x 16 tile never straddles two calls, so quantizing the logical rows in several ranges
    with the whole tensor's amax -- or with the threaded driver -- gives the whole call's bits."""
    x = synth.gradients(shape, seed=11)
    whole = oracle.quantize(x, **kw)
    R = whole.rows
    cuts = [0, 16, 16 * max(1, R // 48), R]
    out = None
    for r0, r1 in zip(cuts[:-1], cuts[1:]):
        if r1 > r0:
            out = oracle.quantize_rows(x, r0, r1, whole.amax, out=out, **kw)
    assert np.array_equal(out.codes, whole.codes) and np.array_equal(out.scales, whole.scales)
    for threads in (2, 5, 64):
        mt = oracle.quantize(x, threads=threads, **kw)
        assert mt.amax == whole.amax and mt.status == whole.status
        assert np.array_equal(mt.codes, whole.codes)
        assert np.array_equal(mt.scales, whole.scales)


def test_row_ranges_reject_misaligned_starts_and_bad_amax():
    x = synth.activations((64, 64), seed=1)
    with pytest.raises(ValueError):
        oracle.quantize_rows(x, 8, 64, 1.0)
    with pytest.raises(ValueError):
        oracle.quantize_rows(x, 0, 64, float("inf"))


def test_threaded_driver_flags_non_finite_input():
    x = synth.activations((256, 256), seed=2)
    x[200, 7] = 0x7FC0  # NaN
    q = oracle.quantize(x, threads=4)
    assert q.status == oracle.NVO_ERR_NONFINITE and np.isinf(q.amax)
    assert not q.codes.any() and not q.scales.any()
