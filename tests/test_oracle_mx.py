"""Pins of the oracle's MXFP4 variant (32-element blocks, E8M0 power-of-two scales, no
tensor scale; the OCP MX definition of the pages' comparison format) against things it does
not compute itself: ml_dtypes' E8M0 and E2M1 conversions, the exact round trip of values
built on the grid, the scale's defining property (the block maximum lands in [4, 8) of the
element scale), the saturation rule and the error bound."""
import ml_dtypes
import numpy as np
import pytest

import oracle
import synth

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_e8m0_decode_matches_ml_dtypes():
    ref = np.arange(255, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    got = np.array([oracle.e8m0_decode(c) for c in range(255)])
    assert np.array_equal(got, ref)


def test_block_max_lands_in_the_top_binade():
    # E = floor(log2 b) - 2, so b / 2^E is in [4, 8) for every b in E8M0's unclamped range
    rng = np.random.default_rng(0)
    b = np.ldexp(rng.uniform(1.0, 2.0, 4000), rng.integers(-120, 120, 4000)).astype(np.float32)
    for v in b:
        e = oracle.mx_exponent(float(v))
        assert 4.0 <= float(v) / 2.0 ** e < 8.0, (v, e)


def test_exponent_clamps_to_e8m0_range():
    assert oracle.mx_exponent(0.0) == -127
    assert oracle.mx_exponent(float(np.float32(1e-40))) == -127      # 2^-133 - 2 < -127
    assert oracle.mx_exponent(float(np.finfo(np.float32).max)) == 125  # 2^127 - 2


@pytest.mark.parametrize("E", [-20, -3, 0, 5, 40])
def test_round_trip_of_grid_values(E):
    # rows of 32 grid values times 2^E with a maximum of 4 or 6: X = 2^E exactly, so the
    # codes are the grid indices and the dequantized values are the inputs
    rng = np.random.default_rng(E + 100)
    idx = rng.integers(0, 8, size=(4, 64))
    idx[:, ::32] = rng.choice([6, 7], size=(4, 2))  # block maxima 4 or 6
    sign = rng.choice([-1.0, 1.0], size=idx.shape)
    x = _bf16(sign * GRID[idx] * 2.0 ** E)
    q = oracle.mx_quantize(x)
    assert np.all(q.scales == E + 127)
    assert np.array_equal(q.dequantize(), synth.bf16_bits_to_f32(x).astype(np.float64))


def test_elements_match_ml_dtypes_rounding_with_saturation():
    x = synth.activations((64, 256), seed=21)
    q = oracle.mx_quantize(x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    E = q.scales.astype(np.int64).repeat(32, axis=1) - 127
    scaled = np.clip(xf / 2.0 ** E, -6.0, 6.0).astype(np.float32)
    ref = scaled.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    deq = q.dequantize() / 2.0 ** E
    assert np.array_equal(np.abs(deq), np.abs(ref))


def test_values_past_six_saturate():
    row = np.full(32, 1.0, dtype=np.float32)
    row[0] = 7.0                          # max 7: E = 0, 7 / 1 clamps to 6
    q = oracle.mx_quantize(_bf16(row[None, :]))
    assert q.scales[0, 0] == 127
    assert q.dequantize()[0, 0] == 6.0


def test_error_bound():
    # round to nearest on a grid whose spacing is at most 2 X, plus saturation of [6, 8) X:
    # |deq - x| <= 2 X
    x = synth.gradients((128, 512), seed=22)
    q = oracle.mx_quantize(x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    X = 2.0 ** (q.scales.astype(np.int64).repeat(32, axis=1) - 127)
    assert np.all(np.abs(q.dequantize() - xf) <= 2 * X)


def test_zero_block_and_transpose():
    z = np.zeros((64, 64), dtype=np.uint16)
    q = oracle.mx_quantize(z)
    assert np.all(q.scales == 0) and np.all(q.codes == 0)
    x = synth.activations((64, 96), seed=23)
    qt = oracle.mx_quantize(x, transpose=True)
    qd = oracle.mx_quantize(np.ascontiguousarray(x.T))
    assert np.array_equal(qt.codes, qd.codes) and np.array_equal(qt.scales, qd.scales)


def test_stochastic_rounding_is_unbiased_per_block():
    # one block repeated over many rows: each row draws other random bits, the mean of the
    # dequantized rows approaches the input.  The block maximum 2.9 sets X = 0.5 and maps to
    # 5.8 X, below the saturation point 6 X (a maximum always lands in [4, 8) X).
    base = np.linspace(-2.9, 2.9, 32).astype(np.float32)
    x = _bf16(np.tile(base, (4096, 1)))
    q = oracle.mx_quantize(x, sr=True, seed=5)
    xf = synth.bf16_bits_to_f32(x[0]).astype(np.float64)
    mean = q.dequantize().mean(axis=0)
    assert np.max(np.abs(mean - xf)) < 0.03


def test_nonfinite_input():
    xf = synth.bf16_bits_to_f32(synth.activations((32, 64), seed=24)).copy()
    xf[3, 7] = np.inf
    q = oracle.mx_quantize(synth.f32_to_bf16_bits(xf))
    assert q.status == oracle.NVO_ERR_NONFINITE
    assert np.all(q.codes == 0) and np.all(q.scales == 0)
