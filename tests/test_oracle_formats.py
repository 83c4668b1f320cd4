"""Pins of the oracle's element and scale codecs (E2M1, E4M3) against closed forms, the
MX specification's value table, and two independent libraries (ml_dtypes, torch)."""
import math

import ml_dtypes
import numpy as np
import torch

import oracle
from conftest import golden_rows


def _f32_from_bits(bits):
    return np.asarray(bits, dtype=np.uint32).view(np.float32)


# ---- E2M1 ------------------------------------------------------------------------------

def test_e2m1_decode_matches_mx_table():
    for code, value in golden_rows("e2m1_values.txt"):
        got = oracle.e2m1_decode(int(code))
        want = float(value)
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), code


def test_e2m1_decode_closed_form_from_bit_fields():
    # value = (-1)^s * 2^(e-1) * (1 + m/2) for e > 0, (-1)^s * m/2 for e = 0 (bias 1)
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = (2.0 ** (e - 1)) * (1 + m / 2) if e > 0 else m / 2
        assert oracle.e2m1_decode(code) == (-mag if s else mag)


def test_e2m1_decode_matches_ml_dtypes():
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for code in range(16):
        assert oracle.e2m1_decode(code) == lib_vals[code]


def test_e2m1_grid_has_16_patterns_and_15_values():
    vals = {oracle.e2m1_decode(c) for c in range(16)}
    assert len(vals) == 15  # +0 and -0 compare equal


def test_e2m1_rtn_ties_go_to_even_code():
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, code in expect.items():
        assert oracle.e2m1_rtn(v) == code
        assert oracle.e2m1_rtn(-v) == code | 8


def test_e2m1_rtn_saturates_and_keeps_negative_zero():
    for v in (6.0, 6.5, 7.0, 100.0, 3.0e38, float("inf")):
        assert oracle.e2m1_rtn(v) == 7
        assert oracle.e2m1_rtn(-v) == 15
    assert oracle.e2m1_rtn(-0.0) == 8
    assert oracle.e2m1_rtn(-0.1) == 8
    assert oracle.e2m1_rtn(0.0) == 0


def test_e2m1_rtn_matches_ml_dtypes_dense_sweep():
    # every FP32 value in [2^-3, 8) (all RTN thresholds lie there) plus a sample below
    bits = np.arange((127 - 3) << 23, (127 + 3) << 23, dtype=np.uint32)
    v = _f32_from_bits(bits)
    rng = np.random.default_rng(11)
    small = rng.uniform(0, 0.125, 200_000).astype(np.float32)
    big = rng.uniform(8, 1e6, 50_000).astype(np.float32)
    v = np.concatenate([v, small, big])
    v = np.concatenate([v, -v[::97]])
    ours = oracle.e2m1_rtn_many(v)
    theirs = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    bad = np.nonzero(ours != theirs)[0]
    assert bad.size == 0, (v[bad[:5]], ours[bad[:5]], theirs[bad[:5]])


# ---- E4M3 ------------------------------------------------------------------------------

def test_e4m3_decode_closed_form_and_range():
    for b in range(0x7F):
        e, m = b >> 3, b & 7
        want = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        assert oracle.e4m3_decode(b) == want
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    vals = [oracle.e4m3_decode(b) for b in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))


def test_e4m3_decode_matches_ml_dtypes():
    lib_vals = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for b in range(0x7F):
        assert oracle.e4m3_decode(b) == lib_vals[b]


def _e4m3_sweep_values():
    # FP32 values in [2^-12, 2^9) with a prime mantissa stride, every tie point between
    # consecutive E4M3 values with its FP32 neighbours, and random draws
    lo, hi = (127 - 12) << 23, (127 + 9) << 23
    bits = np.arange(lo, hi, 7, dtype=np.uint32)
    e4 = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mids = ((e4[:-1] + e4[1:]) / 2).astype(np.float32)
    mid_bits = mids.view(np.uint32)
    ties = np.concatenate([mid_bits - 1, mid_bits, mid_bits + 1]).view(np.float32)
    rng = np.random.default_rng(7)
    rnd = np.exp(rng.uniform(np.log(2.0 ** -14), np.log(2000.0), 1_000_000)).astype(np.float32)
    edge = np.array([0.0, 2.0 ** -10, 448.0, 460.0, 464.0, 464.01, 480.0, 1e6, 3e38],
                    dtype=np.float32)
    return np.concatenate([_f32_from_bits(bits), ties, rnd, edge])


def test_e4m3_encode_matches_ml_dtypes():
    x = _e4m3_sweep_values()
    ours = oracle.e4m3_encode_many(x)
    clamped = np.minimum(x, np.float32(448.0))  # the libraries overflow to NaN; ours saturates
    theirs = clamped.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    bad = np.nonzero(ours != theirs)[0]
    assert bad.size == 0, (x[bad[:5]], ours[bad[:5]], theirs[bad[:5]])


def test_e4m3_encode_matches_torch():
    x = _e4m3_sweep_values()[::5].copy()
    ours = oracle.e4m3_encode_many(x)
    clamped = torch.from_numpy(np.minimum(x, np.float32(448.0)))
    theirs = clamped.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_e4m3_encode_saturates():
    for x in (448.0, 464.0, 465.0, 1000.0, 3.0e38, float("inf")):
        assert oracle.e4m3_encode(x) == 0x7E
    assert oracle.e4m3_encode(0.0) == 0
    assert oracle.e4m3_encode(2.0 ** -10) == 0       # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(1.5 * 2.0 ** -9) == 2  # tie between codes 1 and 2 -> 2
