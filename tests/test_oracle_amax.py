"""Pins of the oracle's stand-alone tensor amax (nvo_amax), the first pass of its quantizer
[P1 Formato NVFP4: one FP32 scale per tensor from its amax], against computations that do not
go through the oracle: numpy's absolute maximum, and the random Hadamard transform as an FP64
matrix product with scipy's Sylvester Hadamard matrix."""
import numpy as np
import pytest
from scipy.linalg import hadamard

import oracle
import synth


def _f32(x):
    return synth.bf16_bits_to_f32(x).astype(np.float64)


def _signs(mask):
    return np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])


def _rht_blocks_fp64(xf, mask, along_rows):
    """y = H diag(s) x / 4 over every 16-block, in FP64; blocks along the rows of xf, or down
    its columns.  Returns the transformed blocks and, per block, sum |x| (the error bound's
    scale)."""
    H = hadamard(16).astype(np.float64)
    s = _signs(mask)
    if along_rows:
        blk = xf.reshape(xf.shape[0], -1, 16)                     # (R, C/16, 16)
    else:
        blk = xf.reshape(-1, 16, xf.shape[1]).transpose(0, 2, 1)  # (R/16, C, 16)
    y = (blk * s) @ H.T / 4.0
    return y, np.abs(blk).sum(axis=-1)


@pytest.mark.parametrize("shape", [(48, 80), (256, 512), (16, 16)])
@pytest.mark.parametrize("transpose", [False, True])
def test_plain_amax_is_numpys_absolute_maximum(shape, transpose):
    x = synth.activations(shape, seed=61)
    a, st = oracle.amax(x, transpose=transpose)
    assert st == oracle.NVO_OK
    assert a == np.float32(np.abs(synth.bf16_bits_to_f32(x)).max())


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("seed", [62, 63])
def test_rht_amax_within_the_fp32_butterfly_bound_of_the_fp64_transform(transpose, seed):
    x = synth.gradients((64, 96), seed=seed)
    mask = oracle.sign_mask_from_seed(seed)
    a, st = oracle.amax(x, transpose=transpose, rht=True, sign_mask=mask)
    assert st == oracle.NVO_OK
    y, l1 = _rht_blocks_fp64(_f32(x), mask, along_rows=not transpose)
    exact = np.abs(y).max()
    # four levels of FP32 additions (and one exact scaling): |error| <= 4 u sum|x| / 4 per value
    bound = 4 * 2.0 ** -24 * l1.max() / 4 + 1e-45
    assert abs(a - exact) <= bound, (a, exact, bound)
    # a plausible slip -- the transform along the other axis -- lands elsewhere
    y_other, _ = _rht_blocks_fp64(_f32(x), mask, along_rows=transpose)
    assert abs(np.abs(y_other).max() - a) > bound


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("rht", [False, True])
def test_amax_equals_the_quantizers_first_pass(transpose, rht):
    x = synth.gradients((96, 160), seed=64)
    mask = oracle.sign_mask_from_seed(64)
    a, _ = oracle.amax(x, transpose=transpose, rht=rht, sign_mask=mask)
    q = oracle.quantize(x, transpose=transpose, rht=rht, sign_mask=mask)
    assert np.float32(a).view(np.uint32) == np.float32(q.amax).view(np.uint32)


@pytest.mark.parametrize("bad", [np.nan, np.inf])
def test_nonfinite_input(bad):
    xf = synth.bf16_bits_to_f32(synth.activations((32, 64), seed=65)).copy()
    xf[7, 9] = bad
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)
    for rht in (False, True):
        a, st = oracle.amax(x, rht=rht)
        assert st == oracle.NVO_ERR_NONFINITE and a == np.inf


def test_rht_needs_whole_blocks():
    x = synth.activations((32, 40), seed=66)
    with pytest.raises(ValueError):
        oracle.amax(x, rht=True)
    with pytest.raises(ValueError):
        oracle.amax(x.T.copy(), transpose=True, rht=True)
