"""GPU parity of the quantizers against the CPU oracle: codes, scales and amax bit-exact on
the same seeded inputs, for every mode of the recipe, ragged shapes and the edge cases."""
import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import assert_quantized_equal, need_gpu, to_device_bf16

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


SHAPES = [(256, 512), (272, 320), (1024, 4096), (4096, 4096)]


def _act(shape, seed=0):
    return synth.activations(shape, seed=seed)


def _grad(shape, seed=1):
    return synth.gradients(shape, seed=seed)


@pytest.mark.parametrize("shape", SHAPES)
def test_rowwise_rtn(shape):
    x = _act(shape)
    qr, _ = B.quantize(to_device_bf16(x), B.ROWWISE)
    assert_quantized_equal(qr, oracle.quantize(x), "rowwise rtn")


@pytest.mark.parametrize("shape", SHAPES)
def test_rowwise_sr(shape):
    x = _grad(shape)
    qr, _ = B.quantize(to_device_bf16(x), B.ROWWISE | B.SR, seed=77, offset=5)
    assert_quantized_equal(qr, oracle.quantize(x, sr=True, seed=77, offset=5), "rowwise sr")


@pytest.mark.parametrize("shape", [(512, 512), (192, 320), (4096, 4096), (320, 1024)])
def test_block2d_both_directions(shape):
    w = synth.weights(shape, seed=2)
    qr, qc = B.quantize(to_device_bf16(w), B.ROWWISE | B.COLWISE | B.BLOCK2D)
    assert_quantized_equal(qr, oracle.quantize(w, block2d=True), "2d row")
    assert_quantized_equal(qc, oracle.quantize(w, transpose=True, block2d=True), "2d col")


@pytest.mark.parametrize("flags", ["row", "col"])
def test_block2d_single_direction(flags):
    w = synth.weights((320, 448), seed=3)
    if flags == "row":
        qr, _ = B.quantize(to_device_bf16(w), B.ROWWISE | B.BLOCK2D)
        assert_quantized_equal(qr, oracle.quantize(w, block2d=True), "2d row only")
    else:
        _, qc = B.quantize(to_device_bf16(w), B.COLWISE | B.BLOCK2D)
        assert_quantized_equal(qc, oracle.quantize(w, transpose=True, block2d=True), "2d col only")


def test_block2d_rows_not_multiple_of_64():
    w = synth.weights((144, 256), seed=4)
    qr, _ = B.quantize(to_device_bf16(w), B.ROWWISE | B.BLOCK2D)
    assert_quantized_equal(qr, oracle.quantize(w, block2d=True), "2d row ragged")


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("shape", [(256, 512), (320, 272), (2048, 1024)])
def test_colwise(sr, shape):
    x = _grad(shape) if sr else _act(shape)
    flags = B.COLWISE | (B.SR if sr else 0)
    _, qc = B.quantize(to_device_bf16(x), flags, seed=9, offset=2)
    assert_quantized_equal(qc, oracle.quantize(x, transpose=True, sr=sr, seed=9, offset=2),
                           "colwise")


@pytest.mark.parametrize("sr", [False, True])
def test_row_and_col_1x16(sr):
    x = _grad((384, 640)) if sr else _act((384, 640))
    flags = B.ROWWISE | B.COLWISE | (B.SR if sr else 0)
    qr, qc = B.quantize(to_device_bf16(x), flags, seed=3, offset=1)
    assert_quantized_equal(qr, oracle.quantize(x, sr=sr, seed=3, offset=1), "row of both")
    assert_quantized_equal(qc, oracle.quantize(x, transpose=True, sr=sr, seed=3, offset=1),
                           "col of both")


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("shape", [(256, 512), (320, 272), (4096, 1024)])
def test_rht_colwise(sr, shape):
    x = _grad(shape) if sr else _act(shape)
    mask = oracle.sign_mask_from_seed(11)
    qc = B.rht_quantize(to_device_bf16(x), mask, B.SR if sr else 0, seed=5, offset=3)
    ref = oracle.quantize(x, transpose=True, rht=True, sign_mask=mask, sr=sr, seed=5, offset=3)
    assert_quantized_equal(qc, ref, "rht colwise")


@pytest.mark.parametrize("mode", ["row", "rowsr", "col", "rht", "2d"])
def test_amax_given(mode):
    x = _act((256, 512))
    amax = 3.5  # below the data's amax: scales and codes saturate
    if mode == "rht":
        out = B.QuantizedTensor(512, 256)
        out.amax.fill_(amax)
        B.rht_quantize(to_device_bf16(x), 0x1234, B.AMAX_GIVEN, out_col=out)
        ref = oracle.quantize(x, transpose=True, rht=True, sign_mask=0x1234, amax=amax)
        assert_quantized_equal(out, ref, mode)
        return
    flags = {"row": B.ROWWISE, "rowsr": B.ROWWISE | B.SR, "col": B.COLWISE,
             "2d": B.ROWWISE | B.COLWISE | B.BLOCK2D}[mode]
    qr = B.QuantizedTensor(256, 512) if flags & B.ROWWISE else None
    qc = B.QuantizedTensor(512, 256) if flags & B.COLWISE else None
    (qr if qr is not None else qc).amax.fill_(amax)
    B.quantize(to_device_bf16(x), flags | B.AMAX_GIVEN, seed=4, out_row=qr, out_col=qc)
    kw = dict(amax=amax, sr=bool(flags & B.SR), seed=4, block2d=bool(flags & B.BLOCK2D))
    if qr is not None:
        assert_quantized_equal(qr, oracle.quantize(x, **kw), mode + " row")
    if qc is not None:
        assert_quantized_equal(qc, oracle.quantize(x, transpose=True, **kw), mode + " col")


def test_strided_input():
    x = _act((128, 768))
    xd = to_device_bf16(x)[:, 64:576]
    qr, _ = B.quantize(xd, B.ROWWISE | B.SR, seed=1)
    assert_quantized_equal(qr, oracle.quantize(np.ascontiguousarray(x[:, 64:576]), sr=True,
                                               seed=1), "strided")
    _, qc = B.quantize(xd, B.COLWISE)
    assert_quantized_equal(qc, oracle.quantize(np.ascontiguousarray(x[:, 64:576]),
                                               transpose=True), "strided col")


@pytest.mark.parametrize("bad", [np.nan, np.inf])
@pytest.mark.parametrize("mode", ["row", "tile", "rht"])
def test_nonfinite_input(bad, mode):
    xf = synth.bf16_bits_to_f32(_act((128, 256))).copy()
    xf[7, 100] = bad
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if mode == "row":
        q, _ = B.quantize(to_device_bf16(x), B.ROWWISE, dev_status=status)
        ref = oracle.quantize(x)
    elif mode == "tile":
        _, q = B.quantize(to_device_bf16(x), B.COLWISE | B.BLOCK2D, dev_status=status)
        ref = oracle.quantize(x, transpose=True, block2d=True)
    else:
        q = B.rht_quantize(to_device_bf16(x), 0xF0F0, B.SR, dev_status=status)
        ref = oracle.quantize(x, transpose=True, rht=True, sign_mask=0xF0F0, sr=True)
    assert ref.status == oracle.NVO_ERR_NONFINITE
    assert int(status.item()) & B.DEVSTAT_NONFINITE
    assert_quantized_equal(q, ref, "nonfinite")


def test_zero_and_tiny_tensors():
    z = np.zeros((128, 256), dtype=np.uint16)
    z[1, 3] = 0x8000
    q, _ = B.quantize(to_device_bf16(z), B.ROWWISE)
    assert_quantized_equal(q, oracle.quantize(z), "zeros")
    tiny = synth.f32_to_bf16_bits(np.full((128, 256), 1e-38, dtype=np.float32))
    tiny[5, 7] = synth.f32_to_bf16_bits(np.float32(-3e-39))
    q, _ = B.quantize(to_device_bf16(tiny), B.ROWWISE | B.SR, seed=2)
    assert_quantized_equal(q, oracle.quantize(tiny, sr=True, seed=2), "tiny")


def test_underflowing_blocks():
    xf = np.zeros((64, 128), dtype=np.float32)
    xf[0, 0] = 1.0
    xf[1:, :] = np.random.default_rng(0).standard_normal((63, 128)) * 1e-7
    x = synth.f32_to_bf16_bits(xf)
    q, _ = B.quantize(to_device_bf16(x), B.ROWWISE)
    assert_quantized_equal(q, oracle.quantize(x), "underflow")
    _, qc = B.quantize(to_device_bf16(x), B.COLWISE | B.SR, seed=8)
    assert_quantized_equal(qc, oracle.quantize(x, transpose=True, sr=True, seed=8), "underflow c")


def test_sr_reproducible_and_seed_dependent():
    xd = to_device_bf16(_grad((256, 256)))
    a, _ = B.quantize(xd, B.ROWWISE | B.SR, seed=1, offset=0)
    b, _ = B.quantize(xd, B.ROWWISE | B.SR, seed=1, offset=0)
    c, _ = B.quantize(xd, B.ROWWISE | B.SR, seed=1, offset=1)
    assert torch.equal(a.codes, b.codes)
    assert not torch.equal(a.codes, c.codes)


@pytest.mark.slow
def test_full_size_rowwise_2e30_sampled():
    """The quantizer sweep's largest tensor (2^30 elements in rows of 4096), one call per
    mode.  The amax is checked against numpy on the whole tensor; codes and scales of sampled
    rows against the oracle given that amax (the SR band is the first 64 rows, whose element
    indices are the same in the sub-matrix)."""
    from nvfp4_testlib import sf_offsets
    rows, cols = synth.quant_sweep_shape(30)
    x = synth.activations((rows, cols), seed=synth.QUANT_SWEEP_SEED)
    xd = to_device_bf16(x)
    amax = float(np.abs(synth.bf16_bits_to_f32(x)).max())
    rng = np.random.default_rng(0)
    rows_s = np.sort(rng.choice(rows, 64, replace=False))
    offs = sf_offsets(rows, cols)

    qn, _ = B.quantize(xd, B.ROWWISE)
    assert float(qn.amax.item()) == amax
    ref = oracle.quantize(x[rows_s], amax=amax)
    assert np.array_equal(qn.codes[torch.from_numpy(rows_s).cuda()].cpu().numpy(), ref.codes)
    assert np.array_equal(qn.scales.cpu().numpy()[offs[rows_s]], ref.scales)
    del qn

    qs, _ = B.quantize(xd, B.ROWWISE | B.SR, seed=3)
    ref = oracle.quantize(x[:64], amax=amax, sr=True, seed=3)
    assert np.array_equal(qs.codes[:64].cpu().numpy(), ref.codes)
    assert np.array_equal(qs.scales.cpu().numpy()[offs[:64]], ref.scales)
