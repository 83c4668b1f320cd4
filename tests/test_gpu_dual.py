"""GPU parity of nvfp4_quantize_row_rht (one activation or gradient quantized row-wise for the
forward / data-gradient GEMM and RHT'd column-wise for the weight-gradient GEMM, from one amax
pass and one quantize pass) against the CPU oracle's two separate quantizations: codes, scales
and amax bit-exact, the column output on SR stream offset + 1."""
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


SHAPES = [(256, 512), (320, 192), (1024, 4096), (4096, 4096)]


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_dual_matches_oracle(sr, shape):
    gen = synth.gradients if sr else synth.activations
    x = gen(shape, seed=11)
    mask = oracle.sign_mask_from_seed(11)
    qr, qc = B.quantize_row_rht(to_device_bf16(x), mask, B.SR if sr else 0, seed=5, offset=3)
    assert_quantized_equal(qr, oracle.quantize(x, sr=sr, seed=5, offset=3), "row")
    assert_quantized_equal(qc, oracle.quantize(x, transpose=True, rht=True, sign_mask=mask,
                                               sr=sr, seed=5, offset=4), "rht col")


def test_dual_equals_the_two_separate_calls():
    x = to_device_bf16(synth.gradients((2048, 1536), seed=12))
    qr, qc = B.quantize_row_rht(x, 0x3C5A, B.SR, seed=9, offset=20)
    sr_row, _ = B.quantize(x, B.ROWWISE | B.SR, seed=9, offset=20)
    sr_col = B.rht_quantize(x, 0x3C5A, B.SR, seed=9, offset=21)
    for got, want in ((qr, sr_row), (qc, sr_col)):
        assert torch.equal(got.codes, want.codes)
        assert torch.equal(got.scales, want.scales)
        assert torch.equal(got.amax, want.amax)


def test_dual_amax_given():
    x = synth.activations((256, 512), seed=13)
    qr, qc = B.QuantizedTensor(256, 512), B.QuantizedTensor(512, 256)
    qr.amax.fill_(3.5)   # below the data's amax: scales and codes saturate
    qc.amax.fill_(2.0)
    B.quantize_row_rht(to_device_bf16(x), 0x1234, B.AMAX_GIVEN | B.SR, seed=2, offset=6,
                       out_row=qr, out_col=qc)
    assert_quantized_equal(qr, oracle.quantize(x, amax=3.5, sr=True, seed=2, offset=6), "row")
    assert_quantized_equal(qc, oracle.quantize(x, transpose=True, rht=True, sign_mask=0x1234,
                                               amax=2.0, sr=True, seed=2, offset=7), "col")


def test_dual_nonfinite_input():
    xf = synth.bf16_bits_to_f32(synth.activations((128, 256), seed=14)).copy()
    xf[70, 9] = np.nan
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    qr, qc = B.quantize_row_rht(to_device_bf16(x), 0xF0F0, B.SR, dev_status=status)
    assert int(status.item()) & B.DEVSTAT_NONFINITE
    assert_quantized_equal(qr, oracle.quantize(x, sr=True), "row")
    assert_quantized_equal(qc, oracle.quantize(x, transpose=True, rht=True, sign_mask=0xF0F0,
                                               sr=True, offset=1), "col")


def test_dual_transform_overflow_only_zeroes_the_column_output():
    # 16 equal bf16 values near the bf16 maximum sum past FLT_MAX inside the transform: the
    # RHT output (and its amax) is not finite while x itself is.
    xf = synth.bf16_bits_to_f32(synth.activations((128, 256), seed=15)).copy()
    xf[16:32, 40] = 3.0e38
    x = synth.f32_to_bf16_bits(xf)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    qr, qc = B.quantize_row_rht(to_device_bf16(x), 0, 0, dev_status=status)
    ref_r = oracle.quantize(x)
    ref_c = oracle.quantize(x, transpose=True, rht=True, sign_mask=0)
    assert ref_r.status == 0 and ref_c.status == oracle.NVO_ERR_NONFINITE
    assert int(status.item()) & B.DEVSTAT_NONFINITE
    assert_quantized_equal(qr, ref_r, "row")
    assert_quantized_equal(qc, ref_c, "col")


def test_dual_strided_input():
    x = synth.gradients((128, 768), seed=16)
    xd = to_device_bf16(x)[:, 64:512]
    xs = np.ascontiguousarray(x[:, 64:512])
    qr, qc = B.quantize_row_rht(xd, 0x0F0F, B.SR, seed=3, offset=8)
    assert_quantized_equal(qr, oracle.quantize(xs, sr=True, seed=3, offset=8), "row")
    assert_quantized_equal(qc, oracle.quantize(xs, transpose=True, rht=True, sign_mask=0x0F0F,
                                               sr=True, seed=3, offset=9), "col")


def test_dual_rejects_bad_arguments():
    x = to_device_bf16(synth.activations((256, 512), seed=16))
    with pytest.raises(B.NVFP4Error) as e:
        B.quantize_row_rht(x, 0, B.ROWWISE)
    assert e.value.status == B.ERR_ARG
    with pytest.raises(B.NVFP4Error) as e:
        B.quantize_row_rht(to_device_bf16(synth.activations((96, 512), seed=16)), 0, 0)
    assert e.value.status == B.ERR_SHAPE
