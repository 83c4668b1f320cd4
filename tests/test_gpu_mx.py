"""GPU parity of the MXFP4 variant (NVFP4_MX: 32-element blocks, E8M0 power-of-two scales, no
tensor scale) against the oracle's MX quantizer: codes bit-exact, each 32-block's E8M0 byte in
both of its 16-element scale slots, for row-wise, column-wise and RHT'd column-wise outputs,
RTN and SR; and nvfp4_gemm_mx against FP64 products of the oracle's dequantized operands."""
import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import (assert_gemm_close, need_gpu, padding_is_zero, qt_to_host,
                           to_device_bf16)

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def assert_mx_equal(qt, ref, what):
    codes, scales, _ = qt_to_host(qt)
    bad = np.argwhere(codes != ref.codes)
    assert bad.size == 0, (what, "codes differ at", bad[:5])
    for half in (0, 1):
        bad = np.argwhere(scales[:, half::2] != ref.scales)
        assert bad.size == 0, (what, "E8M0 scales differ at", half, bad[:5])
    assert padding_is_zero(qt.scales.cpu().numpy(), qt.rows, qt.cols), (what, "padding")


SHAPES = [(256, 512), (320, 192), (1024, 4096)]


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_mx_rowwise_and_colwise(sr, shape):
    x = (synth.gradients if sr else synth.activations)(shape, seed=31)
    flags = B.ROWWISE | B.COLWISE | B.MX | (B.SR if sr else 0)
    qr, qc = B.quantize(to_device_bf16(x), flags, seed=7, offset=2)
    assert_mx_equal(qr, oracle.mx_quantize(x, sr=sr, seed=7, offset=2), "row")
    assert_mx_equal(qc, oracle.mx_quantize(x, transpose=True, sr=sr, seed=7, offset=2), "col")


@pytest.mark.parametrize("sr", [False, True])
def test_mx_rowwise_only_and_rht_colwise(sr):
    x = synth.gradients((512, 1024), seed=32)
    qr, _ = B.quantize(to_device_bf16(x), B.ROWWISE | B.MX | (B.SR if sr else 0), seed=3)
    assert_mx_equal(qr, oracle.mx_quantize(x, sr=sr, seed=3), "row only")
    mask = oracle.sign_mask_from_seed(32)
    qc = B.rht_quantize(to_device_bf16(x), mask, B.MX | (B.SR if sr else 0), seed=3, offset=1)
    assert_mx_equal(qc, oracle.mx_quantize(x, transpose=True, rht=True, sign_mask=mask, sr=sr,
                                           seed=3, offset=1), "rht col")


def test_mx_tiny_and_zero_blocks():
    xf = np.zeros((64, 256), dtype=np.float32)
    xf[1, :] = 3e-39                      # subnormal block maxima: E clamps to -127
    xf[2, :32] = np.float32(2.0) ** -100
    xf[3, 5] = 7.0                        # saturates
    x = synth.f32_to_bf16_bits(xf)
    qr, _ = B.quantize(to_device_bf16(x), B.ROWWISE | B.MX)
    assert_mx_equal(qr, oracle.mx_quantize(x), "tiny/zero")


def test_mx_nonfinite_input():
    xf = synth.bf16_bits_to_f32(synth.activations((128, 256), seed=33)).copy()
    xf[9, 40] = np.nan
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    qr, _ = B.quantize(to_device_bf16(x), B.ROWWISE | B.MX, dev_status=status)
    ref = oracle.mx_quantize(x)
    assert ref.status == oracle.NVO_ERR_NONFINITE
    assert int(status.item()) & B.DEVSTAT_NONFINITE
    assert_mx_equal(qr, ref, "nonfinite")


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (144, 272, 320), (2048, 1024, 4096)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mx_gemm(M, N, K, dtype):
    X = synth.activations((M, K), seed=34)
    W = synth.weights((N, K), seed=34)
    qa, _ = B.quantize(to_device_bf16(X), B.ROWWISE | B.MX)
    qb, _ = B.quantize(to_device_bf16(W), B.ROWWISE | B.MX)
    D = B.gemm(qa, qb, out_dtype=dtype, mx=True)
    D_ref, norm = oracle.gemm_ref(oracle.mx_quantize(X), oracle.mx_quantize(W))
    assert_gemm_close(D.float().cpu().numpy(), D_ref, norm, bf16=dtype == torch.bfloat16,
                      what=f"mx gemm {M}x{N}x{K}")


def test_mx_rejects_2d_scaling():
    x = to_device_bf16(synth.weights((256, 512), seed=35))
    with pytest.raises(B.NVFP4Error) as e:
        B.quantize(x, B.ROWWISE | B.BLOCK2D | B.MX)
    assert e.value.status == B.ERR_ARG
