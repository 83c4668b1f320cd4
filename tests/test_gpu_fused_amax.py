"""nvfp4_gemm_amax: a bf16 GEMM that also emits the maxima the next quantization of its output
needs (max |D| and max |RHT(D)| along the rows), so that quantization can skip its amax pass.

D is the GEMM's own output (FP32 accumulation in an order the oracle does not reproduce), so it
is checked against the oracle's FP64 product within the usual tolerance; every quantity derived
from D -- its two maxima, its quantized operands -- is a function of D's bits, so the oracle
computes the expected value of each from those same bits:
* D is bit-identical to nvfp4_gemm's bf16 output and matches the oracle's FP64 product;
* the fused maxima equal, bit for bit, the oracle's amax of D and of its random Hadamard
  transform along the rows (and the quantizer's own amax pass on D);
* quantizing D with the fused maxima (NVFP4_AMAX_GIVEN) gives exactly the codes, scales and
  amax of the quantization that runs its amax pass, and of the oracle's quantization of D."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import assert_gemm_close, assert_quantized_equal, need_gpu, to_device_bf16

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def _operands(M, N, K, seed):
    X = synth.activations((M, K), seed=seed)
    W = synth.weights((N, K), seed=seed)
    qa, _ = B.quantize(to_device_bf16(X), B.ROWWISE)
    qb, _ = B.quantize(to_device_bf16(W), B.ROWWISE | B.BLOCK2D)
    return X, W, qa, qb


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (192, 320, 320), (1024, 2048, 1024)])
def test_fused_maxima_equal_the_quantizers_amax(M, N, K):
    X, W, qa, qb = _operands(M, N, K, seed=50)
    mask = oracle.sign_mask_from_seed(50)
    D, amax = B.gemm_amax(qa, qb, mask)
    D_plain = B.gemm(qa, qb, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(D.view(torch.int16), D_plain.view(torch.int16))
    D_ref, norm = oracle.gemm_ref(*oracle.fprop_operands(X, W))
    assert_gemm_close(D.float().cpu().numpy(), D_ref, norm, bf16=True, what="gemm_amax D")
    qr, qc = B.quantize_row_rht(D, mask, 0)
    got = amax.cpu().numpy().view(np.uint32)
    want = np.array([qr.amax.item(), qc.amax.item()], dtype=np.float32).view(np.uint32)
    assert np.array_equal(got, want), (got, want)
    # the oracle's maxima of the same bf16 bits: max |D| and max |RHT(D)| with 16-row blocks
    D_bits = D.view(torch.int16).cpu().numpy().view(np.uint16)
    plain, st0 = oracle.amax(D_bits)
    rht, st1 = oracle.amax(D_bits, transpose=True, rht=True, sign_mask=mask)
    assert st0 == 0 and st1 == 0
    want_oracle = np.array([plain, rht], dtype=np.float32).view(np.uint32)
    assert np.array_equal(got, want_oracle), (got, want_oracle)


@pytest.mark.parametrize("sr", [False, True])
def test_quantizing_with_the_fused_maxima_changes_nothing(sr):
    _, _, qa, qb = _operands(512, 1024, 768, seed=51)
    mask = oracle.sign_mask_from_seed(51)
    D, amax = B.gemm_amax(qa, qb, mask)
    flags = B.SR if sr else 0
    want_r, want_c = B.quantize_row_rht(D, mask, flags, seed=9, offset=4)
    got_r, got_c = B.QuantizedTensor(*D.shape), B.QuantizedTensor(D.shape[1], D.shape[0])
    got_r.amax.copy_(amax[0:1])
    got_c.amax.copy_(amax[1:2])
    B.quantize_row_rht(D, mask, flags | B.AMAX_GIVEN, seed=9, offset=4, out_row=got_r,
                       out_col=got_c)
    for got, want in ((got_r, want_r), (got_c, want_c)):
        assert torch.equal(got.codes, want.codes)
        assert torch.equal(got.scales, want.scales)
        assert torch.equal(got.amax, want.amax)


def test_gemm_amax_rejects_a_null_amax_buffer():
    _, _, qa, qb = _operands(256, 256, 256, seed=52)
    out = torch.empty((256, 256), dtype=torch.bfloat16, device="cuda")
    oa, ob = qa.operand(), qb.operand()
    st = B.lib().nvfp4_gemm_amax(ctypes.byref(oa), ctypes.byref(ob),
                                 ctypes.c_void_p(out.data_ptr()), 256, 0, None, None, None)
    assert st == B.ERR_NULL


@pytest.mark.parametrize("T,I,O", [(256, 512, 384), (1024, 2048, 1536)])
def test_dgrad_quantized_equals_the_unfused_sequence(T, I, O):
    """nvfp4_linear_dgrad_quantized = nvfp4_linear_dgrad (bf16) then nvfp4_quantize_row_rht
    (SR) of its dX, bit for bit: dX, both operands' codes and scales, and their amax."""
    dY = synth.gradients((T, O), seed=53)
    W = synth.weights((O, I), seed=53)
    dYd, Wd = to_device_bf16(dY), to_device_bf16(W)
    mask = oracle.sign_mask_from_seed(53)
    dX_ref = B.linear_dgrad(dYd, Wd, 3, 1, out_dtype=torch.bfloat16)
    qr_ref, qc_ref = B.quantize_row_rht(dX_ref, mask, B.SR, seed=11, offset=5)
    dX, qr, qc = B.linear_dgrad_quantized(dYd, Wd, 3, 1, mask, 11, 5)
    torch.cuda.synchronize()
    assert torch.equal(dX.view(torch.int16), dX_ref.view(torch.int16))
    for got, want in ((qr, qr_ref), (qc, qc_ref)):
        assert torch.equal(got.codes, want.codes)
        assert torch.equal(got.scales, want.scales)
        assert torch.equal(got.amax, want.amax)
    D_ref, norm = oracle.gemm_ref(*oracle.dgrad_operands(dY, W, 3, 1))
    assert_gemm_close(dX.float().cpu().numpy(), D_ref, norm, bf16=True, what="dgrad_quantized dX")
    # dX's operands against the oracle's quantization of dX's bits: row-wise SR on stream
    # next_offset, RHT'd column-wise SR on stream next_offset + 1
    dX_bits = dX.view(torch.int16).cpu().numpy().view(np.uint16)
    assert_quantized_equal(qr, oracle.quantize(dX_bits, sr=True, seed=11, offset=5), "dX row")
    assert_quantized_equal(qc, oracle.quantize(dX_bits, transpose=True, rht=True,
                                               sign_mask=mask, sr=True, seed=11, offset=6),
                           "dX col")


def test_dgrad_quantized_rejects_bad_operands():
    T, I, O = 256, 512, 384
    dYd = to_device_bf16(synth.gradients((T, O), seed=54))
    Wd = to_device_bf16(synth.weights((O, I), seed=54))
    with pytest.raises(B.NVFP4Error) as e:
        B.linear_dgrad_quantized(dYd, Wd, 0, 0, 0, 0, 0, out_col=B.QuantizedTensor(T, I))
    assert e.value.status == B.ERR_SHAPE
    dX = torch.empty((T, I), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((B.linear_workspace_bytes(T, I, O),), dtype=torch.uint8, device="cuda")
    oc = B.QuantizedTensor(I, T).operand()
    st = B.lib().nvfp4_linear_dgrad_quantized(
        ctypes.c_void_p(dYd.data_ptr()), ctypes.c_void_p(Wd.data_ptr()), T, I, O, 0, 0,
        ctypes.c_void_p(dX.data_ptr()), 0, 0, 0, None, ctypes.byref(oc),
        ctypes.c_void_p(ws.data_ptr()), None, None)
    assert st == B.ERR_NULL
