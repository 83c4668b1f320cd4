"""The debug build libnvfp4_checked.so (-DNVFP4_BOUNDS_CHECK): every quantizer mode and the
GEMMs run through it on ragged and strided shapes give the oracle's results bit for bit (the
GEMM within its tolerance) and leave NVFP4_DEVSTAT_BOUNDS clear, i.e. no kernel computed a
global access outside its buffer; and its self-test shows that a refused access is recorded
while the context stays usable."""
import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import (assert_gemm_close, assert_quantized_equal, need_gpu, qt_to_host,
                           to_device_bf16)

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _checked():
    need_gpu()
    with B.bounds_checked():
        assert B.is_bounds_checked()
        yield


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _clean(status):
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"


def test_selftest_records_a_refused_store_and_the_context_stays_usable():
    st = _status()
    B.selftest_bounds(st)
    torch.cuda.synchronize()
    assert int(st.item()) == B.DEVSTAT_BOUNDS
    x = synth.activations((256, 512), seed=40)
    st2 = _status()
    qr, _ = B.quantize(to_device_bf16(x), B.ROWWISE, dev_status=st2)
    _clean(st2)
    assert_quantized_equal(qr, oracle.quantize(x), "after the self-test")


@pytest.mark.parametrize("shape", [(272, 320), (48, 64), (1040, 192)])
@pytest.mark.parametrize("sr", [False, True])
def test_rowwise(shape, sr):
    x = synth.gradients(shape, seed=41) if sr else synth.activations(shape, seed=41)
    st = _status()
    flags = B.ROWWISE | (B.SR if sr else 0)
    qr, _ = B.quantize(to_device_bf16(x), flags, seed=3, offset=7, dev_status=st)
    _clean(st)
    assert_quantized_equal(qr, oracle.quantize(x, sr=sr, seed=3, offset=7), "rowwise")


def test_rowwise_strided_input():
    x = synth.activations((272, 448), seed=42)
    xd = to_device_bf16(x)[:, :320]  # rows 448 values apart
    st = _status()
    qr, _ = B.quantize(xd, B.ROWWISE, dev_status=st)
    _clean(st)
    assert_quantized_equal(qr, oracle.quantize(np.ascontiguousarray(x[:, :320])), "strided")


@pytest.mark.parametrize("shape", [(192, 320), (320, 448)])
def test_block2d_both_directions(shape):
    w = synth.weights(shape, seed=43)
    st = _status()
    qr, qc = B.quantize(to_device_bf16(w), B.ROWWISE | B.COLWISE | B.BLOCK2D, dev_status=st)
    _clean(st)
    assert_quantized_equal(qr, oracle.quantize(w, block2d=True), "2d row")
    assert_quantized_equal(qc, oracle.quantize(w, transpose=True, block2d=True), "2d col")


@pytest.mark.parametrize("sr", [False, True])
def test_plain_and_rht_columnwise(sr):
    x = synth.gradients((320, 192), seed=44)
    mask = oracle.sign_mask_from_seed(44)
    st = _status()
    _, qc = B.quantize(to_device_bf16(x), B.COLWISE | (B.SR if sr else 0), seed=2, offset=1,
                       dev_status=st)
    qh = B.rht_quantize(to_device_bf16(x), mask, B.SR if sr else 0, seed=2, offset=1,
                        dev_status=st)
    _clean(st)
    assert_quantized_equal(qc, oracle.quantize(x, transpose=True, sr=sr, seed=2, offset=1),
                           "col")
    assert_quantized_equal(qh, oracle.quantize(x, transpose=True, rht=True, sign_mask=mask,
                                               sr=sr, seed=2, offset=1), "rht col")


@pytest.mark.parametrize("sr", [False, True])
def test_row_and_rht_column_pair(sr):
    x = synth.gradients((320, 448), seed=45)
    xd = to_device_bf16(np.ascontiguousarray(np.pad(x, ((0, 0), (0, 64)))))[:, :448]
    mask = oracle.sign_mask_from_seed(45)
    st = _status()
    qr, qc = B.quantize_row_rht(xd, mask, B.SR if sr else 0, seed=5, offset=3, dev_status=st)
    _clean(st)
    assert_quantized_equal(qr, oracle.quantize(x, sr=sr, seed=5, offset=3), "pair row")
    assert_quantized_equal(qc, oracle.quantize(x, transpose=True, rht=True, sign_mask=mask,
                                               sr=sr, seed=5, offset=4), "pair rht col")


def test_mx_row_and_column():
    x = synth.activations((320, 192), seed=46)
    st = _status()
    qr, qc = B.quantize(to_device_bf16(x), B.ROWWISE | B.COLWISE | B.MX, dev_status=st)
    _clean(st)
    for got, ref in ((qr, oracle.mx_quantize(x)), (qc, oracle.mx_quantize(x, transpose=True))):
        codes, scales, _ = qt_to_host(got)
        assert np.array_equal(codes, ref.codes)
        assert np.array_equal(scales[:, 0::2], ref.scales)
        assert np.array_equal(scales[:, 1::2], ref.scales)


@pytest.mark.parametrize("M,N,K", [(144, 272, 320), (1344, 320, 512)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gemm(M, N, K, dtype):
    X = synth.activations((M, K), seed=47)
    W = synth.weights((N, K), seed=47)
    st = _status()
    qa, _ = B.quantize(to_device_bf16(X), B.ROWWISE, dev_status=st)
    qb, _ = B.quantize(to_device_bf16(W), B.ROWWISE, dev_status=st)
    D = B.gemm(qa, qb, out_dtype=dtype, dev_status=st)
    _clean(st)
    D_ref, norm = oracle.gemm_ref(oracle.quantize(X), oracle.quantize(W))
    assert_gemm_close(D.float().cpu().numpy(), D_ref, norm, bf16=dtype == torch.bfloat16,
                      what=f"checked gemm {M}x{N}x{K}")


def test_linear_layer_and_fused_maxima():
    lin = synth.Linear("checked", 256, 320, 448)
    seed = 48
    X, W, dY = synth.linear_inputs(lin, seed)
    mask = oracle.sign_mask_from_seed(seed)
    Xd, Wd, dYd = to_device_bf16(X), to_device_bf16(W), to_device_bf16(dY)
    st = _status()
    Y = B.linear_fprop(Xd, Wd, dev_status=st)
    dX = B.linear_dgrad(dYd, Wd, seed, 0, dev_status=st)
    dW = B.linear_wgrad(dYd, Xd, mask, seed, 0, dev_status=st)
    qa, qb = oracle.fprop_operands(X, W)
    A, Bq = B.quantize(Xd, B.ROWWISE, dev_status=st)[0], B.quantize(Wd, B.ROWWISE | B.BLOCK2D,
                                                                       dev_status=st)[0]
    D, amax = B.gemm_amax(A, Bq, mask, dev_status=st)
    _clean(st)
    for name, got, (ra, rb) in (("fprop", Y, (qa, qb)),
                                ("dgrad", dX, oracle.dgrad_operands(dY, W, seed, 0)),
                                ("wgrad", dW, oracle.wgrad_operands(dY, X, mask, seed, 0))):
        D_ref, norm = oracle.gemm_ref(ra, rb)
        assert_gemm_close(got.float().cpu().numpy(), D_ref, norm, what=f"checked {name}")
    D_bits = D.view(torch.int16).cpu().numpy().view(np.uint16)
    plain, st0 = oracle.amax(D_bits)
    rht, st1 = oracle.amax(D_bits, transpose=True, rht=True, sign_mask=mask)
    assert st0 == 0 and st1 == 0
    assert amax.cpu().numpy().tolist() == [plain, rht]
