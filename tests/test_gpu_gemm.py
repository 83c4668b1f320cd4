"""GPU parity of the block-scaled FP4 GEMM: the oracle's quantized operands are uploaded
as they are (codes, scales in the MMA layout, amax) and D = A . B^T is compared with the
oracle's FP64 dot products of the dequantized operands, within 1e-3 of
||A[m,:]|| * ||B[n,:]||."""
import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import (assert_gemm_close, assert_quantized_equal, need_gpu,
                           to_device_bf16, upload_quantized)

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def _operands(M, N, K, seed=0, sr=False):
    X = synth.activations((M, K), seed=seed)
    W = synth.weights((N, K), seed=seed)
    qa = oracle.quantize(X, sr=sr, seed=seed)
    qb = oracle.quantize(W, block2d=(N % 16 == 0 and K % 16 == 0))
    return qa, qb


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 64),      # one tile, one MMA step
    (128, 256, 256),     # one tile, one full stage
    (256, 512, 512),     # 2 x 2 tiles
    (144, 272, 320),     # ragged M, N and K (5 MMA steps: a partial last stage)
    (16, 16, 64),        # smallest shape
    (1024, 1536, 2048),  # many tiles, several k blocks per tile
    (384, 768, 4160),    # long K with a ragged last stage
    (1344, 320, 512),    # more rows than columns: raster groups of 4 row tiles, a short last group
    (20480, 528, 256),   # 240 pair tiles over the persistent grid, groups of 4, ragged N
])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gemm_matches_oracle(M, N, K, dtype):
    qa, qb = _operands(M, N, K, seed=M + N + K)
    A, Bq = upload_quantized(qa, B), upload_quantized(qb, B)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    D = B.gemm(A, Bq, out_dtype=dtype, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    D_ref, norm = oracle.gemm_ref(qa, qb)
    assert_gemm_close(D.float().cpu().numpy(), D_ref, norm, bf16=(dtype == torch.bfloat16),
                      what=f"{M}x{N}x{K}")


def test_gemm_output_leading_dimension():
    qa, qb = _operands(256, 256, 512, seed=3)
    A, Bq = upload_quantized(qa, B), upload_quantized(qb, B)
    big = torch.full((256, 400), 7.0, dtype=torch.float32, device="cuda")
    B.gemm(A, Bq, out=big[:, :256].as_strided((256, 256), (400, 1)))
    D_ref, norm = oracle.gemm_ref(qa, qb)
    out = big.cpu().numpy()
    assert_gemm_close(out[:, :256], D_ref, norm)
    assert np.all(out[:, 256:] == 7.0)  # nothing written beyond N


def test_gemm_config_4096_cubed_full_check():
    """One GEMM at the one-layer shape T = I = O = 4096, every entry checked."""
    qa, qb = _operands(4096, 4096, 4096, seed=1)
    D = B.gemm(upload_quantized(qa, B), upload_quantized(qb, B))
    D_ref, norm = oracle.gemm_ref(qa, qb)
    assert_gemm_close(D.cpu().numpy(), D_ref, norm, what="4096^3")


def test_gemm_zero_and_nonfinite_amax():
    qa, qb = _operands(128, 256, 256, seed=2)
    A, Bq = upload_quantized(qa, B), upload_quantized(qb, B)
    A.codes.zero_()
    A.scales.zero_()
    A.amax.fill_(float("inf"))  # a non-finite tensor: quantizer wrote zeros and amax = inf
    D = B.gemm(A, Bq)
    assert torch.count_nonzero(D).item() == 0
    A.amax.fill_(0.0)
    D = B.gemm(A, Bq)
    assert torch.count_nonzero(D).item() == 0


def test_gemm_is_deterministic():
    qa, qb = _operands(512, 512, 1024, seed=4)
    A, Bq = upload_quantized(qa, B), upload_quantized(qb, B)
    d1 = B.gemm(A, Bq)
    d2 = B.gemm(A, Bq)
    assert torch.equal(d1, d2)


def _scaled(bits, k):
    """bf16 values times 2^k, exactly (every value stays a normal number or zero)."""
    return synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(bits) * np.float32(2.0 ** k))


@pytest.mark.parametrize("ka,kb", [(-60, -60), (-70, -45), (-95, -25)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gemm_extreme_amax(ka, kb, dtype):
    """Operands whose tensor scales multiply beyond FP32 (S_A * S_B > FLT_MAX): inputs scaled
    by tiny powers of two, quantized by the GPU (bit-exact with the oracle) and multiplied.
    The decode factor 1 / (S_A S_B) must not collapse to 0: D is compared entry by entry with
    the oracle's FP64 products of the dequantized operands."""
    M, N, K = 256, 512, 512
    X = _scaled(synth.activations((M, K), seed=70), ka)
    W = _scaled(synth.weights((N, K), seed=70), kb)
    qa_ref, qb_ref = oracle.quantize(X), oracle.quantize(W, block2d=True)
    # the extreme case: the product of the two FP32 encode scales exceeds FLT_MAX
    assert oracle.tensor_scale(qa_ref.amax) * oracle.tensor_scale(qb_ref.amax) > 3.4028235e38
    qa, _ = B.quantize(to_device_bf16(X), B.ROWWISE)
    qb, _ = B.quantize(to_device_bf16(W), B.ROWWISE | B.BLOCK2D)
    assert_quantized_equal(qa, qa_ref, "A")
    assert_quantized_equal(qb, qb_ref, "B")
    D = B.gemm(qa, qb, out_dtype=dtype)
    D_ref, norm = oracle.gemm_ref(qa_ref, qb_ref)
    assert np.abs(D_ref).max() > 0
    assert_gemm_close(D.float().cpu().numpy(), D_ref, norm, bf16=(dtype == torch.bfloat16),
                      what=f"2^{ka} x 2^{kb}")


@pytest.mark.parametrize("amax_a,amax_b,sf_hi", [
    (2.0 ** 75.5, 2.0 ** 75.5, 4),      # S_A * S_B below FP32's normal range: 1/x overflows
    (2.0 ** -60, 2.0 ** -60, 0x7E),     # S_A * S_B above FLT_MAX
    (2.0 ** -126, 3.0e38, 0x7E),        # far apart, product ordinary
    (1.0e-40, 1.0e-40, 0x7E),           # subnormal amax: both scales clamp to FLT_MAX
])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gemm_decode_factor_over_the_whole_amax_range(amax_a, amax_b, sf_hi, dtype):
    """The GEMM's contract for arbitrary operands: D = sum_k deq(A) deq(B) with deq = e2m1 x
    sf / S_enc(amax).  Random codes, random scale bytes in [1, sf_hi] and a chosen amax per
    operand, against the oracle's FP64 product."""
    rng = np.random.default_rng(71)
    M, N, K = 128, 256, 256

    def operand(rows, amax):
        codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
        scales = rng.integers(1, sf_hi + 1, size=(rows, K // 16), dtype=np.uint8)
        return oracle.Quantized(codes, scales, float(np.float32(amax)), 0)

    qa, qb = operand(M, amax_a), operand(N, amax_b)
    D = B.gemm(upload_quantized(qa, B), upload_quantized(qb, B), out_dtype=dtype)
    D_ref, norm = oracle.gemm_ref(qa, qb)
    assert_gemm_close(D.float().cpu().numpy(), D_ref, norm, bf16=(dtype == torch.bfloat16),
                      what=f"amax {amax_a:g} x {amax_b:g}")
