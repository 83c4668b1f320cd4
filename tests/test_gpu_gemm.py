"""GPU parity of the block-scaled FP4 GEMM: the oracle's quantized operands are uploaded
as they are (codes, scales in the MMA layout, amax) and D = A . B^T is compared with the
oracle's FP64 dot products of the dequantized operands, within 1e-3 of
||A[m,:]|| * ||B[n,:]||."""
import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import assert_gemm_close, need_gpu, upload_quantized

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
