"""Pins of the oracle's reference GEMM and of the composed linear-layer operands: the plain
FP64 triple loop equals numpy's FP64 matmul, and the quantized layer products stay close to
the unquantized ones (which a wrong scale, a missing transform or a transposed operand
would break)."""
import numpy as np
import pytest

import oracle
import synth


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 128, 512), (128, 256, 256)])
def test_brute_force_loop_equals_numpy_matmul(M, N, K):
    X = synth.activations((M, K), seed=1)
    W = synth.weights((N, K), seed=1)
    qa, qb = oracle.quantize(X), oracle.quantize(W, block2d=True)
    A, B = qa.dequantize(), qb.dequantize()
    D_loop = oracle.gemm_ref_loop(A, B)
    D_np, norm = oracle.gemm_ref(qa, qb)
    assert np.allclose(D_loop, D_np, rtol=1e-12, atol=1e-12 * norm.max())
    assert np.allclose(norm, np.outer(oracle.row_norms(A), oracle.row_norms(B)), rtol=1e-12)


def test_gemm_ref_sampling_matches_full():
    X = synth.activations((64, 128), seed=2)
    W = synth.weights((48, 128), seed=2)
    qa, qb = oracle.quantize(X), oracle.quantize(W)
    D, norm = oracle.gemm_ref(qa, qb)
    rows, cols = np.array([3, 17, 60]), np.array([0, 47, 5])
    Ds, ns = oracle.gemm_ref(qa, qb, rows=rows, cols=cols)
    # BLAS may block the sampled product differently: equal to FP64 rounding
    assert np.allclose(Ds, D[np.ix_(rows, cols)], rtol=1e-13, atol=1e-13 * norm.max())
    assert np.allclose(ns, norm[np.ix_(rows, cols)], rtol=1e-13)


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_linear_layer_products_track_the_unquantized_ones():
    T, I, O = 128, 256, 192
    X, W, dY = synth.linear_inputs(synth.Linear("t", T, I, O), seed=5)
    Xf, Wf, dYf = (synth.bf16_bits_to_f32(a).astype(np.float64) for a in (X, W, dY))
    mask = oracle.sign_mask_from_seed(5)

    qa, qb = oracle.fprop_operands(X, W)
    assert _rel(oracle.gemm_ref(qa, qb)[0], Xf @ Wf.T) < 0.15

    qa, qb = oracle.dgrad_operands(dY, W, seed=5, offset=0)
    assert qb.rows == I and qb.cols == O
    assert _rel(oracle.gemm_ref(qa, qb)[0], dYf @ Wf) < 0.2

    qa, qb = oracle.wgrad_operands(dY, X, mask, seed=5, offset=0)
    assert qa.rows == O and qa.cols == T and qb.rows == I
    # the transform cancels in the product: deq(R dY)^T deq(R X) ~ dY^T X
    assert _rel(oracle.gemm_ref(qa, qb)[0], dYf.T @ Xf) < 0.25
