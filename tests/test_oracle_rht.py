"""Pins of the oracle's 16x16 random Hadamard transform: Sylvester closed form,
orthogonality (H H^T = 16 I), agreement of the butterflies with the dense product, and the
weight-gradient identity that makes the transform free for dW = dY^T X."""
import numpy as np

import oracle


def _matrix(mask):
    """Column j = oracle transform of the unit vector e_j."""
    M = np.zeros((16, 16))
    for j in range(16):
        e = np.zeros(16, dtype=np.float32)
        e[j] = 1.0
        M[:, j] = oracle.rht16(e, mask)
    return M


def _sylvester():
    i = np.arange(16)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


def test_rht_is_sylvester_hadamard_times_signs_over_4():
    H = _sylvester()
    for mask in (0x0000, 0xFFFF, 0xA5C3, 0x0001, 0x8000):
        D = np.diag([-1.0 if (mask >> j) & 1 else 1.0 for j in range(16)])
        assert np.array_equal(_matrix(mask), H @ D / 4.0)


def test_hadamard_h_ht_is_16_identity():
    mask = 0x3C5A
    D = np.diag([-1.0 if (mask >> j) & 1 else 1.0 for j in range(16)])
    H = 4.0 * _matrix(mask) @ D  # strip the signs: D D = I
    assert np.array_equal(H @ H.T, 16.0 * np.eye(16))
    assert np.array_equal(np.abs(H), np.ones((16, 16)))


def test_rht_is_orthonormal():
    M = _matrix(0x9F31)
    assert np.array_equal(M @ M.T, np.eye(16))


def test_butterflies_equal_dense_product():
    rng = np.random.default_rng(5)
    M = _matrix(0x1234)
    for _ in range(200):
        # small integers: every FP32 sum is exact, so the result must match exactly
        x = rng.integers(-1000, 1000, 16).astype(np.float32)
        assert np.array_equal(oracle.rht16(x, 0x1234).astype(np.float64), M @ x)
    for _ in range(200):
        x = (rng.standard_normal(16) * 10.0 ** rng.uniform(-5, 5)).astype(np.float32)
        y = oracle.rht16(x, 0x1234).astype(np.float64)
        ref = M @ x.astype(np.float64)
        # four FP32 butterfly stages: error below 4 * 2^-24 * sum|x| / 4 (plus slack)
        assert np.all(np.abs(y - ref) <= 1.5 * 2.0 ** -24 * np.abs(x).sum() + 1e-45)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-6 * np.linalg.norm(x)


def test_rht_spreads_a_spike_evenly():
    for j in (0, 7, 15):
        x = np.zeros(16, dtype=np.float32)
        x[j] = 64.0
        y = oracle.rht16(x, 0xBEEF)
        assert np.array_equal(np.abs(y), np.full(16, 16.0, dtype=np.float32))


def test_wgrad_identity_in_fp64():
    # (R dY)^T (R X) = dY^T X for R = blockdiag of the orthonormal 16x16 transform along
    # tokens: the random transform of the two wgrad inputs cancels in the product
    rng = np.random.default_rng(9)
    T, O, I = 64, 24, 40
    dY = rng.standard_normal((T, O))
    X = rng.standard_normal((T, I))
    M = _matrix(oracle.sign_mask_from_seed(1))
    R = np.kron(np.eye(T // 16), M)
    lhs = (R @ dY).T @ (R @ X)
    assert np.allclose(lhs, dY.T @ X, rtol=1e-12, atol=1e-12)


def _kurtosis(v):
    v = np.asarray(v, dtype=np.float64).ravel()
    d = v - v.mean()
    return float((d ** 4).mean() / (d ** 2).mean() ** 2)


def test_rht_spreads_the_outliers_of_spiky_gradients():
    # The wgrad transform exists to spread outliers toward a Gaussian-like spread
    # (Pretraining Large Language Models with NVFP4, Resumen tecnico section 2, RHT bullet).
    # On the recipe's spiky gradients (0.5 % of values x100) and outlier activations (1 % x50)
    # the 16-point transform along the tokens divides the kurtosis by roughly 16: each spike's
    # energy lands on all 16 outputs of its block.
    import synth
    for seed, gen in ((0, synth.gradients), (1, synth.gradients), (2, synth.activations)):
        x = gen((512, 128), seed=seed)
        blocks = synth.bf16_bits_to_f32(x).T.reshape(-1, 16).astype(np.float32)
        mask = oracle.sign_mask_from_seed(seed)
        y = np.stack([oracle.rht16(b, mask) for b in blocks])
        before, after = _kurtosis(blocks), _kurtosis(y)
        assert before > 100.0, before
        assert after < before / 8.0, (before, after)
        # energy is kept block by block (orthonormal transform)
        assert np.allclose((y.astype(np.float64) ** 2).sum(1),
                           (blocks.astype(np.float64) ** 2).sum(1), rtol=1e-5)
