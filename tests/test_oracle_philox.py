"""Pins of the oracle's Philox-4x32-10 generator: the published known-answer vectors and
statistical checks of the bits that drive stochastic rounding."""
import numpy as np

import oracle
from conftest import golden_rows


def test_philox_known_answer_vectors():
    rows = golden_rows("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for row in rows:
        w = [int(t, 16) for t in row]
        ctr, key, want = w[0:4], w[4:6], w[6:10]
        assert oracle.philox4x32_10(ctr, key) == want


def test_sr_bits_lane_layout():
    # lane j of element e = 8g + j is half (j & 1) of word j >> 1 of Philox(ctr = g, offset)
    seed, offset = 0x0123456789ABCDEF, 0x1122334455667788
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for g in (0, 1, 5, (1 << 32) + 3):
        w = oracle.philox4x32_10([g & 0xFFFFFFFF, g >> 32, offset & 0xFFFFFFFF, offset >> 32], key)
        for j in range(8):
            half = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFF
            assert oracle.sr_bits(seed, offset, 8 * g + j) == half


def test_sr_bits_are_uniform():
    seed, offset = 1, 0
    n = 1 << 17
    r = np.array([oracle.sr_bits(seed, offset, e) for e in range(n)], dtype=np.uint32)
    assert r.max() < 65536
    # every bit position is balanced within 5 sigma
    for b in range(16):
        ones = int(((r >> b) & 1).sum())
        assert abs(ones - n / 2) < 5 * np.sqrt(n / 4), b
    # chi-square of the high byte over 256 bins (dof 255): well inside [180, 340]
    hist = np.bincount(r >> 8, minlength=256)
    chi2 = float(((hist - n / 256) ** 2 / (n / 256)).sum())
    assert 180 < chi2 < 340, chi2


def test_sr_bits_depend_on_offset_and_seed():
    a = [oracle.sr_bits(3, 0, e) for e in range(64)]
    b = [oracle.sr_bits(3, 1, e) for e in range(64)]
    c = [oracle.sr_bits(4, 0, e) for e in range(64)]
    assert a != b and a != c


def test_sign_mask_from_seed_is_philox_word():
    for seed in (0, 1, 2, 0xDEADBEEFCAFEF00D):
        w = oracle.philox4x32_10([0, 0, 0, 0xFFFFFFFF], [seed & 0xFFFFFFFF, seed >> 32])
        assert oracle.sign_mask_from_seed(seed) == (w[0] & 0xFFFF)
