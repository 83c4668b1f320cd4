"""Host checks of the quantizer kernels' exact-arithmetic identities (no GPU).

* div6_rn, the division-free b / 6 the block-scale step uses, equals IEEE b / 6 (round to
  nearest even) on every finite non-negative FP32 value -- all 2^31 - 2^23 patterns.
* The FMA-pipe stochastic rounding (e2m1_sr_code) gives the oracle's SR magnitude code on
  10^8 (a, r16) pairs: grid points and their neighbours, subnormals, values at and above 6,
  r16 in {0, 65535} and random ones.

Both restate the device functions' FP32 operation sequences in C (tests/kernel_identities.c)
and compare them with IEEE division and with the oracle's nvo_e2m1_sr."""
import ctypes
import os
import subprocess
import threading

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def kid(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("kid") / "libkid.so")
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                    "-frounding-math", "-fno-fast-math", "-o", out,
                    os.path.join(HERE, "kernel_identities.c"), "-lm"], check=True)
    L = ctypes.CDLL(out)
    L.kid_div6_mismatches.argtypes = [ctypes.c_uint32, ctypes.c_uint32,
                                      ctypes.POINTER(ctypes.c_uint32)]
    L.kid_div6_mismatches.restype = ctypes.c_int64
    L.kid_sr_codes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    L.kid_sr_codes.restype = None
    return L


def test_div6_rn_is_ieee_division_on_every_finite_non_negative_float(kid):
    end = 0x7F800000  # +Inf: every pattern below it is a finite non-negative float
    nthreads = max(1, min(16, os.cpu_count() or 1))
    bounds = [end * i // nthreads for i in range(nthreads + 1)]
    results = [None] * nthreads

    def work(i):
        first = ctypes.c_uint32(0)
        n = kid.kid_div6_mismatches(bounds[i], bounds[i + 1], ctypes.byref(first))
        results[i] = (n, first.value)

    threads = [threading.Thread(target=work, args=(i,)) for i in range(nthreads)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    bad = [(n, hex(f)) for n, f in results if n]
    assert not bad, bad


def _sr_cases(rng, n):
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    near = []
    for g in grid:
        u = np.float32(g).view(np.uint32).astype(np.int64)
        for d in range(-3, 4):
            if u + d >= 0:
                near.append(np.uint32(u + d).view(np.float32))
    fixed = np.concatenate([
        np.array(near, dtype=np.float32),
        np.array([1e-45, 1e-40, 1e-38, 1.1754942e-38, 7.0, 8.0, 1e6, 3.4e38], dtype=np.float32),
    ])
    a = np.concatenate([
        fixed,
        rng.uniform(0.0, 7.0, n // 2).astype(np.float32),  # the whole grid and above 6
        (rng.integers(0, 0x00800000, n // 8, dtype=np.uint32)).view(np.float32),  # subnormals
        np.float32(2.0) ** rng.uniform(-126, 3, n - n // 2 - n // 8 - fixed.size).astype(
            np.float32),
    ]).astype(np.float32)
    r16 = rng.integers(0, 65536, a.size, dtype=np.uint32)
    r16[: 2 * fixed.size: 2] = 0
    r16[1: 2 * fixed.size: 2] = 65535
    return a, r16


def test_fma_pipe_stochastic_rounding_matches_the_oracle(kid):
    rng = np.random.default_rng(2024)
    total, batch = 0, 10_000_000
    for i in range(10):
        a, r16 = _sr_cases(rng, batch)
        if i == 0:  # every r16 for a few points between grid values, and at them
            pts = np.array([0.25, 0.75, 1.2, 1.75, 2.5, 3.5, 5.0, 5.999, 0.5, 4.0],
                           dtype=np.float32)
            a = np.concatenate([a, np.repeat(pts, 65536)])
            r16 = np.concatenate([r16, np.tile(np.arange(65536, dtype=np.uint32), pts.size)])
        got = np.zeros(a.size, dtype=np.uint8)
        kid.kid_sr_codes(a.ctypes.data, r16.ctypes.data, a.size, got.ctypes.data)
        want = oracle.e2m1_sr_many(a, r16) & 7
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, [(float(a[j]), int(r16[j]), int(got[j]), int(want[j]))
                               for j in bad[:5]]
        total += a.size
    assert total >= 100_000_000
