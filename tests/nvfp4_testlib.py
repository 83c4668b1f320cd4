"""Helpers shared by the GPU parity tests: moving seeded inputs to the device, the scale
layout documented in include/nvfp4.h (written out here independently of the library), and
the GEMM tolerance check."""
import numpy as np
import pytest
import torch

GEMM_TOL = 1e-3  # |D - D_ref| <= 1e-3 * ||A[m,:]|| * ||B[n,:]|| (FP64 reference)


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip("needs an sm_100 (B200) device")


def to_device_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def sf_offsets(rows: int, cols: int, r=None, j=None) -> np.ndarray:
    """Byte offset of scale (r, j) in the MMA layout: 512-byte tiles of 128 rows x 4 blocks,
    ordered (row tile, block group); inside a tile (r % 32) * 16 + ((r / 32) % 4) * 4 + j % 4.
    All rows x all blocks, or the given row indices r x block indices j."""
    nb = cols // 16
    r = np.arange(rows, dtype=np.int64)[:, None] if r is None else np.asarray(r, np.int64)[:, None]
    j = np.arange(nb, dtype=np.int64)[None, :] if j is None else np.asarray(j, np.int64)[None, :]
    return ((r // 128) * (nb // 4) + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4


def unswizzle(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    return np.asarray(buf, dtype=np.uint8)[sf_offsets(rows, cols)]


def swizzle(plain: np.ndarray, rows: int, cols: int) -> np.ndarray:
    rows_pad = (rows + 127) // 128 * 128
    out = np.zeros(rows_pad * (cols // 16), dtype=np.uint8)
    out[sf_offsets(rows, cols)] = plain
    return out


def padding_is_zero(buf: np.ndarray, rows: int, cols: int) -> bool:
    used = np.zeros(buf.size, dtype=bool)
    used[sf_offsets(rows, cols).ravel()] = True
    return not np.asarray(buf)[~used].any()


def qt_to_host(qt):
    """(codes [R x C/2], row-major scales [R x C/16], amax) of a QuantizedTensor."""
    codes = qt.codes.cpu().numpy()
    scales = unswizzle(qt.scales.cpu().numpy(), qt.rows, qt.cols)
    return codes, scales, float(qt.amax.cpu().item())


def assert_quantized_equal(qt, ref, what=""):
    codes, scales, amax = qt_to_host(qt)
    assert amax == ref.amax or (np.isinf(amax) and np.isinf(ref.amax)), (what, amax, ref.amax)
    bad = np.argwhere(codes != ref.codes)
    assert bad.size == 0, (what, "codes differ at", bad[:5], codes[tuple(bad[0])],
                           ref.codes[tuple(bad[0])])
    bad = np.argwhere(scales != ref.scales)
    assert bad.size == 0, (what, "scales differ at", bad[:5])
    assert padding_is_zero(qt.scales.cpu().numpy(), qt.rows, qt.cols), (what, "padding")


def upload_quantized(ref, binding):
    """A device QuantizedTensor holding the oracle's codes, scales and amax."""
    qt = binding.QuantizedTensor(ref.rows, ref.cols)
    qt.codes.copy_(torch.from_numpy(ref.codes))
    qt.scales.copy_(torch.from_numpy(swizzle(ref.scales, ref.rows, ref.cols)))
    qt.amax.fill_(ref.amax)
    return qt


def assert_gemm_close(D_gpu: np.ndarray, D_ref: np.ndarray, norm: np.ndarray, bf16=False,
                      what=""):
    D_gpu = D_gpu.astype(np.float64)
    err = np.abs(D_gpu - D_ref)
    allowed = GEMM_TOL * norm
    if bf16:  # the output is the bf16 rounding of a value within the FP32 tolerance
        allowed = allowed + 2.0 ** -8 * np.abs(D_ref)
    # below the output format's range a result is its nearest subnormal or zero: one quantum
    # of the format's subnormals (2^-149 in FP32, 2^-133 in bf16) is allowed on top
    allowed = allowed + (2.0 ** -133 if bf16 else 2.0 ** -149)
    zero = norm == 0
    assert np.all(D_gpu[zero] == 0), what
    ratio = np.where(zero, 0.0, err / np.where(zero, 1.0, allowed))
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert ratio.max() <= 1.0, (what, "worst", worst, D_gpu[worst], D_ref[worst], norm[worst])
    return float((err / np.where(zero, 1.0, norm)).max())


def host_threads(cap=64):
    """Host cores this process may run on (the oracle's threaded driver uses them)."""
    import os
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(cap, n))


def _dequantize_rows(q, r0, r1, idx=None):
    """FP64 dequantized rows [r0, r1) (or the rows `idx`) of an oracle Quantized operand."""
    import oracle
    if idx is not None:
        sub = oracle.Quantized(np.ascontiguousarray(q.codes[idx]),
                               np.ascontiguousarray(q.scales[idx]), q.amax, q.status)
    else:
        sub = oracle.Quantized(q.codes[r0:r1], q.scales[r0:r1], q.amax, q.status)
    return sub.dequantize()


def gemm_ref_sampled(qa, qb, rows=None, cols=None, chunk=2048):
    """oracle.gemm_ref restricted to the output rows `rows` (all columns) or the output
    columns `cols` (all rows), with the full operand dequantized in chunks of `chunk` rows so
    that the FP64 copies of large operands never exist whole.  Returns (D_ref, norm)."""
    if rows is not None:
        A = _dequantize_rows(qa, 0, 0, idx=rows)
        na = np.sqrt((A * A).sum(axis=1))
        D = np.empty((len(rows), qb.rows), dtype=np.float64)
        nb = np.empty(qb.rows, dtype=np.float64)
        for n0 in range(0, qb.rows, chunk):
            Bc = _dequantize_rows(qb, n0, min(qb.rows, n0 + chunk))
            D[:, n0:n0 + len(Bc)] = A @ Bc.T
            nb[n0:n0 + len(Bc)] = np.sqrt((Bc * Bc).sum(axis=1))
        return D, np.outer(na, nb)
    Bs = _dequantize_rows(qb, 0, 0, idx=cols)
    nb = np.sqrt((Bs * Bs).sum(axis=1))
    D = np.empty((qa.rows, len(cols)), dtype=np.float64)
    na = np.empty(qa.rows, dtype=np.float64)
    for m0 in range(0, qa.rows, chunk):
        Ac = _dequantize_rows(qa, m0, min(qa.rows, m0 + chunk))
        D[m0:m0 + len(Ac)] = Ac @ Bs.T
        na[m0:m0 + len(Ac)] = np.sqrt((Ac * Ac).sum(axis=1))
    return D, np.outer(na, nb)
