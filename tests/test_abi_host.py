"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function
include/nvfp4.h declares, sizes its buffers as documented, and rejects invalid arguments
before queueing any work."""
import contextlib
import ctypes

import numpy as np
import pytest
import torch

import oracle
from nvfp4_testlib import sf_offsets, swizzle, unswizzle

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding


def test_library_exports_every_declared_function():
    names = B.declared_functions()
    assert len(names) >= 14
    L = B.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    for n in ("nvfp4_quantize", "nvfp4_rht_quantize", "nvfp4_gemm", "nvfp4_linear_fprop",
              "nvfp4_linear_dgrad", "nvfp4_linear_wgrad"):
        assert n in names


def test_version_and_status_strings():
    assert B.lib().nvfp4_version() >= 100
    for s in range(9):
        assert B.lib().nvfp4_status_string(s)


def test_buffer_sizes():
    assert B.codes_bytes(256, 512) == 256 * 256
    assert B.scales_bytes(256, 512) == 256 * 32
    assert B.scales_bytes(272, 320) == 384 * 20  # rows padded to 128
    assert B.scales_bytes(16, 48) == 0           # K not a multiple of 64
    assert B.workspace_bytes(4096, 4096, 0) >= 4 * 148
    assert B.workspace_bytes(4096, 4096, B.AMAX_GIVEN) == 0
    T, I, O = 256, 512, 384
    need = 0
    for ra, ca, rb, cb in ((T, I, O, I), (T, O, I, O), (O, T, I, T)):
        need = max(need, ra * ca // 2 + B.scales_bytes(ra, ca) + rb * cb // 2 +
                   B.scales_bytes(rb, cb))
    assert B.linear_workspace_bytes(T, I, O) >= need
    assert B.linear_workspace_bytes(100, 512, 384) == 0


def test_sign_mask_helper_matches_oracle():
    for seed in (0, 1, 2, 3, 4, 12345678901234567):
        assert B.sign_mask_from_seed(seed) == oracle.sign_mask_from_seed(seed)


def test_scale_layout_helper():
    rows, cols = 272, 320
    plain = np.random.default_rng(0).integers(0, 127, (rows, cols // 16), dtype=np.uint8)
    sw = swizzle(plain, rows, cols)
    assert np.array_equal(B.scales_unswizzle(sw, rows, cols), plain)
    assert np.array_equal(unswizzle(sw, rows, cols), plain)
    offs = sf_offsets(rows, cols)
    assert len(np.unique(offs)) == offs.size           # a bijection onto its image
    assert offs[0, 0] == 0 and offs[1, 0] == 16 and offs[32, 0] == 4 and offs[0, 1] == 1
    assert offs[0, 4] == 512 and offs[128, 0] == 512 * (cols // 64)


class _FakeOp(ctypes.Structure):
    _fields_ = B.Operand._fields_


def _op(rows, cols, base=0x10000):
    return B.Operand(base, base + 0x100000, base + 0x200000, rows, cols)


@pytest.mark.parametrize("case,expected", [
    ("null_x", B.ERR_NULL),
    ("no_outputs", B.ERR_ARG),
    ("2d_with_sr", B.ERR_ARG),
    ("bad_flag", B.ERR_ARG),
    ("rows_not_16", B.ERR_SHAPE),
    ("row_cols_not_64", B.ERR_SHAPE),
    ("col_rows_not_64", B.ERR_SHAPE),
    ("ld_small", B.ERR_SHAPE),
    ("ld_odd", B.ERR_ALIGN),
    ("x_misaligned", B.ERR_ALIGN),
    ("out_shape", B.ERR_SHAPE),
    ("out_null_codes", B.ERR_NULL),
    ("no_workspace", B.ERR_NULL),
    ("empty", B.ERR_SHAPE),
    ("negative_cols", B.ERR_SHAPE),
    ("too_large", B.ERR_SHAPE),
])
def test_quantize_argument_validation(case, expected):
    L = B.lib()
    x = ctypes.c_void_p(0x1000)
    rows, cols, ld, flags = 256, 512, 512, B.ROWWISE
    out_row = _op(256, 512)
    ws = ctypes.c_void_p(0x8000)
    if case == "null_x":
        x = None
    elif case == "no_outputs":
        flags = B.SR
    elif case == "2d_with_sr":
        flags = B.ROWWISE | B.BLOCK2D | B.SR
    elif case == "bad_flag":
        flags = B.ROWWISE | 64
    elif case == "rows_not_16":
        rows = 250
    elif case == "row_cols_not_64":
        cols, ld, out_row = 336, 336, _op(256, 336)
    elif case == "col_rows_not_64":
        flags = B.COLWISE
        rows = 272
    elif case == "ld_small":
        ld = 500
    elif case == "ld_odd":
        ld = 516
    elif case == "x_misaligned":
        x = ctypes.c_void_p(0x1008)
    elif case == "out_shape":
        out_row = _op(128, 512)
    elif case == "out_null_codes":
        out_row = B.Operand(0, 0x2000, 0x3000, 256, 512)
    elif case == "no_workspace":
        ws = None
    elif case == "empty":
        rows, out_row = 0, _op(0, 512)
    elif case == "negative_cols":
        cols, out_row = -512, _op(256, -512)
    elif case == "too_large":
        rows, out_row = 1 << 31, _op(1 << 31, 512)
    out_col = _op(cols, rows) if flags & B.COLWISE else None
    st = L.nvfp4_quantize(x, rows, cols, ld, flags, 0, 0,
                          ctypes.byref(out_row) if flags & B.ROWWISE else None,
                          ctypes.byref(out_col) if out_col is not None else None, ws, None, None)
    assert st == expected


def test_rht_quantize_rejects_rowwise_flags():
    L = B.lib()
    out = _op(512, 256)
    st = L.nvfp4_rht_quantize(ctypes.c_void_p(0x1000), 256, 512, 512, 0x1234, B.ROWWISE, 0, 0,
                              ctypes.byref(out), ctypes.c_void_p(0x8000), None, None)
    assert st == B.ERR_ARG


@pytest.mark.parametrize("case,expected", [
    ("k_mismatch", B.ERR_SHAPE), ("k_not_64", B.ERR_SHAPE), ("m_not_16", B.ERR_SHAPE),
    ("ldd_small", B.ERR_SHAPE), ("ldd_unaligned", B.ERR_ALIGN), ("dtype", B.ERR_ARG),
    ("null_d", B.ERR_NULL), ("m_zero", B.ERR_SHAPE), ("k_too_large", B.ERR_SHAPE)])
def test_gemm_argument_validation(case, expected):
    L = B.lib()
    A, Bo = _op(256, 512), _op(384, 512, base=0x400000)
    D, ldd, dt = ctypes.c_void_p(0x9000), 384, B.OUT_F32
    if case == "k_mismatch":
        Bo = _op(384, 448, base=0x400000)
    elif case == "k_not_64":
        A, Bo = _op(256, 96), _op(384, 96, base=0x400000)
    elif case == "m_not_16":
        A = _op(250, 512)
    elif case == "ldd_small":
        ldd = 300
    elif case == "ldd_unaligned":
        ldd = 386
    elif case == "dtype":
        dt = 7
    elif case == "null_d":
        D = None
    elif case == "m_zero":
        A = _op(0, 512)
    elif case == "k_too_large":
        A, Bo = _op(256, 1 << 31), _op(384, 1 << 31, base=0x400000)
    assert L.nvfp4_gemm(ctypes.byref(A), ctypes.byref(Bo), D, dt, ldd, None, None) == expected


def test_gemm_amax_argument_validation():
    """nvfp4_gemm_amax: bf16 output only, a 4-byte-aligned amax_out pair, the GEMM's shape
    rules; a valid call without a GPU fails with a CUDA/device status, never a crash."""
    L = B.lib()
    A, Bo = _op(256, 512), _op(384, 512, base=0x400000)
    D, amax = ctypes.c_void_p(0x9000), ctypes.c_void_p(0xA000)
    assert L.nvfp4_gemm_amax(ctypes.byref(A), ctypes.byref(Bo), D, 384, 0, None, None,
                             None) == B.ERR_NULL
    assert L.nvfp4_gemm_amax(ctypes.byref(A), ctypes.byref(Bo), D, 384, 0,
                             ctypes.c_void_p(0xA002), None, None) == B.ERR_ALIGN
    # bf16 rows: ldd * 2 bytes must be a multiple of 16
    assert L.nvfp4_gemm_amax(ctypes.byref(A), ctypes.byref(Bo), D, 388, 0, amax, None,
                             None) == B.ERR_ALIGN
    assert L.nvfp4_gemm_amax(ctypes.byref(A), ctypes.byref(_op(384, 448, base=0x400000)), D,
                             384, 0, amax, None, None) == B.ERR_SHAPE
    assert L.nvfp4_gemm_amax(ctypes.byref(A), ctypes.byref(Bo), D, 384, 0x1234, amax, None,
                             None) in (B.ERR_CUDA, B.ERR_DEVICE)


def test_dgrad_quantized_argument_validation():
    L = B.lib()
    p = ctypes.c_void_p(0x1000)
    assert L.nvfp4_linear_dgrad_quantized(p, p, 256, 512, 384, 0, 0, p, 0, 0, 0, None, None,
                                          None, None, None) == B.ERR_NULL
    assert L.nvfp4_linear_dgrad_quantized(p, p, 100, 512, 384, 0, 0, p, 0, 0, 0, None, None,
                                          p, None, None) == B.ERR_SHAPE


def test_gemm_mx_argument_validation():
    L = B.lib()
    A, Bo = _op(256, 512), _op(384, 512, base=0x400000)
    D = ctypes.c_void_p(0x9000)
    assert L.nvfp4_gemm_mx(ctypes.byref(A), ctypes.byref(_op(384, 96, base=0x400000)), D,
                           B.OUT_F32, 384, None, None) == B.ERR_SHAPE
    assert L.nvfp4_gemm_mx(ctypes.byref(A), ctypes.byref(Bo), None, B.OUT_F32, 384, None,
                           None) == B.ERR_NULL
    assert L.nvfp4_gemm_mx(ctypes.byref(A), ctypes.byref(Bo), D, 5, 384, None,
                           None) == B.ERR_ARG


def test_linear_argument_validation():
    L = B.lib()
    p = ctypes.c_void_p(0x1000)
    assert L.nvfp4_linear_fprop(p, p, 100, 512, 512, p, 0, p, None, None) == B.ERR_SHAPE
    assert L.nvfp4_linear_dgrad(p, p, 256, 512, 512, 0, 0, p, 9, p, None, None) == B.ERR_ARG
    assert L.nvfp4_linear_wgrad(p, p, 256, 512, 512, 0, 0, 0, None, 0, p, None, None) == B.ERR_NULL


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_valid_call_without_gpu_fails_cleanly():
    L = B.lib()
    out = _op(256, 512)
    st = L.nvfp4_quantize(ctypes.c_void_p(0x1000), 256, 512, 512, B.ROWWISE, 0, 0,
                          ctypes.byref(out), None, ctypes.c_void_p(0x8000), None, None)
    assert st in (B.ERR_CUDA, B.ERR_DEVICE)


def test_binding_rejects_bad_output_tensors_before_calling():
    A = B.QuantizedTensor(128, 256, device="cpu")
    Bq = B.QuantizedTensor(256, 256, device="cpu")
    with pytest.raises(TypeError):
        B.gemm(A, Bq, out=torch.empty((128, 256), dtype=torch.float16))
    with pytest.raises(ValueError):
        B.gemm(A, Bq, out=torch.empty((128, 200), dtype=torch.float32))
    with pytest.raises(ValueError):  # host tensor
        B.gemm(A, Bq, out=torch.empty((128, 256), dtype=torch.bfloat16))


def test_wait_selftest_rejects_a_null_status_word():
    # argument checks come before any device access
    assert B.lib().nvfp4_selftest_wait_timeout(None, None) == B.ERR_NULL


def test_checked_build_exports_the_same_functions_and_says_it_is_checked():
    names = B.declared_functions()
    assert "nvfp4_bounds_checked" in names and "nvfp4_selftest_bounds" in names
    assert B.lib().nvfp4_bounds_checked() == 0
    with B.bounds_checked() as L:
        assert L is B.lib()
        missing = [n for n in names if not hasattr(L, n)]
        assert not missing, missing
        assert L.nvfp4_bounds_checked() == 1
        assert B.is_bounds_checked()
    # the block routes calls only while it is open
    assert not B.is_bounds_checked()


def test_bounds_selftest_argument_checks():
    # the normal build refuses before any device access; the checked build checks the
    # status word before any device access
    assert B.lib().nvfp4_selftest_bounds(ctypes.c_void_p(0x1000), None) == B.ERR_ARG
    with B.bounds_checked() as L:
        assert L.nvfp4_selftest_bounds(None, None) == B.ERR_NULL
        assert L.nvfp4_selftest_bounds(ctypes.c_void_p(0x1002), None) == B.ERR_ALIGN


def test_checked_build_rejects_invalid_arguments_like_the_normal_one():
    out = _op(256, 512)
    for lib_ctx in (contextlib.nullcontext(B.lib()), B.bounds_checked()):
        with lib_ctx as L:
            # cols not a multiple of 64, and a flag combination the API refuses
            assert L.nvfp4_quantize(ctypes.c_void_p(0x1000), 256, 520, 520, B.ROWWISE, 0, 0,
                                    ctypes.byref(out), None, ctypes.c_void_p(0x8000), None,
                                    None) == B.ERR_SHAPE
            assert L.nvfp4_quantize(ctypes.c_void_p(0x1000), 256, 512, 512,
                                    B.BLOCK2D | B.SR | B.ROWWISE, 0, 0, ctypes.byref(out), None,
                                    ctypes.c_void_p(0x8000), None, None) == B.ERR_ARG
