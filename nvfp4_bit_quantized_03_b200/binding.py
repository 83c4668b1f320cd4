"""ctypes binding of libnvfp4.so (include/nvfp4.h).

Argument marshalling only: PyTorch owns the device memory and the streams; every step of the
quantizers and GEMMs runs in the library's CUDA kernels.  There is no fallback: if the
library is missing or a call fails, an exception is raised.

Inside a ``with bounds_checked():`` block the same calls go to libnvfp4_checked.so, the debug
build whose kernels check every global access against its buffer (NVFP4_DEVSTAT_BOUNDS).
"""
import contextlib
import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")
CHECKED_LIB_PATH = os.path.join(_PKG, "libnvfp4_checked.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "nvfp4.h")

# status codes and flags (include/nvfp4.h)
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_DEVICE, ERR_CUDA, ERR_NONFINITE, ERR_TIMEOUT, ERR_ARG = range(9)
DEVSTAT_NONFINITE, DEVSTAT_TIMEOUT, DEVSTAT_BOUNDS = 1, 2, 4
ROWWISE, COLWISE, BLOCK2D, SR, AMAX_GIVEN, MX = 1, 2, 4, 8, 16, 32
OUT_F32, OUT_BF16 = 0, 1


class NVFP4Error(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {lib().nvfp4_status_string(status).decode()} (status {status})")


class Operand(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("amax", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


_libs = {}               # path -> configured CDLL
_active = LIB_PATH       # the library calls go to
_poison = False


def set_output_poisoning(enabled: bool):
    """Debug aid for tests: when enabled, every output buffer this module allocates is first
    filled with a pattern no kernel writes (codes and scales 0xFF bytes, FP32 / bf16 results and
    amax NaN; workspaces 0xFF bytes), so that a kernel that leaves part of its output unwritten,
    or reads scratch it did not write, cannot pass a check by finding an earlier, identical
    result in recycled memory."""
    global _poison
    _poison = bool(enabled)


def _poisoned(t):
    if _poison:
        if t.dtype == torch.uint8:
            t.fill_(0xFF)
        else:
            t.fill_(float("nan"))
    return t


def lib():
    """The library calls go to: libnvfp4.so, or libnvfp4_checked.so inside bounds_checked()
    (raises if it has not been built)."""
    L = _libs.get(_active)
    if L is None:
        L = _libs[_active] = _open(_active)
    return L


@contextlib.contextmanager
def bounds_checked():
    """Route every call of this module made inside the block to libnvfp4_checked.so (the
    -DNVFP4_BOUNDS_CHECK build: an out-of-extent global access is skipped and sets
    NVFP4_DEVSTAT_BOUNDS in the call's status word).  Yields that library.  The switch is
    process-wide, not per thread: other threads' calls inside the block go there too."""
    global _active
    prev = _active
    _active = CHECKED_LIB_PATH
    try:
        yield lib()
    finally:
        _active = prev


def _open(path):
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not found at {path}; build it with "
                          "`python -m nvfp4_bit_quantized_03_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(path)
    i64, u64, u16, vp, i32 = (ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint16,
                              ctypes.c_void_p, ctypes.c_int)
    op = ctypes.POINTER(Operand)
    sz = ctypes.c_size_t
    L.nvfp4_version.argtypes, L.nvfp4_version.restype = [], i32
    L.nvfp4_status_string.argtypes, L.nvfp4_status_string.restype = [i32], ctypes.c_char_p
    L.nvfp4_codes_bytes.argtypes, L.nvfp4_codes_bytes.restype = [i64, i64], sz
    L.nvfp4_scales_bytes.argtypes, L.nvfp4_scales_bytes.restype = [i64, i64], sz
    L.nvfp4_workspace_bytes.argtypes = [i64, i64, ctypes.c_uint]
    L.nvfp4_workspace_bytes.restype = sz
    L.nvfp4_linear_workspace_bytes.argtypes = [i64, i64, i64]
    L.nvfp4_linear_workspace_bytes.restype = sz
    L.nvfp4_sign_mask_from_seed.argtypes, L.nvfp4_sign_mask_from_seed.restype = [u64], u16
    L.nvfp4_scales_unswizzle.argtypes = [vp, i64, i64, vp]
    L.nvfp4_scales_unswizzle.restype = i32
    L.nvfp4_quantize.argtypes = [vp, i64, i64, i64, ctypes.c_uint, u64, u64, op, op, vp, vp, vp]
    L.nvfp4_quantize.restype = i32
    L.nvfp4_rht_quantize.argtypes = [vp, i64, i64, i64, u16, ctypes.c_uint, u64, u64, op, vp,
                                     vp, vp]
    L.nvfp4_rht_quantize.restype = i32
    L.nvfp4_quantize_row_rht.argtypes = [vp, i64, i64, i64, u16, ctypes.c_uint, u64, u64, op,
                                         op, vp, vp, vp]
    L.nvfp4_quantize_row_rht.restype = i32
    L.nvfp4_gemm.argtypes = [op, op, vp, i32, i64, vp, vp]
    L.nvfp4_gemm.restype = i32
    L.nvfp4_gemm_mx.argtypes = [op, op, vp, i32, i64, vp, vp]
    L.nvfp4_gemm_mx.restype = i32
    L.nvfp4_gemm_amax.argtypes = [op, op, vp, i64, u16, vp, vp, vp]
    L.nvfp4_gemm_amax.restype = i32
    L.nvfp4_selftest_wait_timeout.argtypes = [vp, vp]
    L.nvfp4_selftest_wait_timeout.restype = i32
    L.nvfp4_bounds_checked.argtypes, L.nvfp4_bounds_checked.restype = [], i32
    L.nvfp4_selftest_bounds.argtypes, L.nvfp4_selftest_bounds.restype = [vp, vp], i32
    L.nvfp4_linear_fprop.argtypes = [vp, vp, i64, i64, i64, vp, i32, vp, vp, vp]
    L.nvfp4_linear_fprop.restype = i32
    L.nvfp4_linear_dgrad.argtypes = [vp, vp, i64, i64, i64, u64, u64, vp, i32, vp, vp, vp]
    L.nvfp4_linear_dgrad.restype = i32
    L.nvfp4_linear_wgrad.argtypes = [vp, vp, i64, i64, i64, u16, u64, u64, vp, i32, vp, vp, vp]
    L.nvfp4_linear_wgrad.restype = i32
    L.nvfp4_linear_dgrad_quantized.argtypes = [vp, vp, i64, i64, i64, u64, u64, vp, u16, u64,
                                               u64, op, op, vp, vp, vp]
    L.nvfp4_linear_dgrad_quantized.restype = i32
    return L


def declared_functions():
    """Names of the functions include/nvfp4.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def _check(status, what):
    if status != OK:
        raise NVFP4Error(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ---- sizes and host helpers -------------------------------------------------------------

def codes_bytes(rows, cols):
    return lib().nvfp4_codes_bytes(rows, cols)


def scales_bytes(rows, cols):
    return lib().nvfp4_scales_bytes(rows, cols)


def workspace_bytes(rows, cols, flags=0):
    return lib().nvfp4_workspace_bytes(rows, cols, flags)


def linear_workspace_bytes(T, I, O):
    return lib().nvfp4_linear_workspace_bytes(T, I, O)


def sign_mask_from_seed(seed):
    return lib().nvfp4_sign_mask_from_seed(seed)


def scales_unswizzle(swizzled, rows, cols):
    """Host (numpy uint8) MMA-layout scales -> row-major [rows x cols/16]."""
    import numpy as np
    src = np.ascontiguousarray(swizzled, dtype=np.uint8)
    out = np.zeros((rows, cols // 16), dtype=np.uint8)
    _check(lib().nvfp4_scales_unswizzle(src.ctypes.data_as(ctypes.c_void_p), rows, cols,
                                        out.ctypes.data_as(ctypes.c_void_p)), "scales_unswizzle")
    return out


# ---- device buffers ---------------------------------------------------------------------

class QuantizedTensor:
    """A quantized operand whose buffers torch allocated: codes [rows x cols/2] uint8,
    scales (MMA layout) uint8, amax float32[1]."""

    def __init__(self, rows, cols, device="cuda"):
        self.rows, self.cols = rows, cols
        self.codes = _poisoned(torch.empty((rows, cols // 2), dtype=torch.uint8, device=device))
        self.scales = _poisoned(torch.empty((scales_bytes(rows, cols),), dtype=torch.uint8,
                                            device=device))
        self.amax = _poisoned(torch.zeros((1,), dtype=torch.float32, device=device))

    def operand(self):
        return Operand(self.codes.data_ptr(), self.scales.data_ptr(), self.amax.data_ptr(),
                       self.rows, self.cols)


def _dtype_code(dtype):
    if dtype == torch.float32:
        return OUT_F32
    if dtype == torch.bfloat16:
        return OUT_BF16
    raise TypeError(f"unsupported output dtype {dtype}")


def _workspace(nbytes, device):
    if nbytes == 0:
        return None
    return _poisoned(torch.empty((nbytes,), dtype=torch.uint8, device=device))


def quantize(x, flags, seed=0, offset=0, out_row=None, out_col=None, workspace=None,
             dev_status=None, stream=None):
    """nvfp4_quantize on a 2D bf16 CUDA tensor (row stride x.stride(0))."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if flags & ROWWISE and out_row is None:
        out_row = QuantizedTensor(rows, cols, x.device)
    if flags & COLWISE and out_col is None:
        out_col = QuantizedTensor(cols, rows, x.device)
    if workspace is None:
        workspace = _workspace(workspace_bytes(rows, cols, flags), x.device)
    op_r = out_row.operand() if out_row is not None else None
    op_c = out_col.operand() if out_col is not None else None
    st = lib().nvfp4_quantize(_ptr(x), rows, cols, x.stride(0), flags, seed, offset,
                              ctypes.byref(op_r) if op_r is not None else None,
                              ctypes.byref(op_c) if op_c is not None else None,
                              _ptr(workspace), _ptr(dev_status), _stream(stream))
    _check(st, "nvfp4_quantize")
    return out_row, out_col


def rht_quantize(x, sign_mask, flags=0, seed=0, offset=0, out_col=None, workspace=None,
                 dev_status=None, stream=None):
    """nvfp4_rht_quantize: x^T random-Hadamard-transformed and quantized along x's rows."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if out_col is None:
        out_col = QuantizedTensor(cols, rows, x.device)
    if workspace is None:
        workspace = _workspace(workspace_bytes(rows, cols, flags), x.device)
    op_c = out_col.operand()
    st = lib().nvfp4_rht_quantize(_ptr(x), rows, cols, x.stride(0), sign_mask, flags, seed,
                                  offset, ctypes.byref(op_c), _ptr(workspace), _ptr(dev_status),
                                  _stream(stream))
    _check(st, "nvfp4_rht_quantize")
    return out_col


def quantize_row_rht(x, sign_mask, flags=0, seed=0, offset=0, out_row=None, out_col=None,
                     workspace=None, dev_status=None, stream=None):
    """nvfp4_quantize_row_rht: x row-wise (stream `offset`) and x^T RHT'd column-wise (stream
    `offset + 1`) from one amax pass and one quantize pass."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if out_row is None:
        out_row = QuantizedTensor(rows, cols, x.device)
    if out_col is None:
        out_col = QuantizedTensor(cols, rows, x.device)
    if workspace is None:
        workspace = _workspace(workspace_bytes(rows, cols, flags), x.device)
    op_r, op_c = out_row.operand(), out_col.operand()
    st = lib().nvfp4_quantize_row_rht(_ptr(x), rows, cols, x.stride(0), sign_mask, flags, seed,
                                      offset, ctypes.byref(op_r), ctypes.byref(op_c),
                                      _ptr(workspace), _ptr(dev_status), _stream(stream))
    _check(st, "nvfp4_quantize_row_rht")
    return out_row, out_col


def _check_out(out, rows, cols, what):
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"{what}: output must be float32 or bfloat16, got {out.dtype}")
    if tuple(out.shape) != (rows, cols) or out.stride(1) != 1 or not out.is_cuda:
        raise ValueError(f"{what}: output must be a CUDA [{rows} x {cols}] tensor with unit "
                         f"column stride, got {tuple(out.shape)} strides {out.stride()}")


def gemm(A, B, out=None, out_dtype=torch.float32, dev_status=None, stream=None, mx=False):
    """nvfp4_gemm (nvfp4_gemm_mx with `mx`): D = A . B^T (A, B QuantizedTensor).  The output
    type is out.dtype when `out` is given, else `out_dtype`."""
    name = "nvfp4_gemm_mx" if mx else "nvfp4_gemm"
    if out is None:
        out = _poisoned(torch.empty((A.rows, B.rows), dtype=out_dtype, device=A.codes.device))
    _check_out(out, A.rows, B.rows, name)
    d_dtype = _dtype_code(out.dtype)
    oa, ob = A.operand(), B.operand()
    st = getattr(lib(), name)(ctypes.byref(oa), ctypes.byref(ob), _ptr(out), d_dtype,
                              out.stride(0), _ptr(dev_status), _stream(stream))
    _check(st, name)
    return out


def gemm_amax(A, B, sign_mask, out=None, amax_out=None, dev_status=None, stream=None):
    """nvfp4_gemm_amax: bf16 D = A . B^T plus amax_out = [max |D|, max |RHT(D)|] (FP32)."""
    if out is None:
        out = _poisoned(torch.empty((A.rows, B.rows), dtype=torch.bfloat16,
                                    device=A.codes.device))
    _check_out(out, A.rows, B.rows, "nvfp4_gemm_amax")
    assert out.dtype == torch.bfloat16
    if amax_out is None:
        amax_out = _poisoned(torch.empty(2, dtype=torch.float32, device=A.codes.device))
    oa, ob = A.operand(), B.operand()
    st = lib().nvfp4_gemm_amax(ctypes.byref(oa), ctypes.byref(ob), _ptr(out), out.stride(0),
                               sign_mask, _ptr(amax_out), _ptr(dev_status), _stream(stream))
    _check(st, "nvfp4_gemm_amax")
    return out, amax_out


def selftest_wait_timeout(dev_status, stream=None):
    """nvfp4_selftest_wait_timeout: a bounded wait that nothing satisfies; after it the device
    status word has NVFP4_DEVSTAT_TIMEOUT set."""
    _check(lib().nvfp4_selftest_wait_timeout(_ptr(dev_status), _stream(stream)),
           "nvfp4_selftest_wait_timeout")


def is_bounds_checked():
    """nvfp4_bounds_checked of the library calls currently go to."""
    return bool(lib().nvfp4_bounds_checked())


def selftest_bounds(dev_status, stream=None):
    """nvfp4_selftest_bounds (checked build only): one refused store past a buffer's declared
    end; after it the device status word has NVFP4_DEVSTAT_BOUNDS set."""
    _check(lib().nvfp4_selftest_bounds(_ptr(dev_status), _stream(stream)),
           "nvfp4_selftest_bounds")


def linear_fprop(X, W, out=None, out_dtype=torch.float32, workspace=None, dev_status=None,
                 stream=None):
    T, I = X.shape
    O = W.shape[0]
    if out is None:
        out = _poisoned(torch.empty((T, O), dtype=out_dtype, device=X.device))
    _check_out(out, T, O, "nvfp4_linear_fprop")
    if workspace is None:
        workspace = _workspace(linear_workspace_bytes(T, I, O), X.device)
    st = lib().nvfp4_linear_fprop(_ptr(X), _ptr(W), T, I, O, _ptr(out), _dtype_code(out.dtype),
                                  _ptr(workspace), _ptr(dev_status), _stream(stream))
    _check(st, "nvfp4_linear_fprop")
    return out


def linear_dgrad(dY, W, seed, offset, out=None, out_dtype=torch.float32, workspace=None,
                 dev_status=None, stream=None):
    T, O = dY.shape
    I = W.shape[1]
    if out is None:
        out = _poisoned(torch.empty((T, I), dtype=out_dtype, device=dY.device))
    _check_out(out, T, I, "nvfp4_linear_dgrad")
    if workspace is None:
        workspace = _workspace(linear_workspace_bytes(T, I, O), dY.device)
    st = lib().nvfp4_linear_dgrad(_ptr(dY), _ptr(W), T, I, O, seed, offset, _ptr(out),
                                  _dtype_code(out.dtype), _ptr(workspace), _ptr(dev_status),
                                  _stream(stream))
    _check(st, "nvfp4_linear_dgrad")
    return out


def linear_dgrad_quantized(dY, W, seed, offset, sign_mask, next_seed, next_offset, out=None,
                           out_row=None, out_col=None, workspace=None, dev_status=None,
                           stream=None):
    """nvfp4_linear_dgrad_quantized: bf16 dX = dY . W plus dX's row-wise SR and RHT'd
    column-wise SR operands for the previous layer (returns dX, dX_row, dX_col)."""
    T, O = dY.shape
    I = W.shape[1]
    if out is None:
        out = _poisoned(torch.empty((T, I), dtype=torch.bfloat16, device=dY.device))
    _check_out(out, T, I, "nvfp4_linear_dgrad_quantized")
    if out.dtype != torch.bfloat16:
        raise TypeError("nvfp4_linear_dgrad_quantized: dX must be bfloat16")
    if out_row is None:
        out_row = QuantizedTensor(T, I, dY.device)
    if out_col is None:
        out_col = QuantizedTensor(I, T, dY.device)
    if workspace is None:
        workspace = _workspace(linear_workspace_bytes(T, I, O), dY.device)
    op_r, op_c = out_row.operand(), out_col.operand()
    st = lib().nvfp4_linear_dgrad_quantized(_ptr(dY), _ptr(W), T, I, O, seed, offset, _ptr(out),
                                            sign_mask, next_seed, next_offset,
                                            ctypes.byref(op_r), ctypes.byref(op_c),
                                            _ptr(workspace), _ptr(dev_status), _stream(stream))
    _check(st, "nvfp4_linear_dgrad_quantized")
    return out, out_row, out_col


def linear_wgrad(dY, X, sign_mask, seed, offset, out=None, out_dtype=torch.float32,
                 workspace=None, dev_status=None, stream=None):
    T, O = dY.shape
    I = X.shape[1]
    if out is None:
        out = _poisoned(torch.empty((O, I), dtype=out_dtype, device=dY.device))
    _check_out(out, O, I, "nvfp4_linear_wgrad")
    if workspace is None:
        workspace = _workspace(linear_workspace_bytes(T, I, O), dY.device)
    st = lib().nvfp4_linear_wgrad(_ptr(dY), _ptr(X), T, I, O, sign_mask, seed, offset, _ptr(out),
                                  _dtype_code(out.dtype), _ptr(workspace), _ptr(dev_status),
                                  _stream(stream))
    _check(st, "nvfp4_linear_wgrad")
    return out
