"""NVFP4 CPU oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.

Python access to the plain C oracle in ``nvfp4_oracle.c`` (loaded with ctypes), plus the
compositions the tests compare against: the quantized operands of the three training GEMMs
of one linear layer and their FP64 reference products.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  It shares no code with the CUDA library and imports nothing from it.

Sources are cited as in the C file: [P1] "Pretraining Large Language Models with NVFP4"
(gist.science), Resumen tecnico section 2 "Metodologia Propuesta"; [P3] news.hamidun.com,
"Como Funciona".
"""
import ctypes
import numpy as np

from . import build as _build

_lib = None

NVO_OK = 0
NVO_ERR_NONFINITE = 6


def lib():
    """Build (if stale) and load liboracle.so."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u8, u16, u32, u64, i64 = (ctypes.c_uint8, ctypes.c_uint16, ctypes.c_uint32,
                                  ctypes.c_uint64, ctypes.c_int64)
        vp, fp, dp = ctypes.c_void_p, ctypes.c_float, ctypes.c_double
        L.nvo_e2m1_decode.argtypes, L.nvo_e2m1_decode.restype = [u8], dp
        L.nvo_e2m1_rtn.argtypes, L.nvo_e2m1_rtn.restype = [fp], u8
        L.nvo_e2m1_sr.argtypes, L.nvo_e2m1_sr.restype = [fp, u32], u8
        L.nvo_e4m3_decode.argtypes, L.nvo_e4m3_decode.restype = [u8], dp
        L.nvo_e4m3_rne_satfinite.argtypes, L.nvo_e4m3_rne_satfinite.restype = [fp], u8
        L.nvo_philox4x32_10.argtypes, L.nvo_philox4x32_10.restype = [vp, vp, vp], None
        L.nvo_sr_bits.argtypes, L.nvo_sr_bits.restype = [u64, u64, u64], u32
        L.nvo_sign_mask_from_seed.argtypes, L.nvo_sign_mask_from_seed.restype = [u64], u16
        L.nvo_rht16.argtypes, L.nvo_rht16.restype = [vp, u16, vp], None
        L.nvo_tensor_scale.argtypes, L.nvo_tensor_scale.restype = [fp], fp
        L.nvo_block_scale.argtypes, L.nvo_block_scale.restype = [fp, fp], u8
        L.nvo_element_factor.argtypes, L.nvo_element_factor.restype = [fp, u8], fp
        L.nvo_quantize.argtypes = [vp, i64, i64, i64, ctypes.c_int, ctypes.c_int, u16,
                                   ctypes.c_int, ctypes.c_int, u64, u64, ctypes.c_int, fp,
                                   vp, vp, ctypes.POINTER(fp)]
        L.nvo_quantize.restype = ctypes.c_int
        L.nvo_quantize_rows.argtypes = [vp, i64, i64, i64, ctypes.c_int, ctypes.c_int, u16,
                                        ctypes.c_int, ctypes.c_int, u64, u64, fp, i64, i64,
                                        vp, vp]
        L.nvo_quantize_rows.restype = ctypes.c_int
        L.nvo_quantize_mt.argtypes = [vp, i64, i64, i64, ctypes.c_int, ctypes.c_int, u16,
                                      ctypes.c_int, ctypes.c_int, u64, u64, ctypes.c_int, fp,
                                      vp, vp, ctypes.POINTER(fp), ctypes.c_int]
        L.nvo_quantize_mt.restype = ctypes.c_int
        L.nvo_amax.argtypes = [vp, i64, i64, i64, ctypes.c_int, ctypes.c_int, u16,
                               ctypes.POINTER(fp)]
        L.nvo_amax.restype = ctypes.c_int
        L.nvo_dequantize.argtypes, L.nvo_dequantize.restype = [vp, vp, fp, i64, i64, vp], None
        L.nvo_gemm_ref.argtypes, L.nvo_gemm_ref.restype = [vp, vp, i64, i64, i64, vp], None
        L.nvo_row_norms.argtypes, L.nvo_row_norms.restype = [vp, i64, i64, vp], None
        L.nvo_e2m1_rtn_many.argtypes, L.nvo_e2m1_rtn_many.restype = [vp, i64, vp], None
        L.nvo_e2m1_sr_many.argtypes, L.nvo_e2m1_sr_many.restype = [vp, vp, i64, vp], None
        L.nvo_e4m3_many.argtypes, L.nvo_e4m3_many.restype = [vp, i64, vp], None
        L.nvo_mx_exponent.argtypes, L.nvo_mx_exponent.restype = [fp], ctypes.c_int
        L.nvo_e8m0_decode.argtypes, L.nvo_e8m0_decode.restype = [u8], dp
        L.nvo_mx_quantize.argtypes = [vp, i64, i64, i64, ctypes.c_int, ctypes.c_int, u16,
                                      ctypes.c_int, u64, u64, vp, vp]
        L.nvo_mx_quantize.restype = ctypes.c_int
        L.nvo_mx_dequantize.argtypes, L.nvo_mx_dequantize.restype = [vp, vp, i64, i64, vp], None
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---- scalar codecs ---------------------------------------------------------------------

def e2m1_decode(code: int) -> float:
    return lib().nvo_e2m1_decode(code)


def e2m1_rtn(v: float) -> int:
    return lib().nvo_e2m1_rtn(v)


def e2m1_sr(v: float, r16: int) -> int:
    return lib().nvo_e2m1_sr(v, r16)


def e2m1_rtn_many(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.shape, dtype=np.uint8)
    lib().nvo_e2m1_rtn_many(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_sr_many(v: np.ndarray, r16: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    r = np.ascontiguousarray(r16, dtype=np.uint32)
    assert r.shape == v.shape
    out = np.zeros(v.shape, dtype=np.uint8)
    lib().nvo_e2m1_sr_many(_ptr(v), _ptr(r), v.size, _ptr(out))
    return out


def e4m3_encode_many(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, dtype=np.uint8)
    lib().nvo_e4m3_many(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(b: int) -> float:
    return lib().nvo_e4m3_decode(b)


def e4m3_encode(x: float) -> int:
    return lib().nvo_e4m3_rne_satfinite(x)


def philox4x32_10(ctr, key):
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().nvo_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return [int(v) for v in out]


def sr_bits(seed: int, offset: int, e: int) -> int:
    return lib().nvo_sr_bits(seed, offset, e)


def sign_mask_from_seed(seed: int) -> int:
    return lib().nvo_sign_mask_from_seed(seed)


def rht16(x, sign_mask: int) -> np.ndarray:
    xa = np.ascontiguousarray(x, dtype=np.float32)
    assert xa.shape == (16,)
    y = np.zeros(16, dtype=np.float32)
    lib().nvo_rht16(_ptr(xa), sign_mask, _ptr(y))
    return y


def tensor_scale(amax: float) -> float:
    return lib().nvo_tensor_scale(amax)


def block_scale(b: float, s_enc: float) -> int:
    return lib().nvo_block_scale(b, s_enc)


# ---- tensor quantization ---------------------------------------------------------------

class Quantized:
    """A quantized operand in the oracle's plain layout: codes [R x C/2] (even column in
    the low nibble), scales [R x C/16] E4M3 bytes row-major, FP32 tensor amax."""

    def __init__(self, codes, scales, amax, status):
        self.codes, self.scales, self.amax, self.status = codes, scales, amax, status

    @property
    def rows(self):
        return self.codes.shape[0]

    @property
    def cols(self):
        return self.codes.shape[1] * 2

    def dequantize(self) -> np.ndarray:
        R, C = self.rows, self.cols
        out = np.zeros((R, C), dtype=np.float64)
        lib().nvo_dequantize(_ptr(self.codes), _ptr(self.scales), self.amax, R, C, _ptr(out))
        return out


def quantize(x_bf16: np.ndarray, *, transpose=False, rht=False, sign_mask=0, block2d=False,
             sr=False, seed=0, offset=0, amax=None, threads=1) -> Quantized:
    """Quantize the bf16 matrix ``x_bf16`` (np.uint16 bit patterns, rows x cols) along its
    rows (or, with ``transpose``, along its columns, i.e. quantize x^T).  ``threads`` > 1
    runs the oracle's threaded driver (the same two passes over ranges of rows, same bits)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    R, C = (cols, rows) if transpose else (rows, cols)
    codes = np.zeros((R, C // 2), dtype=np.uint8)
    scales = np.zeros((R, C // 16), dtype=np.uint8)
    amax_out = ctypes.c_float(0.0)
    args = (_ptr(x), rows, cols, cols, int(transpose), int(rht), sign_mask, int(block2d),
            int(sr), seed, offset, int(amax is not None), 0.0 if amax is None else float(amax),
            _ptr(codes), _ptr(scales), ctypes.byref(amax_out))
    if threads > 1:
        st = lib().nvo_quantize_mt(*args, int(threads))
    else:
        st = lib().nvo_quantize(*args)
    if st not in (NVO_OK, NVO_ERR_NONFINITE):
        raise ValueError(f"oracle quantize rejected the arguments (status {st})")
    return Quantized(codes, scales, amax_out.value, st)


def quantize_rows(x_bf16: np.ndarray, r_begin: int, r_end: int, amax: float, *,
                  transpose=False, rht=False, sign_mask=0, block2d=False, sr=False, seed=0,
                  offset=0, out: Quantized = None) -> Quantized:
    """Quantize only logical rows [r_begin, r_end) of the matrix ``quantize`` would quantize,
    with the given (whole-tensor) amax, into ``out`` (a full-size Quantized, created if None);
    the other rows are left as they are.  r_begin is a multiple of 16."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    R, C = (cols, rows) if transpose else (rows, cols)
    if out is None:
        out = Quantized(np.zeros((R, C // 2), dtype=np.uint8),
                        np.zeros((R, C // 16), dtype=np.uint8), float(amax), NVO_OK)
    st = lib().nvo_quantize_rows(_ptr(x), rows, cols, cols, int(transpose), int(rht), sign_mask,
                                 int(block2d), int(sr), seed, offset, float(amax), r_begin,
                                 r_end, _ptr(out.codes), _ptr(out.scales))
    if st != NVO_OK:
        raise ValueError(f"oracle quantize_rows rejected the arguments (status {st})")
    return out


def amax(x_bf16: np.ndarray, *, transpose=False, rht=False, sign_mask=0):
    """The tensor amax ``quantize`` would compute for the same arguments (its first pass), on
    its own and without materialising x^T: returns (amax, status)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    out = ctypes.c_float(0.0)
    st = lib().nvo_amax(_ptr(x), rows, cols, cols, int(transpose), int(rht), sign_mask,
                        ctypes.byref(out))
    if st not in (NVO_OK, NVO_ERR_NONFINITE):
        raise ValueError(f"oracle amax rejected the arguments (status {st})")
    return out.value, st


# ---- MXFP4, the comparison format ------------------------------------------------------

class MXQuantized:
    """An MXFP4 operand in the oracle's plain layout: codes [R x C/2] as NVFP4, scales
    [R x C/32] E8M0 bytes row-major (scale = 2^(byte - 127)); no tensor scale."""

    def __init__(self, codes, scales, status):
        self.codes, self.scales, self.status = codes, scales, status

    @property
    def rows(self):
        return self.codes.shape[0]

    @property
    def cols(self):
        return self.codes.shape[1] * 2

    def dequantize(self) -> np.ndarray:
        R, C = self.rows, self.cols
        out = np.zeros((R, C), dtype=np.float64)
        lib().nvo_mx_dequantize(_ptr(self.codes), _ptr(self.scales), R, C, _ptr(out))
        return out


def mx_exponent(b: float) -> int:
    return lib().nvo_mx_exponent(b)


def e8m0_decode(code: int) -> float:
    return lib().nvo_e8m0_decode(code)


def mx_quantize(x_bf16: np.ndarray, *, transpose=False, rht=False, sign_mask=0, sr=False,
                seed=0, offset=0) -> MXQuantized:
    """MXFP4-quantize the bf16 matrix ``x_bf16`` along its rows (or, with ``transpose``,
    quantize x^T), in blocks of 32 with E8M0 power-of-two scales."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    R, C = (cols, rows) if transpose else (rows, cols)
    codes = np.zeros((R, C // 2), dtype=np.uint8)
    scales = np.zeros((R, C // 32), dtype=np.uint8)
    st = lib().nvo_mx_quantize(_ptr(x), rows, cols, cols, int(transpose), int(rht), sign_mask,
                               int(sr), seed, offset, _ptr(codes), _ptr(scales))
    if st not in (NVO_OK, NVO_ERR_NONFINITE):
        raise ValueError(f"oracle MX quantize rejected the arguments (status {st})")
    return MXQuantized(codes, scales, st)


def gemm_ref_loop(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """D = A . B^T by the plain FP64 triple loop (tiny shapes only)."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = A.shape
    N = B.shape[0]
    D = np.zeros((M, N), dtype=np.float64)
    lib().nvo_gemm_ref(_ptr(A), _ptr(B), M, N, K, _ptr(D))
    return D


def row_norms(A: np.ndarray) -> np.ndarray:
    A = np.ascontiguousarray(A, dtype=np.float64)
    out = np.zeros(A.shape[0], dtype=np.float64)
    lib().nvo_row_norms(_ptr(A), A.shape[0], A.shape[1], _ptr(out))
    return out


def gemm_ref(qa, qb, rows=None, cols=None):
    """Reference D = deq(A) . deq(B)^T in FP64 (numpy matmul as the dot-product step) and
    the normaliser ||A[m,:]|| * ||B[n,:]|| for each entry, optionally restricted to the
    sampled output rows and columns."""
    A = qa.dequantize()
    B = qb.dequantize()
    if rows is not None:
        A = A[rows]
    if cols is not None:
        B = B[cols]
    D = A @ B.T
    norm = np.outer(np.sqrt((A * A).sum(axis=1)), np.sqrt((B * B).sum(axis=1)))
    return D, norm


# ---- the three GEMMs of one linear layer -----------------------------------------------
# [P1 Escalado 2D y Redondeo Estocastico]: weights are scaled in 16x16 blocks so fprop
# and dgrad see the same quantized W; gradients (dY) use stochastic rounding; [P1 RHT] the
# two wgrad inputs pass the 16x16 random Hadamard transform along the token axis.
# READING: dgrad's row-wise dY draws from stream `offset`, wgrad's column-wise dY from
# `offset + 1`, so the two quantizations of one dY are independent; X is RHT'd and rounded
# to nearest for wgrad.

def fprop_operands(X, W):
    """Y = X . W^T: A = X quantized along I (1x16, RTN), B = W along I (16x16, RTN)."""
    return quantize(X), quantize(W, block2d=True)


def dgrad_operands(dY, W, seed, offset):
    """dX = dY . W: A = dY along O (1x16, SR), B = W^T along O (16x16, RTN)."""
    return (quantize(dY, sr=True, seed=seed, offset=offset),
            quantize(W, transpose=True, block2d=True))


def wgrad_operands(dY, X, sign_mask, seed, offset):
    """dW = dY^T . X: A = dY^T along T (RHT, SR), B = X^T along T (RHT, RTN)."""
    return (quantize(dY, transpose=True, rht=True, sign_mask=sign_mask, sr=True, seed=seed,
                     offset=offset + 1),
            quantize(X, transpose=True, rht=True, sign_mask=sign_mask))
