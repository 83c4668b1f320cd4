"""nvfp4_quantize_noalloc: the quantizer entry point for callers that cannot allocate device
memory where they quantize (a framework that owns all device memory through a fixed arena, or
a latency-critical loop that must stay out of cudaMalloc / cudaFree).  It keeps the amax
pass's scratch in a static device array instead of a caller workspace.

Called through the C ABI and compared with nvfp4_quantize on the same inputs, bit for bit (the
tolerance every quantizer test uses), on two calls in a row: a large tensor, then a smaller
one whose amax pass uses fewer scratch slots than the first left behind.  This file is
collected last so that a failure here stops a `-x` run only after every other test ran."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from nvfp4_testlib import need_gpu, to_device_bf16

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = pytest.mark.gpu


def _noalloc():
    f = B.lib().nvfp4_quantize_noalloc
    op = ctypes.POINTER(B.Operand)
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint,
                  ctypes.c_uint64, ctypes.c_uint64, op, op, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _call_noalloc(x, flags, seed, offset, out_row, out_col, status):
    o_r = out_row.operand() if out_row is not None else None
    o_c = out_col.operand() if out_col is not None else None
    return _noalloc()(ctypes.c_void_p(x.data_ptr()), x.shape[0], x.shape[1], x.stride(0), flags,
                      seed, offset, ctypes.byref(o_r) if o_r is not None else None,
                      ctypes.byref(o_c) if o_c is not None else None,
                      ctypes.c_void_p(status.data_ptr()),
                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same(a, b):
    return (torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
            and torch.equal(a.amax, b.amax))


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    need_gpu()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cases = [((4096, 8192), B.ROWWISE | B.COLWISE | B.SR, synth.gradients, 7),
             ((256, 512), B.ROWWISE, synth.activations, 0)]
    for shape, flags, gen, seed in cases:
        x = to_device_bf16(gen(shape, seed=seed))
        rows, cols = shape
        got_r = B.QuantizedTensor(rows, cols) if flags & B.ROWWISE else None
        got_c = B.QuantizedTensor(cols, rows) if flags & B.COLWISE else None
        st = _call_noalloc(x, flags, seed, 3, got_r, got_c, status)
        assert st == B.OK, B.lib().nvfp4_status_string(st)
        want_r, want_c = B.quantize(x, flags, seed=seed, offset=3)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        if got_r is not None:
            assert _same(got_r, want_r), f"row-wise output differs for {shape}"
        if got_c is not None:
            assert _same(got_c, want_c), f"column-wise output differs for {shape}"


def test_noalloc_two_calls_queued_on_one_stream_without_a_sync():
    """Calls queued back to back on one stream are ordered: the second call's amax pass
    overwrites the scratch slots only after the first call's quantize pass has read them."""
    need_gpu()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cases = [((8192, 4096), B.ROWWISE | B.SR, synth.gradients, 21),
             ((2048, 1024), B.ROWWISE | B.COLWISE, synth.activations, 22)]
    got = []
    for shape, flags, gen, seed in cases:
        x = to_device_bf16(gen(shape, seed=seed))
        rows, cols = shape
        r = B.QuantizedTensor(rows, cols) if flags & B.ROWWISE else None
        c = B.QuantizedTensor(cols, rows) if flags & B.COLWISE else None
        st = _call_noalloc(x, flags, seed, 1, r, c, status)
        assert st == B.OK, B.lib().nvfp4_status_string(st)
        got.append((x, flags, seed, r, c))
    for x, flags, seed, r, c in got:
        want_r, want_c = B.quantize(x, flags, seed=seed, offset=1)
        if r is not None:
            assert _same(r, want_r)
        if c is not None:
            assert _same(c, want_c)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_noalloc_amax_given_and_mx():
    """NVFP4_AMAX_GIVEN (no amax pass, the scratch is not touched) and the MXFP4 flag through
    this entry point, against nvfp4_quantize with the same flags."""
    need_gpu()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = to_device_bf16(synth.activations((1024, 2048), seed=23))
    want_r, _ = B.quantize(x, B.ROWWISE)
    got_r = B.QuantizedTensor(1024, 2048)
    got_r.amax.copy_(want_r.amax)
    st = _call_noalloc(x, B.ROWWISE | B.AMAX_GIVEN, 0, 0, got_r, None, status)
    assert st == B.OK
    assert _same(got_r, want_r)
    flags = B.ROWWISE | B.COLWISE | B.MX
    got_r, got_c = B.QuantizedTensor(1024, 2048), B.QuantizedTensor(2048, 1024)
    assert _call_noalloc(x, flags, 0, 0, got_r, got_c, status) == B.OK
    want_r, want_c = B.quantize(x, flags)
    assert _same(got_r, want_r) and _same(got_c, want_c)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_noalloc_rejects_bad_arguments_like_the_workspace_entry_point():
    need_gpu()
    out = B.QuantizedTensor(256, 512)
    x = to_device_bf16(synth.activations((256, 512), seed=1))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _call_noalloc(x, B.ROWWISE | B.BLOCK2D | B.SR, 0, 0, out, None, status) == B.ERR_ARG
    bad = B.QuantizedTensor(128, 512)
    assert _call_noalloc(x, B.ROWWISE, 0, 0, bad, None, status) == B.ERR_SHAPE
    assert np.all(status.cpu().numpy() == 0)
