"""Failure detection without a GPU fault: the device-side waits of the GEMM are bounded, and a
wait that nothing satisfies ends with NVFP4_DEVSTAT_TIMEOUT in the status word instead of
hanging.  The self-test entry point runs the GEMM's own wait routine on an mbarrier that
nothing completes (50 ms limit); afterwards the context must still be usable."""
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import assert_gemm_close, need_gpu, to_device_bf16

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    need_gpu()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.selftest_wait_timeout(status)
    torch.cuda.synchronize()
    assert int(status.item()) & B.DEVSTAT_TIMEOUT
    assert not int(status.item()) & B.DEVSTAT_NONFINITE

    # the same context still computes correctly
    X = synth.activations((256, 512), seed=40)
    W = synth.weights((512, 512), seed=40)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = B.linear_fprop(to_device_bf16(X), to_device_bf16(W), dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    D_ref, norm = oracle.gemm_ref(*oracle.fprop_operands(X, W))
    assert_gemm_close(Y.cpu().numpy(), D_ref, norm, what="fprop after a timed-out wait")

