"""GPU parity of the three training GEMMs of a linear layer (fprop, dgrad, wgrad) through the
C ABI, against the oracle's composition of the recipe: whole outputs at the small workloads,
sampled rows and columns at the 12B-class MLP shapes the benchmark runs."""
import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import assert_gemm_close, need_gpu, to_device_bf16

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def _run_layer(lin, seed, rows=None, cols=None, dtype=torch.float32):
    X, W, dY = synth.linear_inputs(lin, seed)
    mask = oracle.sign_mask_from_seed(seed)
    Xd, Wd, dYd = to_device_bf16(X), to_device_bf16(W), to_device_bf16(dY)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = B.linear_fprop(Xd, Wd, out_dtype=dtype, dev_status=status)
    dX = B.linear_dgrad(dYd, Wd, seed, 0, out_dtype=dtype, dev_status=status)
    dW = B.linear_wgrad(dYd, Xd, mask, seed, 0, out_dtype=dtype, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    bf16 = dtype == torch.bfloat16
    checks = [("fprop", Y, oracle.fprop_operands(X, W)),
              ("dgrad", dX, oracle.dgrad_operands(dY, W, seed, 0)),
              ("wgrad", dW, oracle.wgrad_operands(dY, X, mask, seed, 0))]
    for name, D, (qa, qb) in checks:
        r = None if rows is None else rows(qa.rows)
        c = None if cols is None else cols(qb.rows)
        D_ref, norm = oracle.gemm_ref(qa, qb, rows=r, cols=c)
        Dh = D.float()
        if r is not None:
            Dh = Dh[torch.from_numpy(r).cuda()]
        if c is not None:
            Dh = Dh[:, torch.from_numpy(c).cuda()]
        assert_gemm_close(Dh.cpu().numpy(), D_ref, norm, bf16=bf16, what=f"{lin.name} {name}")


@pytest.mark.parametrize("T,I,O", [(256, 512, 512), (192, 320, 448), (512, 1024, 256)])
def test_linear_small(T, I, O):
    _run_layer(synth.Linear("t", T, I, O), seed=T + I + O)


def test_linear_bf16_outputs():
    _run_layer(synth.Linear("t", 256, 512, 384), seed=5, dtype=torch.bfloat16)


def test_fprop_small_workload():
    """Single fprop linear, X [256 x 512], W [512 x 512], FP32 out, seed 0."""
    wl = synth.fprop_small()
    lin = wl.linears[0]
    X, W, _ = synth.linear_inputs(lin, wl.seed)
    Y = B.linear_fprop(to_device_bf16(X), to_device_bf16(W))
    D_ref, norm = oracle.gemm_ref(*oracle.fprop_operands(X, W))
    assert_gemm_close(Y.cpu().numpy(), D_ref, norm, what="fprop small")


def test_one_layer_4096_full():
    wl = synth.layer_4096()
    _run_layer(wl.linears[0], wl.seed)
