"""Whole-tensor parity at the 12B-class MLP shapes (tokens 8192, 5120 <-> 20480) and the
8B-class dense layer (tokens 16384, d 4096: QKV 4096 -> 6144, O 4096 -> 4096, gate and up
4096 -> 14336, down 14336 -> 4096).

For every linear:
* every quantized operand the benchmark step produces -- W row-wise and column-wise with 16 x 16
  scales, X row-wise and RHT'd column-wise, dY row-wise with stochastic rounding (stream 0) and
  RHT'd column-wise with stochastic rounding (stream 1) -- is compared with the oracle's whole
  tensor, every code and every scale, bit for bit (the oracle runs its threaded driver over
  ranges of rows, which gives the single-threaded call's bits);
* fprop, dgrad and wgrad through the C ABI's linear entry points are compared with the oracle's
  FP64 products on 256 sampled output rows x all columns and all rows x 256 sampled columns,
  within 1e-3 of ||A[m,:]|| ||B[n,:]||."""
import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import (assert_gemm_close, assert_quantized_equal, gemm_ref_sampled,
                           host_threads, need_gpu, to_device_bf16)

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLES = 256


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def _sample(n, seed):
    rng = np.random.default_rng(seed + n)
    return np.sort(rng.choice(n, size=min(SAMPLES, n), replace=False))


def _check_linear(wl, which):
    names = [l.name for l in wl.linears]
    idx = names.index(which)
    lin = wl.linears[idx]
    X, W, dY = synth.linear_inputs(lin, wl.seed, layer_index=idx)
    mask = oracle.sign_mask_from_seed(wl.seed)
    seed = wl.seed
    th = host_threads()
    Xd, Wd, dYd = to_device_bf16(X), to_device_bf16(W), to_device_bf16(dY)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    # the benchmark step's operand quantizations, one call per tensor
    w_row, w_col = B.quantize(Wd, B.ROWWISE | B.COLWISE | B.BLOCK2D, dev_status=status)
    x_row, x_col = B.quantize_row_rht(Xd, mask, 0, dev_status=status)
    dy_row, dy_col = B.quantize_row_rht(dYd, mask, B.SR, seed=seed, offset=0, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    ref = {
        "W row": oracle.quantize(W, block2d=True, threads=th),
        "W col": oracle.quantize(W, transpose=True, block2d=True, threads=th),
        "X row": oracle.quantize(X, threads=th),
        "X col": oracle.quantize(X, transpose=True, rht=True, sign_mask=mask, threads=th),
        "dY row": oracle.quantize(dY, sr=True, seed=seed, offset=0, threads=th),
        "dY col": oracle.quantize(dY, transpose=True, rht=True, sign_mask=mask, sr=True,
                                  seed=seed, offset=1, threads=th),
    }
    got = {"W row": w_row, "W col": w_col, "X row": x_row, "X col": x_col, "dY row": dy_row,
           "dY col": dy_col}
    for name, q in got.items():
        assert_quantized_equal(q, ref[name], f"{wl.name} {which} {name}")
    del got, w_row, w_col, x_row, x_col, dy_row, dy_col

    # the three GEMMs through the linear entry points, sampled against the oracle
    outs = {"fprop": (B.linear_fprop(Xd, Wd, dev_status=status), ref["X row"], ref["W row"]),
            "dgrad": (B.linear_dgrad(dYd, Wd, seed, 0, dev_status=status), ref["dY row"],
                      ref["W col"]),
            "wgrad": (B.linear_wgrad(dYd, Xd, mask, seed, 0, dev_status=status), ref["dY col"],
                      ref["X col"])}
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for k, (name, (D, qa, qb)) in enumerate(outs.items()):
        r, c = _sample(qa.rows, 2 * k), _sample(qb.rows, 2 * k + 1)
        Dr, nr = gemm_ref_sampled(qa, qb, rows=r)
        assert_gemm_close(D[torch.from_numpy(r).cuda()].cpu().numpy(), Dr, nr,
                          what=f"{which} {name} rows")
        Dc, nc = gemm_ref_sampled(qa, qb, cols=c)
        assert_gemm_close(D[:, torch.from_numpy(c).cuda()].cpu().numpy(), Dc, nc,
                          what=f"{which} {name} cols")


@pytest.mark.parametrize("which", ["up", "down"])
def test_mlp_12b_linear(which):
    _check_linear(synth.mlp_12b(), which)


@pytest.mark.parametrize("which", ["qkv", "o", "gate", "up", "down"])
def test_dense_8b_linear(which):
    _check_linear(synth.dense_8b_layer(), which)
