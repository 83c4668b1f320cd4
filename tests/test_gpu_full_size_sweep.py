"""Full-size parity of the quantizer sweep's largest tensor (2^30 bf16 elements in rows of
4096, the sweep's generator and seed) in the output modes the row-wise full-size test does not
cover: column-wise 1x16 (RTN and SR), 16x16 2D (both orientations) and the RHT'd column-wise
output (RTN and SR).

The oracle cannot quantize a tensor this size whole, so:
* the whole-tensor amax (plain, or over the RHT'd blocks down the columns) comes from the
  oracle's stand-alone amax pass, and the GPU's must equal it bit for bit;
* codes and scales of sampled blocks are compared with the oracle run on the sub-matrix that
  holds them, given that amax: a block depends only on its own 16 (or 16x16) values and the
  tensor scale;
* with stochastic rounding the column-wise output's element index is (output row) x rows +
  (input row). So the sample is the first 16 output rows over their whole length: the
  sub-matrix x[:, :16] has all the rows, hence the same indices."""
import numpy as np
import pytest
import torch

import oracle
import synth
from nvfp4_testlib import need_gpu, sf_offsets, to_device_bf16

nv = pytest.importorskip("nvfp4_bit_quantized_03_b200")
B = nv.binding

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SEED, OFFSET = 21, 4


@pytest.fixture(scope="module")
def sweep_tensor():
    need_gpu()
    rows, cols = synth.quant_sweep_shape(30)
    x = synth.activations((rows, cols), seed=synth.QUANT_SWEEP_SEED)
    mask = oracle.sign_mask_from_seed(synth.QUANT_SWEEP_SEED)
    amax, st = oracle.amax(x)
    assert st == oracle.NVO_OK
    amax_rht, st = oracle.amax(x, transpose=True, rht=True, sign_mask=mask)
    assert st == oracle.NVO_OK
    yield {"x": x, "xd": to_device_bf16(x), "mask": mask, "amax": amax, "amax_rht": amax_rht}
    torch.cuda.empty_cache()


def _same_amax(qt, want):
    got = np.float32(qt.amax.item()).view(np.uint32)
    assert got == np.float32(want).view(np.uint32), (qt.amax.item(), want)


def _check_block(qt, ref, rows_idx, c0, what):
    """qt's output rows `rows_idx`, columns [c0, c0 + ref width) against the oracle result
    `ref` for exactly those rows and columns."""
    n = ref.codes.shape[1] * 2
    ri = torch.from_numpy(np.asarray(rows_idx, np.int64)).cuda()
    codes = qt.codes[ri, c0 // 2:(c0 + n) // 2].cpu().numpy()
    bad = np.argwhere(codes != ref.codes)
    assert bad.size == 0, (what, "codes differ at", bad[:5])
    offs = sf_offsets(qt.rows, qt.cols, r=rows_idx, j=np.arange(c0 // 16, (c0 + n) // 16))
    scales = qt.scales[torch.from_numpy(offs).cuda()].cpu().numpy()
    bad = np.argwhere(scales != ref.scales)
    assert bad.size == 0, (what, "scales differ at", bad[:5])


def _col_sample(rows, cols, rng, n_rows=1024, n_cols=32):
    """Sampled output rows (input columns) and a 16-aligned band of input rows."""
    orows = np.sort(rng.choice(cols, n_cols, replace=False))
    r0 = 16 * int(rng.integers(0, (rows - n_rows) // 16 + 1))
    return orows, r0, n_rows


def test_colwise_rtn_full_size(sweep_tensor):
    x, t = sweep_tensor["x"], sweep_tensor
    rows, cols = x.shape
    _, qc = B.quantize(t["xd"], B.COLWISE)
    _same_amax(qc, t["amax"])
    orows, r0, n = _col_sample(rows, cols, np.random.default_rng(1))
    ref = oracle.quantize(x[r0:r0 + n][:, orows], transpose=True, amax=t["amax"])
    _check_block(qc, ref, orows, r0, "colwise rtn")


def test_colwise_sr_full_size(sweep_tensor):
    x, t = sweep_tensor["x"], sweep_tensor
    _, qc = B.quantize(t["xd"], B.COLWISE | B.SR, seed=SEED, offset=OFFSET)
    _same_amax(qc, t["amax"])
    ref = oracle.quantize(x[:, :16], transpose=True, sr=True, seed=SEED, offset=OFFSET,
                          amax=t["amax"])
    _check_block(qc, ref, np.arange(16), 0, "colwise sr")


def test_block2d_full_size(sweep_tensor):
    x, t = sweep_tensor["x"], sweep_tensor
    rows, cols = x.shape
    qr, qc = B.quantize(t["xd"], B.ROWWISE | B.COLWISE | B.BLOCK2D)
    _same_amax(qr, t["amax"])
    _same_amax(qc, t["amax"])
    rng = np.random.default_rng(2)
    for _ in range(2):
        r0 = 16 * int(rng.integers(0, rows // 16 - 4))
        ref = oracle.quantize(x[r0:r0 + 64], block2d=True, amax=t["amax"])
        _check_block(qr, ref, np.arange(r0, r0 + 64), 0, "2d row")
        c0 = 16 * int(rng.integers(0, cols // 16 - 2))
        b0 = 16 * int(rng.integers(0, (rows - 1024) // 16 + 1))
        ref = oracle.quantize(x[b0:b0 + 1024, c0:c0 + 32], transpose=True, block2d=True,
                              amax=t["amax"])
        _check_block(qc, ref, np.arange(c0, c0 + 32), b0, "2d col")


def test_rht_colwise_rtn_full_size(sweep_tensor):
    x, t = sweep_tensor["x"], sweep_tensor
    rows, cols = x.shape
    qc = B.rht_quantize(t["xd"], t["mask"])
    _same_amax(qc, t["amax_rht"])
    orows, r0, n = _col_sample(rows, cols, np.random.default_rng(3))
    ref = oracle.quantize(x[r0:r0 + n][:, orows], transpose=True, rht=True,
                          sign_mask=t["mask"], amax=t["amax_rht"])
    _check_block(qc, ref, orows, r0, "rht colwise rtn")


def test_rht_colwise_sr_full_size(sweep_tensor):
    x, t = sweep_tensor["x"], sweep_tensor
    qc = B.rht_quantize(t["xd"], t["mask"], B.SR, seed=SEED, offset=OFFSET)
    _same_amax(qc, t["amax_rht"])
    ref = oracle.quantize(x[:, :16], transpose=True, rht=True, sign_mask=t["mask"], sr=True,
                          seed=SEED, offset=OFFSET, amax=t["amax_rht"])
    _check_block(qc, ref, np.arange(16), 0, "rht colwise sr")
