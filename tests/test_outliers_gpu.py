"""GPU parity of the sparse outlier separation against the oracle, and the
separated pipeline (separate -> quantize the bulk -> dequantize -> scatter).

The row mean and deviation are fp64 reductions in a different order on each
side, so an element whose deviation lies within a relative 1e-12 of the row's
threshold could be classified differently; every other element must agree,
and on these inputs no element comes that close (the tests assert equality).
"""
from __future__ import annotations

import ml_dtypes
import numpy as np
import pytest
import torch

from activation_quantization_block_b200 import fp4q, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _inputs(rows, cols, seed):
    w = synthetic.llm_weight(rows, cols, seed=seed).float().numpy()
    rng = np.random.default_rng(seed)
    for r in range(max(3, rows - 8), rows):                        # 5 % spikes of +-0.5: the 2 % cap binds,
        pos = rng.choice(cols, max(1, cols // 20), replace=False)  # and equal deviations tie
        w[r, pos] = np.where(np.arange(len(pos)) % 2 == 0, 0.5, -0.5)
    w[0] = 0.0                                                     # a zero row
    w[1] = 0.03125                                                 # a constant row
    w[2, ::7] = 0.5                                                # many equal spikes: ties at the cap
    return torch.from_numpy(w.astype(ml_dtypes.bfloat16).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("shape", [(64, 1024), (40, 4096), (3, 14336), (17, 8)])
def test_separation_matches_oracle(orc, dev, shape):
    rows, cols = shape
    x = _inputs(rows, cols, seed=rows + cols)
    o = fp4q.separate_outliers(x.to(dev))
    torch.cuda.synchronize()
    bulk, oc, ov, cnt, mu, thr = orc.separate_outliers(synthetic.bf16_bits(x))
    cap = orc.outlier_capacity(cols)
    assert fp4q.fp4q_outlier_capacity(cols, 0.02) == cap
    assert np.array_equal(o.count.cpu().numpy(), cnt)
    if cap:
        gc = o.cols.cpu().numpy().view(np.uint16)[:, :cap]
        gv = o.vals.cpu().numpy().view(np.uint16)[:, :cap]
        for r in range(rows):
            assert np.array_equal(gc[r, :cnt[r]], oc[r, :cnt[r]]) and np.array_equal(gv[r, :cnt[r]], ov[r, :cnt[r]])
    assert np.array_equal(synthetic.bf16_bits(o.bulk), bulk)
    assert cnt[0] == 0 and cnt[1] == 0
    if rows > 8 and cap:
        assert (cnt[-8:] == cap).all()


def test_scatter_puts_values_back(dev):
    rows, cols = 33, 2048
    cap = fp4q.fp4q_outlier_capacity(cols, 0.02)
    rng = np.random.default_rng(3)
    cnt = rng.integers(0, cap + 1, rows).astype(np.int32)
    oc = np.zeros((rows, cap), np.uint16)
    ov = rng.standard_normal((rows, cap)).astype(np.float16)
    want = np.zeros((rows, cols), np.float32)
    for r in range(rows):
        oc[r, :cnt[r]] = np.sort(rng.choice(cols, cnt[r], replace=False))
        want[r, oc[r, :cnt[r]]] = ov[r, :cnt[r]].astype(np.float32)
    o = fp4q.Outliers(None, torch.from_numpy(oc.view(np.int16)).to(dev), torch.from_numpy(ov).to(dev),
                      torch.from_numpy(cnt).to(dev))
    y = torch.zeros(rows, cols, dtype=torch.bfloat16, device=dev)
    fp4q.scatter_outliers(o, y)
    torch.cuda.synchronize()
    assert np.array_equal(synthetic.bf16_bits(y), want.astype(ml_dtypes.bfloat16).view(np.uint16))


def test_scatter_skips_columns_at_or_past_cols(dev):
    """Hand-made slots whose columns lie in [cols, ldy) or beyond: nothing may land
    in the padding columns of a strided y, nor past the last row's cols elements."""
    rows, cols, ldy, guard = 5, 256, 264, 64
    cap = fp4q.fp4q_outlier_capacity(cols, 0.02)            # 5
    oc = np.zeros((rows, cap), np.uint16)
    ov = np.full((rows, cap), 7.0, np.float16)
    cnt = np.full(rows, cap, np.int32)
    for r in range(rows):
        oc[r] = [r, cols, cols + 3, ldy - 1, ldy + 40][:cap]   # one valid column, the rest out of range
    o = fp4q.Outliers(None, torch.from_numpy(oc.view(np.int16)).to(dev), torch.from_numpy(ov).to(dev),
                      torch.from_numpy(cnt).to(dev))
    # y ends right after (rows-1)*ldy + cols elements; a guard region follows
    n = (rows - 1) * ldy + cols
    buf = torch.full((n + guard,), -3.0, dtype=torch.bfloat16, device=dev)
    st = fp4q.fp4q_scatter_outliers(o.cols, o.vals, o.count, rows, cols, cap, buf, ldy)
    assert st == 0, fp4q.fp4q_status_string(st)
    torch.cuda.synchronize()
    got = buf.float().cpu().numpy()
    want = np.full(n + guard, -3.0, np.float32)
    for r in range(rows):
        want[r * ldy + r] = 7.0
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt", ["nvfp4_razer", "nvfp4_razer_w"])
def test_separated_pipeline_lowers_the_error(orc, dev, fmt):
    """A 4096 x 4096 LLM weight (0.1 % outliers x20): the bulk's codes match the
    oracle's quantization of the oracle's bulk on sampled rows, and the
    reconstruction with the outliers scattered back has a lower error than
    quantizing x directly."""
    x = synthetic.llm_weight(4096, 4096, seed=61, device=dev)
    o = fp4q.separate_outliers(x)
    qb = fp4q.quantize(o.bulk, fmt)
    y = fp4q.scatter_outliers(o, fp4q.dequantize(qb, fmt))
    qx = fp4q.quantize(x, fmt)
    yx = fp4q.dequantize(qx, fmt)
    torch.cuda.synchronize()
    err_sep = ((y.double() - x.double()) ** 2).mean().item()
    err_dir = ((yx.double() - x.double()) ** 2).mean().item()
    assert err_sep < 0.8 * err_dir, (err_sep, err_dir)           # measured about 0.66
    pick = torch.tensor([0, 1, 2048, 4095], device=dev)
    bulk, _, _, _, _, _ = orc.separate_outliers(synthetic.bf16_bits(x[pick]))
    assert np.array_equal(synthetic.bf16_bits(o.bulk[pick]), bulk)
    rc, rs, _, _ = orc.quantize(bulk, fmt, tensor_scale=qb.tensor_scale.item(), want_sse=False)
    assert np.array_equal(qb.codes[pick].cpu().numpy(), rc) and np.array_equal(qb.scales[pick].cpu().numpy(), rs)


def test_separation_of_a_strided_matrix(orc, dev):
    """x with a row stride above cols: the same result as its dense copy."""
    big = _inputs(48, 2048 + 64, seed=77).to(dev)
    x = big[:, :2048]
    assert x.stride(0) == 2048 + 64
    o = fp4q.separate_outliers(x)
    od = fp4q.separate_outliers(x.contiguous())
    torch.cuda.synchronize()
    assert torch.equal(o.bulk, od.bulk) and torch.equal(o.count, od.count)
    assert torch.equal(o.cols, od.cols) and torch.equal(o.vals, od.vals)
    bulk, _, _, cnt, _, _ = orc.separate_outliers(synthetic.bf16_bits(x.contiguous()))
    assert np.array_equal(synthetic.bf16_bits(o.bulk), bulk) and np.array_equal(o.count.cpu().numpy(), cnt)
