"""fp4q_quantize_batch against per-tensor fp4q_quantize calls (and the oracle).

The batch must produce bit-identical codes, scales and tensor scales to calling
fp4q_quantize on each tensor in order; each MSE agrees to fp64 summation order.
"""
from __future__ import annotations

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


def _mixed_tensors(dev, fmt, rotate, seed=40):
    shapes = [(2048, 2048), (17, 96), (1, 64), (300, 4096), (5, 32), (64, 1024), (1024, 4096)]
    if fmt != "mxfp4" and not rotate:
        shapes += [(9, 80), (3, 16), (1, 4112)]          # cols % 32 == 16
    xs = [synthetic.llm_weight(r, c, seed=seed + i, device=dev) for i, (r, c) in enumerate(shapes)]
    big = synthetic.activation_t3(256, 1024, seed=seed + 99, device=dev)
    xs.append(big[:, :512])                               # strided rows
    xs.append(torch.zeros(0, 64, dtype=torch.bfloat16, device=dev))   # empty
    xs.append(torch.zeros(64, 64, dtype=torch.bfloat16, device=dev))  # all zero
    return xs


def _per_tensor(xs, fmt, rotate, scales=None):
    outs = []
    for i, x in enumerate(xs):
        ts = None if scales is None else scales[i].clone()
        outs.append(fp4q.quantize(x, fmt, rotate, tensor_scale=ts))
    torch.cuda.synchronize()
    return outs


def _compare(got, want, xs):
    for g, w, x in zip(got, want, xs):
        assert torch.equal(g.codes, w.codes)
        assert torch.equal(g.scales, w.scales)
        assert torch.equal(g.tensor_scale, w.tensor_scale)
        a, b = g.mse.item(), w.mse.item()
        assert a == b or abs(a - b) <= 1e-12 * abs(b)


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "mxfp4", "nvfp4_razer_w"])
@pytest.mark.parametrize("rotate", [False, True])
def test_batch_equals_per_tensor_calls(dev, fmt, rotate):
    xs = _mixed_tensors(dev, fmt, rotate)
    want = _per_tensor(xs, fmt, rotate)
    got = fp4q.quantize_batch(xs, fmt, rotate)
    torch.cuda.synchronize()
    _compare(got, want, xs)
    assert fp4q.fp4q_device_errors()[1] == 0


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "nvfp4_razer_w"])
def test_batch_with_given_scales(dev, fmt):
    xs = _mixed_tensors(dev, fmt, False, seed=50)
    scales = [torch.tensor([s], dtype=torch.float32, device=dev) for s in np.geomspace(1e-6, 1e-2, len(xs))]
    want = _per_tensor(xs, fmt, False, scales)
    outs = [fp4q.empty_like_quantized(x, fmt) for x in xs]
    for o, s in zip(outs, scales):
        o.tensor_scale.copy_(s)
    got = fp4q.quantize_batch(xs, fmt, False, outs=outs, scale_given=True)
    torch.cuda.synchronize()
    _compare(got, want, xs)


def test_batch_of_many_tensors(dev):
    """A long chain (250 tensors): partial slots rotate many times."""
    xs = [synthetic.llm_weight(32 + (i % 5) * 16, 256, seed=1000 + i, device=dev) for i in range(250)]
    want = _per_tensor(xs, "nvfp4_razer", False)
    got = fp4q.quantize_batch(xs, "nvfp4_razer", False)
    torch.cuda.synchronize()
    _compare(got, want, xs)


def test_batch_without_mse(dev):
    xs = [synthetic.llm_weight(512, 1024, seed=60 + i, device=dev) for i in range(4)]
    want = _per_tensor(xs, "nvfp4_razer", False)
    got = fp4q.quantize_batch(xs, "nvfp4_razer", False, want_mse=False)
    torch.cuda.synchronize()
    for g, w in zip(got, want):
        assert torch.equal(g.codes, w.codes) and torch.equal(g.scales, w.scales)
        assert g.mse is None


def test_batch_llama3_8b_layer_against_oracle(orc, dev):
    """One Llama-3-8B-shaped layer in one batch; sampled rows against the oracle."""
    xs = [synthetic.llm_weight(r, c, seed=synthetic.tensor_seed(2, 0, i), device=dev)
          for i, (_, r, c) in enumerate(synthetic.LLAMA3_8B_LAYER)]
    got = fp4q.quantize_batch(xs, "nvfp4_razer", False)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    for x, q in zip(xs, got):
        rows = x.shape[0]
        amax = max(orc.tensor_amax(synthetic.bf16_bits(x[r0:r0 + 4096])) for r0 in range(0, rows, 4096))
        ts = orc.tensor_scale_from_amax(amax)
        assert q.tensor_scale.item() == np.float32(ts)
        pick = np.unique(np.concatenate([[0, rows - 1], rng.choice(rows, 24, replace=False)]))
        idx = torch.from_numpy(pick).to(dev)
        rc, rs, _, _ = orc.quantize(synthetic.bf16_bits(x[idx]), "nvfp4_razer", False, tensor_scale=ts,
                                    want_sse=False)
        assert np.array_equal(q.codes[idx].cpu().numpy(), rc)
        assert np.array_equal(q.scales[idx].cpu().numpy(), rs)
