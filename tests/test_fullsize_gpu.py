"""Whole-tensor oracle parity at full size: the benchmark's Llama-3-8B layers and
the Llama-3-70B MLP block, every row of every tensor compared with the oracle.

* Unrotated: codes, scales and tensor scale bit-exact; MSE within 1e-5 relative
  (only the fp64 summation order differs).
* MXFP4 with rotation: code mismatches (decision ties of the fp32 butterfly)
  at most 1e-4 of the elements, scales counted per element of their block;
  MSE within 1e-3 relative.
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


def _rel(a, b):
    return abs(a - b) / max(abs(b), 1e-300)


def _exact(orc, x: torch.Tensor, q, fmt):
    xb = synthetic.bf16_bits(x)
    rc, rs, rts, rsse = orc.quantize(xb, fmt, False)
    if fmt != "mxfp4":
        assert q.tensor_scale.item() == rts
    assert np.array_equal(q.scales.cpu().numpy(), rs)
    assert np.array_equal(q.codes.cpu().numpy(), rc)
    assert _rel(q.mse.item(), rsse / x.numel()) <= 1e-5


def test_two_llama3_8b_layers_in_one_batch_against_oracle(orc, dev):
    """Two full layers (14 tensors, 436 M elements) in one fp4q_quantize_batch call, so
    that the partial-sum slots rotate at real sizes; every tensor compared whole."""
    xs = [synthetic.llm_weight(r, c, seed=synthetic.tensor_seed(2, layer, i), device=dev)
          for layer in (0, 1) for i, (_, r, c) in enumerate(synthetic.LLAMA3_8B_LAYER)]
    got = fp4q.quantize_batch(xs, "nvfp4_razer", False)
    torch.cuda.synchronize()
    assert fp4q.fp4q_device_errors()[1] == 0
    for x, q in zip(xs, got):
        _exact(orc, x, q, "nvfp4_razer")


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "mxfp4", "nvfp4_razer_w"])
def test_llama3_70b_mlp_gate_and_down_against_oracle(orc, dev, fmt):
    """gate (28672 x 8192) and down (8192 x 28672), row scale LogNormal(0, 0.5) x
    N(0, 0.015^2), quantized whole by single calls and compared whole."""
    for i in (0, 2):
        _, r, c = synthetic.LLAMA3_70B_MLP[i]
        x = synthetic.mlp_row_scaled(r, c, seed=synthetic.tensor_seed(3, 0, i), device=dev)
        q = fp4q.quantize(x, fmt)
        torch.cuda.synchronize()
        _exact(orc, x, q, fmt)
        del x, q
        torch.cuda.empty_cache()


def test_llama3_70b_mlp_down_mxfp4_rotated_against_oracle(orc, dev):
    _, r, c = synthetic.LLAMA3_70B_MLP[2]
    x = synthetic.mlp_row_scaled(r, c, seed=synthetic.tensor_seed(3, 0, 2), device=dev)
    q = fp4q.quantize(x, "mxfp4", rotate=True)
    torch.cuda.synchronize()
    rc, rs, _, rsse = orc.quantize(synthetic.bf16_bits(x), "mxfp4", True)
    codes, scales = q.codes.cpu().numpy(), q.scales.cpu().numpy()
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(r, c)
    rnib = np.stack([rc & 15, rc >> 4], -1).reshape(r, c)
    bad = (nib != rnib) | np.repeat(scales != rs, 32, axis=1)
    assert bad.mean() <= 1e-4, f"{bad.sum()} of {x.numel()} codes differ"
    assert _rel(q.mse.item(), rsse / x.numel()) <= 1e-3
