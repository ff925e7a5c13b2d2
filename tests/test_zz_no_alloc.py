"""fp4q_quantize_noalloc, the entry point for callers that cannot allocate device
memory (a plugin inside a program that owns all GPU memory, or a latency path that
cannot afford an allocation): through the C ABI, its outputs must equal those of
fp4q_quantize, which takes a caller-allocated workspace -- on two calls in a row,
so that the second call runs on scratch the first one left behind.

This file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.
"""
from __future__ import annotations

import pytest
import torch

from activation_quantization_block_b200 import fp4q, synthetic

pytestmark = pytest.mark.gpu


def _outputs(x, fmt):
    rows, cols = x.shape
    B = fp4q.block_size(fmt)
    d = x.device
    return (torch.full((rows, cols // 2), 0xEE, dtype=torch.uint8, device=d),
            torch.full((rows, cols // B), 0xEE, dtype=torch.uint8, device=d),
            torch.full((1,), -1.0, dtype=torch.float32, device=d),
            torch.full((1,), -1.0, dtype=torch.float64, device=d))


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "mxfp4", "nvfp4_razer_w"])
@pytest.mark.parametrize("rotate", [0, 1])
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(fmt, rotate):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    # a large call, another shape, then a small one of much larger magnitude: its
    # few CTAs write only the first partial slots, so slots left behind by the
    # larger calls would change its tensor scale or its MSE if they were read
    xs = [synthetic.llm_weight(1024, 2048, seed=31, device=dev),
          synthetic.activation_t3(512, 4096, seed=32, device=dev),
          (synthetic.llm_weight(64, 256, seed=33, device=dev).float() * 1.0e3).to(torch.bfloat16)]
    for x in xs:   # one call after another, each on other data
        rows, cols = x.shape
        ref = _outputs(x, fmt)
        ws = torch.zeros(fp4q.fp4q_workspace_size(rows, cols, fmt, rotate), dtype=torch.uint8, device=dev)
        st = fp4q.fp4q_quantize(x, rows, cols, cols, fmt, rotate, 0, *ref, ws, ws.numel())
        assert st == 0, fp4q.fp4q_status_string(st)
        got = _outputs(x, fmt)
        st = fp4q.fp4q_quantize_noalloc(x, rows, cols, cols, fmt, rotate, 0, *got)
        assert st == 0, fp4q.fp4q_status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref[0])                     # codes: bit-exact
        assert torch.equal(got[1], ref[1])                     # scales: bit-exact
        assert torch.equal(got[2], ref[2])                     # tensor scale: bit-exact
        assert torch.equal(got[3], ref[3])                     # MSE: same kernels, same order, bit-exact


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    """Failure path on the GPU without a fault: a barrier that nothing completes.
    The bounded wait gives up after 2 s, the error word says so, and the next
    call quantizes correctly."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import time
    dev = torch.device("cuda:0")
    assert fp4q.fp4q_device_errors(clear=True)[0] == 0
    t0 = time.perf_counter()
    assert fp4q.fp4q_selftest_timeout() == 0
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 >= 1.5                       # the wait ran to its limit
    st, bits = fp4q.fp4q_device_errors(clear=True)
    assert st == 0 and bits == 0x1                                # FP4Q_DEVICE_ERROR_PIPELINE_TIMEOUT
    assert fp4q.fp4q_device_errors()[1] == 0                      # cleared
    x = synthetic.llm_weight(256, 1024, seed=5, device=dev)
    q = fp4q.quantize(x, "nvfp4_razer")
    y = fp4q.dequantize(q, "nvfp4_razer")
    torch.cuda.synchronize()
    assert fp4q.fp4q_device_errors()[1] == 0
    assert torch.isfinite(q.mse).all() and 0 < q.mse.item() < 1e-4 and y.shape == x.shape
