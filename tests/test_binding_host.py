"""The torch-level wrappers of the binding on the CPU, with the C entry points replaced by
recorders: every wrapper allocates its outputs, passes them through in the C argument order,
and turns a non-success status into Fp4qError.  (The device checks themselves are in
test_abi.py; on a GPU the same wrappers run for real in every parity test.)"""
from __future__ import annotations

import contextlib

import pytest
import torch

from activation_quantization_block_b200 import fp4q


@pytest.fixture
def stubbed(monkeypatch):
    calls = []

    def recorder(name, status=0):
        def f(*args, **kw):
            calls.append((name, args))
            return status
        return f

    def first_device(*ts):
        for t in ts:
            if t is not None:
                return t.device
        raise TypeError("no tensor given")

    monkeypatch.setattr(fp4q, "_device", first_device)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(fp4q, "_stream", lambda s: 0)
    for name in ("fp4q_quantize", "fp4q_tensor_scale", "fp4q_quantize_batch", "fp4q_dequantize", "fp4q_error",
                 "fp4q_mma_pack", "fp4q_gemm", "fp4q_separate_outliers", "fp4q_scatter_outliers"):
        monkeypatch.setattr(fp4q, name, recorder(name))
    monkeypatch.setattr(fp4q, "fp4q_batch_workspace_size", lambda *a: 64)
    monkeypatch.setattr(fp4q, "fp4q_mma_planes", lambda f: 2 if fp4q._fmt(f) in (1, 3) else 1)
    monkeypatch.setattr(fp4q, "fp4q_mma_sf_bytes", lambda r, c: 512)
    monkeypatch.setattr(fp4q, "fp4q_outlier_capacity", lambda c, f: int(c * f))
    monkeypatch.setattr(fp4q, "workspace_for", lambda d, s=None: torch.empty(64, dtype=torch.uint8))
    return calls, recorder


def test_every_wrapper_reaches_its_entry_point(stubbed):
    calls, _ = stubbed
    x = torch.zeros(8, 64, dtype=torch.bfloat16)
    q = fp4q.quantize(x, "nvfp4_razer")
    assert q.codes.shape == (8, 32) and q.scales.shape == (8, 4) and q.mse.shape == (1,)
    assert fp4q.quantize(x, "mxfp4", want_mse=False).scales.shape == (8, 2)
    fp4q.quantize(x, tensor_scale=torch.ones(1), out=q)
    fp4q.tensor_scale(x)
    assert len(fp4q.quantize_batch([x, x])) == 2
    fp4q.quantize_batch([x], outs=[q], scale_given=True)
    y = fp4q.dequantize(q)
    assert y.shape == (8, 64) and y.dtype == torch.bfloat16
    fp4q.error(x, q)
    op = fp4q.mma_operand(q, "nvfp4_razer")
    assert op.nplanes == 2 and op.planes.shape == (8, 64)
    assert fp4q.gemm(op, op).shape == (8, 8)
    o = fp4q.separate_outliers(x)
    assert o.bulk.shape == (8, 64) and o.count.shape == (8,)
    fp4q.scatter_outliers(o, y)
    names = [n for n, _ in calls]
    assert names == ["fp4q_quantize", "fp4q_quantize", "fp4q_quantize", "fp4q_tensor_scale", "fp4q_quantize_batch",
                     "fp4q_quantize_batch", "fp4q_dequantize", "fp4q_error", "fp4q_mma_pack", "fp4q_gemm",
                     "fp4q_separate_outliers", "fp4q_scatter_outliers"]
    # flags: computed scale 0, given scale FLAG_TENSOR_SCALE_GIVEN; batch with scale_given likewise
    assert calls[0][1][6] == 0 and calls[2][1][6] == fp4q.FLAG_TENSOR_SCALE_GIVEN
    assert calls[5][1][4] == fp4q.FLAG_TENSOR_SCALE_GIVEN


def test_a_failing_status_raises(stubbed, monkeypatch):
    _, recorder = stubbed
    monkeypatch.setattr(fp4q, "fp4q_quantize", recorder("fp4q_quantize", status=2))
    with pytest.raises(fp4q.Fp4qError, match="FP4Q_ERROR_SHAPE"):
        fp4q.quantize(torch.zeros(8, 64, dtype=torch.bfloat16))


def test_gemm_checks_inner_dimensions(stubbed):
    a = fp4q.MmaOperand(torch.zeros(8, 128, dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8), torch.ones(1), 1)
    w = fp4q.MmaOperand(torch.zeros(8, 128, dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8), torch.ones(1), 2)
    with pytest.raises(ValueError, match="inner dimensions"):
        fp4q.gemm(a, w)
