"""One tensor split by rows: fp4q_tensor_scale and quantize_row_sharded.

CPU (no GPU): the oracle shows that the row split reproduces the whole tensor
(the largest per-part tensor scale is the whole tensor's, the parts quantized
with it concatenate to the whole tensor's codes and scales, the error sums add
up); two gloo ranks run the exchange protocol of quantize_row_sharded with the
two local calls done by the oracle, including a rank that fails.

GPU: fp4q_tensor_scale equals the tensor scale fp4q_quantize computes (bit for
bit) and the oracle's; a split emulated on one device reproduces the whole
tensor through the C ABI; quantize_row_sharded without a group equals
fp4q.quantize.
"""
from __future__ import annotations

import datetime
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch

from activation_quantization_block_b200 import fp4q, shard, synthetic

FMTS = ["nvfp4", "nvfp4_razer", "mxfp4", "nvfp4_razer_w"]
NV_FMTS = ["nvfp4", "nvfp4_razer", "nvfp4_razer_w"]


def _splits(rows: int):
    """Row ranges of three parts: an empty one, a ragged one and the rest."""
    a = rows // 3 + 1
    return [(0, 0), (0, a), (a, rows)]


# ------------------------------------------------------------------ oracle, CPU

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rotate", [False, True])
def test_oracle_row_split_reproduces_the_whole_tensor(orc, fmt, rotate):
    x = synthetic.bf16_bits(synthetic.llm_weight(67, 96, seed=11))
    codes, scales, ts, sse = orc.quantize(x, fmt, rotate)
    parts = [x[a:b] for a, b in _splits(x.shape[0])]
    given = None
    if fmt != "mxfp4":
        part_ts = [orc.tensor_scale_from_amax(orc.tensor_amax(p, rotate), fmt) if p.shape[0] else 0.0
                   for p in parts]
        given = max(part_ts)
        assert np.float32(given) == ts
    outs = [orc.quantize(p, fmt, rotate, tensor_scale=given) for p in parts if p.shape[0]]
    assert np.array_equal(np.concatenate([o[0] for o in outs]), codes)
    assert np.array_equal(np.concatenate([o[1] for o in outs]), scales)
    total = sum(o[3] for o in outs)
    assert abs(total - sse) <= 1e-12 * sse


class _OracleOps:
    """The two local calls of quantize_row_sharded (tensor scale, quantize with it)
    done by the oracle on CPU tensors, with the binding's argument checks."""
    MXFP4 = fp4q.MXFP4
    Quantized = fp4q.Quantized
    _fmt = staticmethod(fp4q._fmt)

    def __init__(self, orc):
        self.orc = orc

    @staticmethod
    def _bits(x):
        if x.dtype != torch.bfloat16 or x.dim() != 2:
            raise TypeError("x must be a 2-D bf16 tensor")
        return synthetic.bf16_bits(x)

    def tensor_scale(self, x, fmt, rotate, out):
        b = self._bits(x)
        out[0] = self.orc.tensor_scale_from_amax(self.orc.tensor_amax(b, rotate), fmt) if b.shape[0] else 0.0
        return out

    def quantize(self, x, fmt, rotate, tensor_scale=None, want_mse=True):
        b = self._bits(x)
        rows, cols = b.shape
        if rows == 0:   # as the C ABI: nothing to encode, the error sum is 0
            codes = np.zeros((0, cols // 2), np.uint8)
            scales = np.zeros((0, cols // fp4q.block_size(fmt)), np.uint8)
            sse = 0.0
        else:
            given = None if tensor_scale is None else float(tensor_scale[0])
            codes, scales, _, sse = self.orc.quantize(b, fmt, rotate, tensor_scale=given, want_sse=want_mse)
        n = b.size
        mse = torch.tensor([sse / n if n else 0.0], dtype=torch.float64) if want_mse else None
        return fp4q.Quantized(torch.from_numpy(codes), torch.from_numpy(scales), tensor_scale, mse)


CASES = [("nvfp4_razer", False), ("nvfp4_razer_w", True), ("mxfp4", True), ("nvfp4", False)]


def _whole(rows=61, cols=128):
    return synthetic.llm_weight(rows, cols, seed=12)


def _rank_main(rank, world, port, split, out, fail_rank, fail_kind):
    import torch.distributed as dist
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        shard.fp4q = _OracleOps(oracle)
        x = _whole()
        x_local = x[split[rank]:split[rank + 1]]
        if rank == fail_rank:
            if fail_kind == "type":           # fails in the tensor-scale step
                x_local = x_local.float()
            else:                              # fails in the quantize step: cols not a multiple of 16
                x_local = x_local[:, :40].contiguous()
        res = []
        for fmt, rotate in (CASES if fail_rank < 0 else CASES[:1]):
            try:
                q = shard.quantize_row_sharded(x_local, fmt, rotate)
                res.append(("ok", fmt, rotate, q.codes.numpy(), q.scales.numpy(), float(q.tensor_scale[0]),
                            float(q.mse[0])))
            except RuntimeError as e:
                res.append(("raised", fmt, rotate, str(e)))
        out.put((rank, res))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_two_ranks(split, fail_rank=-1, fail_kind=""):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, split, q, fail_rank, fail_kind)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("split", [(0, 25, 61), (0, 0, 61)])
def test_two_gloo_ranks_quantize_one_tensor_split_by_rows(orc, split):
    res = _run_two_ranks(split)
    xb = synthetic.bf16_bits(_whole())
    for i, (fmt, rotate) in enumerate(CASES):
        r0, r1 = res[0][i], res[1][i]
        assert r0[0] == "ok" and r1[0] == "ok"
        codes, scales, ts, sse = orc.quantize(xb, fmt, rotate)
        assert np.array_equal(np.concatenate([r0[3], r1[3]]), codes)
        assert np.array_equal(np.concatenate([r0[4], r1[4]]), scales)
        for r in (r0, r1):
            if fmt != "mxfp4":
                assert np.float32(r[5]) == ts
            assert abs(r[6] - sse / xb.size) <= 1e-12 * (sse / xb.size)


@pytest.mark.parametrize("fail_kind", ["type", "shape"])
def test_a_failing_rank_makes_every_rank_raise(orc, fail_kind):
    res = _run_two_ranks((0, 25, 61), fail_rank=1, fail_kind=fail_kind)
    assert res[1][0][0] == "raised" and "local call failed" in res[1][0][3]
    assert res[0][0][0] == "raised" and "1 other rank" in res[0][0][3]


def test_single_process_needs_no_group(orc, monkeypatch):
    monkeypatch.setattr(shard, "fp4q", _OracleOps(orc))
    x = _whole()
    q = shard.quantize_row_sharded(x, "nvfp4_razer", False)
    codes, scales, ts, sse = orc.quantize(synthetic.bf16_bits(x), "nvfp4_razer", False)
    assert np.array_equal(q.codes.numpy(), codes) and np.array_equal(q.scales.numpy(), scales)
    assert np.float32(q.tensor_scale[0].item()) == ts
    assert abs(q.mse.item() - sse / x.numel()) <= 1e-12 * sse / x.numel()


# ------------------------------------------------------------------ CUDA path

@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _tensor_scale_guarded(x, fmt, rotate):
    """fp4q_tensor_scale into slot 1 of a 4-float buffer; the other slots must stay untouched."""
    buf = torch.full((4,), -7.0, dtype=torch.float32, device=x.device)
    out = fp4q.tensor_scale(x, fmt, rotate, out=buf[1:2])
    torch.cuda.synchronize()
    host = buf.cpu()
    assert host[0] == -7.0 and host[2] == -7.0 and host[3] == -7.0
    return np.float32(out.item())


SHAPES = [(3, 64), (129, 4096), (1000, 96), (14336, 4096)]
_inputs: dict = {}


def _weight(shape):
    """Seeded LLM-weight input of this shape (bf16 on the CPU), generated once per module."""
    if shape not in _inputs:
        _inputs[shape] = synthetic.llm_weight(*shape, seed=13, device="cpu")
    return _inputs[shape]


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", NV_FMTS)
@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_tensor_scale_equals_the_quantize_scale_and_the_oracle(orc, dev, fmt, rotate, shape):
    x = _weight(shape).to(dev)
    ts = _tensor_scale_guarded(x, fmt, rotate)
    q = fp4q.quantize(x, fmt, rotate, want_mse=False)
    assert ts == np.float32(q.tensor_scale.item())
    want = np.float32(orc.tensor_scale_from_amax(orc.tensor_amax(synthetic.bf16_bits(x), rotate), fmt))
    if rotate:
        assert abs(float(ts) - float(want)) <= 1e-6 * float(want)
    else:
        assert ts == want


@pytest.mark.gpu
def test_tensor_scale_of_a_strided_view(orc, dev):
    wide = synthetic.llm_weight(257, 4160, seed=14, device="cpu").to(dev)
    x = wide[:, 32:32 + 4096]
    for fmt in NV_FMTS:
        ts = _tensor_scale_guarded(x, fmt, False)
        want = orc.tensor_scale_from_amax(orc.tensor_amax(synthetic.bf16_bits(x), False), fmt)
        assert ts == np.float32(want)


@pytest.mark.gpu
def test_tensor_scale_of_an_empty_tensor_is_zero(dev):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    assert _tensor_scale_guarded(x, "nvfp4_razer", False) == 0.0


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rotate", [False, True])
def test_row_split_on_one_device_reproduces_the_whole_tensor(dev, fmt, rotate):
    """The exchange emulated on one device: parts in turn, the maximum scale taken between."""
    x = synthetic.llm_weight(4099, 1024, seed=15, device="cpu").to(dev)
    whole = fp4q.quantize(x, fmt, rotate)
    parts = [x[a:b] for a, b in _splits(x.shape[0])]
    given = None
    if fmt != "mxfp4":
        given = torch.stack([fp4q.tensor_scale(p, fmt, rotate) for p in parts]).max().reshape(1)
        assert given.item() == whole.tensor_scale.item()
    outs = [fp4q.quantize(p, fmt, rotate, tensor_scale=given) for p in parts]
    assert torch.equal(torch.cat([o.codes for o in outs]), whole.codes)
    assert torch.equal(torch.cat([o.scales for o in outs]), whole.scales)
    sse = sum(o.mse.item() * p.numel() for o, p in zip(outs, parts))
    ref = whole.mse.item()
    assert abs(sse / x.numel() - ref) <= 1e-12 * ref


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_row_sharded_without_a_group_equals_quantize(dev, fmt):
    x = synthetic.llm_weight(1000, 2048, seed=16, device="cpu").to(dev)
    q = shard.quantize_row_sharded(x, fmt, False)
    w = fp4q.quantize(x, fmt, False)
    assert torch.equal(q.codes, w.codes) and torch.equal(q.scales, w.scales)
    if fmt != "mxfp4":
        assert q.tensor_scale.item() == w.tensor_scale.item()
    assert abs(q.mse.item() - w.mse.item()) <= 1e-14 * w.mse.item()
