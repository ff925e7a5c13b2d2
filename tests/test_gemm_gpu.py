"""GPU parity of the tensor-core operand form and the W4A4 product.

* Operand form (fp4q_mma_pack): planes and scale atoms byte-exact against the
  oracle, from the same codes and scales.
* Product (fp4q_gemm): against the oracle's binary64 product of the two
  reconstructions.  The tensor cores multiply codes and scales exactly and
  accumulate in fp32; the tolerance per output is
      |y - Y| <= 2^-8 |Y| + (P K / 64 + 70) 2^-24 sum_k |a^_k w^_k|,
  the first term for the bf16 rounding of y (half an ulp is 2^-9 relative;
  doubled for the fp32 rounding of s_a s_w and of the scaling), the second for
  fp32 accumulation over P K / 64 MMA steps of 64 products each (P = a_np *
  w_np passes) plus the rounding of each reconstruction (x^ = RN(q RN(dec s_t))
  against the exact q dec s_t the tensor core uses).
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


def _quantized(orc, x, fmt):
    """GPU quantization of x, checked against the oracle's codes and scales."""
    q = fp4q.quantize(x, fmt, want_mse=False)
    torch.cuda.synchronize()
    rc, rs, rts, _ = orc.quantize(synthetic.bf16_bits(x), fmt, want_sse=False)
    assert np.array_equal(q.codes.cpu().numpy(), rc) and np.array_equal(q.scales.cpu().numpy(), rs)
    assert q.tensor_scale.item() == np.float32(rts)
    return q


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "nvfp4_razer_w"])
@pytest.mark.parametrize("shape", [(1, 16), (37, 592), (300, 1024), (128, 4096)])
def test_mma_pack_matches_oracle(orc, dev, fmt, shape):
    rows, cols = shape
    x = synthetic.llm_weight(rows, cols, seed=rows + cols, device="cpu").to(dev)
    q = _quantized(orc, x, fmt)
    op = fp4q.mma_operand(q, fmt)
    torch.cuda.synchronize()
    rp, rsf = orc.mma_pack(q.codes.cpu().numpy(), q.scales.cpu().numpy(), fmt)
    assert op.nplanes == orc.mma_planes(fmt)
    assert np.array_equal(op.planes.cpu().numpy(), rp)
    assert op.sf.numel() == rsf.size and np.array_equal(op.sf.cpu().numpy(), rsf)


def _check_gemm(orc, dev, a_fmt, w_fmt, M, N, K, seed):
    a = synthetic.activation_t3(M, K, seed=seed, device="cpu").to(dev)
    w = synthetic.llm_weight(N, K, seed=seed + 1, device="cpu").to(dev)
    qa, qw = _quantized(orc, a, a_fmt), _quantized(orc, w, w_fmt)
    oa, ow = fp4q.mma_operand(qa, a_fmt), fp4q.mma_operand(qw, w_fmt)
    y = fp4q.gemm(oa, ow)
    torch.cuda.synchronize()
    assert fp4q.fp4q_device_errors()[1] == 0
    ah, _ = orc.dequantize(qa.codes.cpu().numpy(), qa.scales.cpu().numpy(), qa.tensor_scale.item(), a_fmt)
    wh, _ = orc.dequantize(qw.codes.cpu().numpy(), qw.scales.cpu().numpy(), qw.tensor_scale.item(), w_fmt)
    Y, Yabs = orc.gemm(ah, wh)
    yf = y.float().cpu().numpy().astype(np.float64)
    passes = oa.nplanes * ow.nplanes
    tol = 2.0 ** -8 * np.abs(Y) + (passes * K / 64 + 70) * 2.0 ** -24 * Yabs
    bad = np.abs(yf - Y) > tol
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outputs out of tolerance; worst relative to sum|a w|: "
                           f"{(np.abs(yf - Y) / np.maximum(Yabs, 1e-300)).max():.3e}")
    return yf, Y


@pytest.mark.parametrize("a_fmt,w_fmt", [("nvfp4", "nvfp4"), ("nvfp4_razer", "nvfp4"),
                                         ("nvfp4", "nvfp4_razer_w"), ("nvfp4_razer", "nvfp4_razer_w"),
                                         ("nvfp4_razer", "nvfp4_razer")])
@pytest.mark.parametrize("M,N,K", [(200, 264, 512), (7, 8, 256), (512, 1024, 2048)])
def test_gemm_matches_oracle(orc, dev, a_fmt, w_fmt, M, N, K):
    _check_gemm(orc, dev, a_fmt, w_fmt, M, N, K, seed=M + N + K)


def test_gemm_razer_passes_matter(orc, dev):
    """Dropping the second plane (reading 0b1000 as -0, as the tensor core does)
    moves the product measurably: the special values are really counted."""
    M, N, K = 128, 256, 1024
    a = synthetic.activation_t3(M, K, seed=71, device="cpu").to(dev)
    w = synthetic.llm_weight(N, K, seed=72, device="cpu").to(dev)
    qa, qw = _quantized(orc, a, "nvfp4_razer"), _quantized(orc, w, "nvfp4_razer_w")
    oa, ow = fp4q.mma_operand(qa, "nvfp4_razer"), fp4q.mma_operand(qw, "nvfp4_razer_w")
    full = fp4q.gemm(oa, ow).float()
    one = fp4q.gemm(oa._replace(nplanes=1, planes=oa.planes[:, :K // 2].contiguous()),
                    ow._replace(nplanes=1, planes=ow.planes[:, :K // 2].contiguous())).float()
    torch.cuda.synchronize()
    assert (full - one).abs().max().item() > 0


def test_gemm_large_sampled(orc, dev):
    """A prefill-sized product (M 2048, N 4096, K 4096, RaZeR x weight mode):
    sampled rows against the oracle."""
    M, N, K = 2048, 4096, 4096
    a = synthetic.activation_t3(M, K, seed=81, device=dev)
    w = synthetic.llm_weight(N, K, seed=82, device=dev)
    qa, qw = fp4q.quantize(a, "nvfp4_razer", want_mse=False), fp4q.quantize(w, "nvfp4_razer_w", want_mse=False)
    oa, ow = fp4q.mma_operand(qa, "nvfp4_razer"), fp4q.mma_operand(qw, "nvfp4_razer_w")
    y = fp4q.gemm(oa, ow)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 127, 128, 1000, M - 1])
    idx = torch.from_numpy(rows).to(dev)
    ah, _ = orc.dequantize(qa.codes[idx].cpu().numpy(), qa.scales[idx].cpu().numpy(), qa.tensor_scale.item(),
                           "nvfp4_razer")
    wh, _ = orc.dequantize(qw.codes.cpu().numpy(), qw.scales.cpu().numpy(), qw.tensor_scale.item(),
                           "nvfp4_razer_w")
    Y, Yabs = orc.gemm(ah, wh)
    yf = y[idx].float().cpu().numpy().astype(np.float64)
    tol = 2.0 ** -8 * np.abs(Y) + (4 * K / 64 + 70) * 2.0 ** -24 * Yabs
    assert np.all(np.abs(yf - Y) <= tol)


@pytest.mark.parametrize("M,N,K,ldy", [(1, 264, 512, 264), (130, 520, 1280, 528), (257, 8, 768, 16)])
def test_gemm_ragged_shapes_and_strided_output(orc, dev, M, N, K, ldy):
    """M and N off the 128 / 256 tile grid, K an odd number of 256-element k-tiles, and an output
    row stride above N (the columns past N stay untouched)."""
    a = synthetic.activation_t3(M, K, seed=M, device="cpu").to(dev)
    w = synthetic.llm_weight(N, K, seed=N, device="cpu").to(dev)
    qa, qw = _quantized(orc, a, "nvfp4_razer"), _quantized(orc, w, "nvfp4_razer_w")
    buf = torch.full((M, ldy), -3.0, dtype=torch.bfloat16, device=dev)
    y = fp4q.gemm(fp4q.mma_operand(qa, "nvfp4_razer"), fp4q.mma_operand(qw, "nvfp4_razer_w"), out=buf[:, :N])
    torch.cuda.synchronize()
    if ldy > N:
        assert torch.all(buf[:, N:] == -3.0)
    ah, _ = orc.dequantize(qa.codes.cpu().numpy(), qa.scales.cpu().numpy(), qa.tensor_scale.item(), "nvfp4_razer")
    wh, _ = orc.dequantize(qw.codes.cpu().numpy(), qw.scales.cpu().numpy(), qw.tensor_scale.item(), "nvfp4_razer_w")
    Y, Yabs = orc.gemm(ah, wh)
    yf = y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(yf - Y) <= 2.0 ** -8 * np.abs(Y) + (4 * K / 64 + 70) * 2.0 ** -24 * Yabs)
