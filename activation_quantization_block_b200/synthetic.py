"""Seeded synthetic inputs shaped like the workloads block-FP4 quantization runs on.

This module draws random numbers and builds tensors; it holds none of the
quantization arithmetic, so both the CUDA path and the CPU oracle can be fed
from it.  Every generator takes an explicit seed and a torch device and uses
its own ``torch.Generator``: the same (seed, device) pair always gives the same
bytes.  Values are drawn in fp32 and rounded to bf16 (round to nearest even)
by ``Tensor.to(torch.bfloat16)``.

Workloads (sizes as used by the tests and the benchmark):

* LLM weight: N(0, 0.02^2), then exactly floor(0.001 * numel) entries at
  distinct uniform positions multiplied by 20 ("0.1 % outliers x20").
* Activation-like: column c has scale s_c ~ LogNormal(0, 1); entries are
  s_c * t, t Student-t with 3 degrees of freedom (z / sqrt(chi2_3 / 3)).
* 70B-style MLP weight: per-row scale ~ LogNormal(0, 0.5) times N(0, 0.015^2).
* Packed tensors for dequantization: uniform random nibbles; NVFP4 scale
  bytes uniform over the finite positive E4M3 codes 0x01..0x7E (bit 7 random
  for RaZeR), tensor scale 1; MXFP4 scale bytes 127 + U{-20..20}.
"""
from __future__ import annotations

import torch

# Llama-3-8B projection shapes (rows x cols of each bf16 weight matrix), one layer.
LLAMA3_8B_LAYER = (
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 14336, 4096),
    ("up_proj", 14336, 4096),
    ("down_proj", 4096, 14336),
)
LLAMA3_8B_LAYERS = 32

# Llama-3-70B MLP block shapes.
LLAMA3_70B_MLP = (
    ("gate_proj", 28672, 8192),
    ("up_proj", 28672, 8192),
    ("down_proj", 8192, 28672),
)


def tensor_seed(base: int, layer: int, index: int) -> int:
    """Seed of tensor ``index`` of layer ``layer`` in a workload whose seed is ``base``."""
    return int(base) * 1_000_000 + int(layer) * 100 + int(index)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def llm_weight(rows: int, cols: int, seed: int, device="cpu", std: float = 0.02,
               outlier_frac: float = 1e-3, outlier_mult: float = 20.0) -> torch.Tensor:
    """bf16 [rows, cols]: N(0, std^2) with floor(frac * numel) entries scaled by ``outlier_mult``."""
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).mul_(std)
    n = rows * cols
    k = int(outlier_frac * n)
    if k > 0:
        idx = torch.randperm(n, generator=g, device=device)[:k]
        x.view(-1)[idx] *= outlier_mult
    return x.to(torch.bfloat16)


def activation_t3(rows: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [rows, cols]: column scale LogNormal(0, 1) times Student-t(3) entries."""
    g = _gen(seed, device)
    s = torch.randn(cols, generator=g, device=device, dtype=torch.float32).exp_()
    z = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(rows, cols, device=device, dtype=torch.float32)
    for _ in range(3):
        chi2.add_(torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).square_())
    t = z.div_(chi2.div_(3.0).sqrt_())
    return t.mul_(s).to(torch.bfloat16)


def mlp_row_scaled(rows: int, cols: int, seed: int, device="cpu", std: float = 0.015,
                   row_sigma: float = 0.5) -> torch.Tensor:
    """bf16 [rows, cols]: per-row LogNormal(0, row_sigma) scale times N(0, std^2)."""
    g = _gen(seed, device)
    s = torch.randn(rows, 1, generator=g, device=device, dtype=torch.float32).mul_(row_sigma).exp_()
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).mul_(std)
    return x.mul_(s).to(torch.bfloat16)


def random_packed(rows: int, cols: int, fmt: str, seed: int, device="cpu"):
    """Random valid packed tensor: ``(codes u8 [rows, cols/2], scales u8 [rows, cols/B], tensor_scale f32 [1])``.

    ``fmt`` is "nvfp4", "nvfp4_razer", "mxfp4" (or "mxfp4_ceil", the same stored format) or
    "nvfp4_razer_w".
    """
    g = _gen(seed, device)
    codes = torch.randint(0, 256, (rows, cols // 2), generator=g, device=device, dtype=torch.int32)
    if fmt in ("mxfp4", "mxfp4_ceil"):
        scales = torch.randint(127 - 20, 127 + 21, (rows, cols // 32), generator=g, device=device,
                               dtype=torch.int32)
    elif fmt == "nvfp4_razer_w":
        # any 6-bit scale value, any of the four selectors
        scales = torch.randint(0, 256, (rows, cols // 16), generator=g, device=device, dtype=torch.int32)
    else:
        scales = torch.randint(1, 0x7F, (rows, cols // 16), generator=g, device=device,
                               dtype=torch.int32)
        if fmt == "nvfp4_razer":
            sign = torch.randint(0, 2, scales.shape, generator=g, device=device, dtype=torch.int32)
            scales = scales | (sign << 7)
    ts = torch.ones(1, device=device, dtype=torch.float32)
    return codes.to(torch.uint8), scales.to(torch.uint8), ts


def bf16_bits(x: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bit patterns (copied to host)."""
    return x.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")
