"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Tolerances (stated in the interface contract):
* unrotated paths: codes, scales and tensor scale bit-exact; bf16
  reconstruction bit-exact; MSE within 1e-5 relative (fp64 summation order);
* rotated paths: the fp32 butterfly may round where the oracle's sum is exact,
  so codes may differ at decision ties -- at most 1e-4 of elements -- and the
  MSE agrees within 1e-3 relative; given the same codes, the reconstruction
  agrees within 1e-6 of the group's largest magnitude before bf16 rounding
  (MXFP4 reconstructions are exact in fp32, hence bit-exact).
"""
from __future__ import annotations

import ml_dtypes
import numpy as np
import pytest
import torch

from activation_quantization_block_b200 import fp4q, synthetic
from tests import bruteforce as bf

pytestmark = pytest.mark.gpu

FMTS = ["nvfp4", "nvfp4_razer", "mxfp4", "nvfp4_razer_w"]
NV_FMTS = ["nvfp4", "nvfp4_razer", "nvfp4_razer_w"]


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def bits(t: torch.Tensor) -> np.ndarray:
    return synthetic.bf16_bits(t)


def run_gpu(x: torch.Tensor, fmt, rotate, tensor_scale=None, want_mse=True, guard=64, extra_flags=0):
    """Quantize through the C ABI into guarded buffers; check the guards; return numpy results."""
    rows, cols = x.shape
    B = fp4q.block_size(fmt)
    dev = x.device
    ncode, nscale = rows * cols // 2, rows * cols // B
    cbuf = torch.full((ncode + guard,), 0xA5, dtype=torch.uint8, device=dev)
    sbuf = torch.full((nscale + 16 + guard,), 0x5A, dtype=torch.uint8, device=dev)
    codes = cbuf[:ncode].view(rows, cols // 2)
    scales = sbuf[:nscale].view(rows, cols // B)
    ts = torch.zeros(1, dtype=torch.float32, device=dev) if tensor_scale is None else \
        torch.tensor([tensor_scale], dtype=torch.float32, device=dev)
    mse = torch.full((1,), -1.0, dtype=torch.float64, device=dev) if want_mse else None
    ws = torch.empty(fp4q.fp4q_workspace_size(rows, cols, fmt, rotate), dtype=torch.uint8, device=dev)
    ld = x.stride(0) if rows > 1 else cols
    flags = (fp4q.FLAG_TENSOR_SCALE_GIVEN if tensor_scale is not None else 0) | extra_flags
    st = fp4q.fp4q_quantize(x, rows, cols, ld, fmt, rotate, flags, codes, scales, ts, mse, ws, ws.numel())
    assert st == 0, fp4q.fp4q_status_string(st)
    torch.cuda.synchronize()
    assert torch.all(cbuf[ncode:] == 0xA5), "codes guard overwritten"
    assert torch.all(sbuf[nscale:] == 0x5A), "scales guard overwritten"
    return (codes.cpu().numpy(), scales.cpu().numpy(), np.float32(ts.item()),
            mse.item() if want_mse else None)


def run_dequant(codes, scales, ts, rows, cols, fmt, rotate, dev, ld=None, guard=32):
    ld = ld or cols
    c = torch.from_numpy(np.ascontiguousarray(codes)).to(dev)
    s = torch.from_numpy(np.ascontiguousarray(scales)).to(dev)
    t = torch.tensor([float(ts)], dtype=torch.float32, device=dev)
    ybuf = torch.full((rows * ld + guard,), -7.0, dtype=torch.bfloat16, device=dev)
    y = ybuf[:rows * ld].view(rows, ld)
    st = fp4q.fp4q_dequantize(c, s, t, rows, cols, fmt, rotate, y, ld)
    assert st == 0, fp4q.fp4q_status_string(st)
    torch.cuda.synchronize()
    assert torch.all(ybuf[rows * ld:] == -7.0)
    if ld > cols and rows > 0:
        assert torch.all(y[:, cols:] == -7.0), "padding columns overwritten"
    return bits(y[:, :cols])


def run_error(x, codes, scales, ts, fmt, rotate):
    dev = x.device
    rows, cols = x.shape
    c = torch.from_numpy(np.ascontiguousarray(codes)).to(dev)
    s = torch.from_numpy(np.ascontiguousarray(scales)).to(dev)
    t = torch.tensor([float(ts)], dtype=torch.float32, device=dev)
    mse = torch.full((1,), -1.0, dtype=torch.float64, device=dev)
    ws = torch.empty(fp4q.fp4q_workspace_size(rows, cols, fmt, rotate), dtype=torch.uint8, device=dev)
    ld = x.stride(0) if rows > 1 else cols
    st = fp4q.fp4q_error(x, ld, c, s, t, rows, cols, fmt, rotate, mse, ws, ws.numel())
    assert st == 0, fp4q.fp4q_status_string(st)
    torch.cuda.synchronize()
    return mse.item()


def rel(a, b):
    return abs(a - b) / max(abs(b), 1e-300)


def check_exact(orc, x: torch.Tensor, fmt, tensor_scale=None):
    """Unrotated: bit-exact codes/scales/tensor scale/dequant; MSE to 1e-5 (quantize and error)."""
    xb = bits(x)
    n = x.numel()
    codes, scales, ts, mse = run_gpu(x, fmt, False, tensor_scale)
    rc, rs, rts, rsse = orc.quantize(xb, fmt, False, tensor_scale=tensor_scale)
    assert np.array_equal(scales, rs)
    assert np.array_equal(codes, rc)
    if fmt != "mxfp4":
        assert ts == rts
    ref = rsse / n if n else 0.0
    assert (mse == 0.0 and ref == 0.0) or rel(mse, ref) <= 1e-5
    if n:
        y = run_dequant(codes, scales, ts, x.shape[0], x.shape[1], fmt, False, x.device)
        _, ry = orc.dequantize(rc, rs, rts, fmt, False)
        assert np.array_equal(y, ry)
        e = run_error(x, codes, scales, ts, fmt, False)
        assert (e == 0.0 and ref == 0.0) or rel(e, ref) <= 1e-5
    return codes, scales, ts, mse


def check_rotated(orc, x: torch.Tensor, fmt):
    xb = bits(x)
    n = x.numel()
    B = fp4q.block_size(fmt)
    codes, scales, ts, mse = run_gpu(x, fmt, True)
    rc, rs, rts, rsse = orc.quantize(xb, fmt, True)
    ref = rsse / n
    assert rel(mse, ref) <= 1e-3
    if fmt != "mxfp4":
        assert rel(float(ts), float(rts)) <= 1e-6
    # code mismatches, counting every element of a block whose scale differs
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(x.shape)
    rnib = np.stack([rc & 15, rc >> 4], -1).reshape(x.shape)
    bad = nib != rnib
    bad |= np.repeat(scales != rs, B, axis=1)
    assert bad.mean() <= 1e-4, f"{bad.sum()} of {n} codes differ"
    # error kernel on the GPU's own codes agrees with the oracle's error of those codes
    e = run_error(x, codes, scales, ts, fmt, True)
    assert rel(e, mse) <= 1e-4
    re_ = orc.error(xb, codes, scales, float(ts), fmt, True) / n
    assert rel(e, re_) <= 1e-4
    return codes, scales, ts


def check_dequant_rotated(orc, codes, scales, ts, rows, cols, fmt, dev):
    y = run_dequant(codes, scales, ts, rows, cols, fmt, True, dev)
    r32, r16 = orc.dequantize(codes, scales, float(ts), fmt, True)
    if fmt == "mxfp4":
        assert np.array_equal(y, r16)
        return
    gmax = np.repeat(np.abs(r32).reshape(rows, cols // 32, 32).max(-1), 32, axis=1)
    tol = (1e-6 * gmax).astype(np.float32)
    lo = (r32 - tol).astype(ml_dtypes.bfloat16).astype(np.float32)
    hi = (r32 + tol).astype(ml_dtypes.bfloat16).astype(np.float32)
    yf = (y.astype(np.uint32) << 16).view(np.float32)
    assert np.all((yf >= lo) & (yf <= hi))


# ------------------------------------------------------------------ workloads at parity sizes

def test_weight_2048_nvfp4_and_razer(orc, dev):
    """2048 x 2048 LLM weight, N(0, 0.02^2) with 0.1 % outliers x20, seed 0."""
    x = synthetic.llm_weight(2048, 2048, seed=0, device="cpu").to(dev)
    for fmt in NV_FMTS:
        check_exact(orc, x, fmt)


@pytest.mark.parametrize("rotate", [False, True])
def test_activation_t3_mxfp4(orc, dev, rotate):
    """Activation-like 8192 x 4096 (log-normal column scale x Student-t(3)), seed 1, MXFP4 +- rotation."""
    x = synthetic.activation_t3(8192, 4096, seed=1, device="cpu").to(dev)
    if rotate:
        codes, scales, ts = check_rotated(orc, x, "mxfp4")
        check_dequant_rotated(orc, codes[:512], scales[:512], ts, 512, 4096, "mxfp4", dev)
    else:
        check_exact(orc, x, "mxfp4")


@pytest.mark.parametrize("fmt", NV_FMTS)
def test_nvfp4_rotated(orc, dev, fmt):
    x = synthetic.activation_t3(512, 1024, seed=5, device="cpu").to(dev)
    codes, scales, ts = check_rotated(orc, x, fmt)
    check_dequant_rotated(orc, codes, scales, ts, 512, 1024, fmt, dev)


@pytest.mark.parametrize("fmt", FMTS)
def test_row_scaled_mlp_slice(orc, dev, fmt):
    """70B-style MLP weight rows (per-row log-normal(0, 0.5) x N(0, 0.015^2)), seed 3, a 1024 x 8192 slice."""
    x = synthetic.mlp_row_scaled(1024, 8192, seed=3, device="cpu").to(dev)
    check_exact(orc, x, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rotate", [False, True])
def test_dequantize_random_packed(orc, dev, fmt, rotate):
    """Seeded random codes and valid scales (seed 4), 8192 x 4096 and a ragged 3 x 4128."""
    for rows, cols in ((8192, 4096), (3, 4128)):
        codes, scales, ts = synthetic.random_packed(rows, cols, fmt, seed=4)
        c, s, t = codes.numpy(), scales.numpy(), float(ts[0])
        if rotate:
            check_dequant_rotated(orc, c, s, t, rows, cols, fmt, dev)
        else:
            y = run_dequant(c, s, t, rows, cols, fmt, False, dev)
            _, ry = orc.dequantize(c, s, t, fmt, False)
            assert np.array_equal(y, ry)


# ------------------------------------------------------------------ edge cases

def _bf(a) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, dtype=np.float32).astype(ml_dtypes.bfloat16).view(np.int16)).view(
        torch.bfloat16)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(1, 32), (1, 64), (3, 96), (7, 160), (33, 224), (1, 4096 + 32)])
def test_small_and_ragged_shapes(orc, dev, fmt, shape):
    x = synthetic.llm_weight(*shape, seed=sum(shape), device="cpu").to(dev)
    check_exact(orc, x, fmt)


@pytest.mark.parametrize("fmt", NV_FMTS)
@pytest.mark.parametrize("shape", [(1, 16), (3, 16), (5, 48), (9, 80), (1, 4112)])
def test_half_unit_shapes(orc, dev, fmt, shape):
    """cols % 32 == 16: units straddle rows and the last unit is a single block."""
    x = synthetic.llm_weight(*shape, seed=7, device="cpu").to(dev)
    check_exact(orc, x, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("cols,ld", [(64, 72), (96, 128), (48, 56), (32, 4096)])
def test_strided_rows(orc, dev, fmt, cols, ld):
    if cols % fp4q.block_size(fmt):
        pytest.skip("shape not allowed for the format")
    big = synthetic.llm_weight(37, ld, seed=9, device="cpu").to(dev)
    x = big[:, :cols]
    check_exact(orc, x, fmt)
    if cols % 32 == 0:
        check_rotated(orc, x, fmt)
    # strided output for dequantize
    codes, scales, ts, _ = run_gpu(x, fmt, False)
    y = run_dequant(codes, scales, ts, 37, cols, fmt, False, dev, ld=ld)
    _, ry = orc.dequantize(codes, scales, float(ts), fmt, False)
    assert np.array_equal(y, ry)


@pytest.mark.parametrize("fmt", FMTS)
def test_zeros_and_zero_rows(orc, dev, fmt):
    x = torch.zeros(8, 64, dtype=torch.bfloat16)
    codes, scales, ts, mse = check_exact(orc, x.to(dev), fmt)
    assert not codes.any() and not scales.any() and mse == 0.0 and ts == 0.0
    y = synthetic.llm_weight(8, 64, seed=3)
    y[2] = 0
    y[5, :32] = 0
    check_exact(orc, y.to(dev), fmt)


def _nibbles(codes: np.ndarray) -> np.ndarray:
    out = np.zeros((codes.shape[0], codes.shape[1] * 2), dtype=np.int64)
    out[:, 0::2] = codes & 0x0F
    out[:, 1::2] = codes >> 4
    return out


@pytest.mark.parametrize("fmt", FMTS)
def test_extreme_magnitudes(orc, dev, fmt):
    rng = np.random.default_rng(8)
    sub = rng.integers(1, 128, size=(4, 64)) * 2.0 ** -133 * rng.choice([-1, 1], size=(4, 64))
    sub[rng.random(sub.shape) < 0.2] = 0.0                          # zeros among them
    near = rng.uniform(-1.5, 1.5, size=(4, 64)) * 2.0 ** -126       # absmax up to 6 * 2^-128
    near[0, :7] = 0.0
    for tiny in (sub, near):
        # bf16 subnormals (and their neighbours): for NVFP4 formats every block's
        # RN(1 / den) overflows, and elements are scaled by division instead
        xt = _bf(tiny)
        codes, scales, ts, _ = check_exact(orc, xt.to(dev), fmt)
        assert np.all(_nibbles(codes)[bits(xt) == 0] == 0), "a zero must stay code +0"
        bcodes, bscales, bts = bf.quantize_bruteforce(bits(xt), fmt, False)
        assert np.array_equal(codes, bcodes) and np.array_equal(scales, bscales)
        if fmt != "mxfp4":
            assert ts == bts and 0 < ts < 2.0 ** -120
        check_rotated(orc, xt.to(dev), fmt)
    big = rng.standard_normal((4, 64)) * 1e37
    big[1, 3] = 3.3895313892515355e38                              # largest bf16
    big[2, 7] = -3.3895313892515355e38
    check_exact(orc, _bf(big).to(dev), fmt)
    mixed = rng.standard_normal((4, 64)) * 1e-3
    mixed[0, 0] = 1e30
    mixed[3, 5] = 1e-38
    check_exact(orc, _bf(mixed).to(dev), fmt)


@pytest.mark.parametrize("fmt", NV_FMTS)
def test_tensor_scale_given(orc, dev, fmt):
    x = synthetic.llm_weight(64, 256, seed=10, device="cpu").to(dev)
    for ts in (1.0, 3.0e-5, 2.0 ** -12, 0.0):
        check_exact(orc, x, fmt, tensor_scale=ts)


def test_representable_inputs_are_fixed_points(orc, dev):
    """Quantizing the bf16 reconstruction returns the same codes (all formats); what
    remains of the error is only the bf16 rounding of the reconstruction."""
    x = synthetic.llm_weight(128, 512, seed=12, device="cpu").to(dev)
    for fmt in FMTS:
        q = fp4q.quantize(x, fmt)
        y = fp4q.dequantize(q, fmt)
        q2 = fp4q.quantize(y, fmt)
        assert torch.equal(q.codes, q2.codes) and torch.equal(q.scales, q2.scales)
        assert q2.mse.item() < 1e-2 * q.mse.item()


def test_razer_worked_block_on_gpu(orc, dev):
    d = 448 * 2.0 ** -9
    x = np.zeros((1, 16), np.float32)
    x[0, 0], x[0, 1] = 6 * d, 5 * d
    for sign, sbyte in ((1, 0x7E), (-1, 0xFE)):
        codes, scales, ts, mse = check_exact(orc, _bf(sign * x).to(dev), "nvfp4_razer")
        assert scales[0, 0] == sbyte and (codes[0, 0] >> 4) == 8 and mse == 0.0


def test_razer_both_signs_tie_breaks(orc, dev):
    """Blocks holding candidates of both signs, including exact ties of the two gains."""
    rng = np.random.default_rng(13)
    d = 448 * 2.0 ** -9
    rows = []
    for _ in range(256):
        v = rng.choice([0.0, 0.5, 1.0, 3.0, -2.0], size=16)
        v[0] = 6.0
        k = rng.integers(1, 4)
        pos = rng.choice(np.arange(1, 16), size=2 * k, replace=False)
        mags = rng.choice([4.75, 5.0, 5.25, 4.875, 5.125], size=k)
        v[pos[:k]] = mags
        v[pos[k:]] = -rng.permutation(mags) if rng.random() < 0.5 else -rng.choice([4.75, 5.0, 5.25], size=k)
        rows.append(v * d)
    check_exact(orc, _bf(np.array(rows)).to(dev), "nvfp4_razer")


def test_razer_weight_worked_blocks_on_gpu(orc, dev):
    """RaZeR weight mode: a block at the largest E3M3 scale holding 6, and 2.5 or
    5 of either sign, is reproduced exactly with the selector of that value."""
    d = 30 * 2.0 ** -6                       # den = 30 * s_t with s_t = 2^-6
    for special, sel in ((5.0, 0), (-5.0, 1), (2.5, 2), (-2.5, 3)):
        x = np.zeros((1, 16), np.float32)
        x[0, 0], x[0, 1] = 6 * d, special * d
        codes, scales, ts, mse = check_exact(orc, _bf(x).to(dev), "nvfp4_razer_w", tensor_scale=2.0 ** -6)
        assert scales[0, 0] == (sel << 6) | 0x3F and (codes[0, 0] >> 4) == 8 and mse == 0.0


def test_razer_weight_candidates_and_ties(orc, dev):
    """Blocks with candidates of all four special values (gains of 5 and of 2.5
    equal, larger or smaller; both signs; exact ties go to the lower selector)."""
    rng = np.random.default_rng(21)
    d = 2.0 ** -3                            # block max 6 d: E3M3 16 (0x38), den = 16 * 2^-7
    rows = []
    for _ in range(512):
        v = rng.choice([0.0, 0.5, -1.0, 1.5, 3.0, -4.0], size=16)
        v[0] = 6.0
        pos = rng.permutation(np.arange(1, 16))
        n5, n2 = rng.integers(0, 4, size=2)
        m5 = rng.choice([4.625, 4.75, 4.875, 5.0, 5.125, 5.25, 5.375], size=n5)
        m2 = rng.choice([2.3125, 2.375, 2.4375, 2.5, 2.5625, 2.625, 2.6875], size=n2)
        v[pos[:n5]] = m5 * rng.choice([-1, 1], size=n5)
        v[pos[n5:n5 + n2]] = m2 * rng.choice([-1, 1], size=n2)
        rows.append(v * d)
    x = _bf(np.array(rows)).to(dev)
    codes, scales, _, _ = check_exact(orc, x, "nvfp4_razer_w", tensor_scale=2.0 ** -7)
    assert np.all(scales & 0x3F == 0x38)
    assert len(np.unique(scales >> 6)) == 4          # every selector occurs


def test_razer_weight_small_block_scales(orc, dev):
    """Blocks far below the tensor maximum: E3M3 subnormal scales (m * 2^-5),
    the boundary to the smallest normal (0.25) and the rounding ties there."""
    rng = np.random.default_rng(22)
    rows = rng.standard_normal((64, 256)) * 0.02
    rows[0, 0] = 30.0                                 # tensor maximum
    # block absmaxes a_b = t * 6 s_t for t near k * 2^-5 and 0.25
    s_t = np.float32(30.0) / np.float32(180.0)
    ts = np.concatenate([np.arange(1, 10) * 2.0 ** -5, np.arange(1, 10) * 2.0 ** -5 + 2.0 ** -6,
                         [0.2421875, 0.25, 0.2578125, 0.234375, 0.4 * 2.0 ** -5, 0.6 * 2.0 ** -5]])
    for i, t in enumerate(ts):
        r, b = 1 + i // 16, i % 16
        blk = rng.standard_normal(16) * 0.1 * t * 6 * s_t
        blk[rng.integers(16)] = t * 6 * s_t
        rows[r, 16 * b:16 * b + 16] = blk
    check_exact(orc, _bf(rows).to(dev), "nvfp4_razer_w")


def test_empty_tensor(dev):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    q = fp4q.quantize(x, "nvfp4_razer")
    torch.cuda.synchronize()
    assert q.tensor_scale.item() == 0.0 and q.mse.item() == 0.0 and q.codes.numel() == 0


# ------------------------------------------------------------------ full sizes, sampled

def _sampled_rows_check(orc, x: torch.Tensor, fmt, nrows=64, seed=0):
    """Whole-tensor quantize on the GPU; the oracle recomputes the tensor amax over
    the whole tensor and sampled rows one by one."""
    rows, cols = x.shape
    q = fp4q.quantize(x, fmt)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed)
    pick = np.unique(np.concatenate([[0, rows - 1], rng.choice(rows, nrows, replace=False)]))
    xs = bits(x[torch.from_numpy(pick).to(x.device)])
    ts = None
    if fmt != "mxfp4":
        amax = 0.0
        for r0 in range(0, rows, 4096):   # bounded host copies
            amax = max(amax, orc.tensor_amax(bits(x[r0:r0 + 4096])))
        ts = orc.tensor_scale_from_amax(amax, fmt)
        assert q.tensor_scale.item() == np.float32(ts)
    rc, rs, _, _ = orc.quantize(xs, fmt, False, tensor_scale=ts, want_sse=False)
    idx = torch.from_numpy(pick).to(x.device)
    assert np.array_equal(q.codes[idx].cpu().numpy(), rc)
    assert np.array_equal(q.scales[idx].cpu().numpy(), rs)
    # whole-tensor MSE: fused quantize pass vs the error kernel (independent partitions)
    e = fp4q.error(x, q, fmt)
    torch.cuda.synchronize()
    assert rel(q.mse.item(), e.item()) <= 1e-6
    return q


def test_llama3_8b_layer_sampled(orc, dev):
    """One Llama-3-8B-shaped layer (seed 2), NVFP4_RAZER, as the benchmark launches it."""
    for i, (name, r, c) in enumerate(synthetic.LLAMA3_8B_LAYER):
        x = synthetic.llm_weight(r, c, seed=synthetic.tensor_seed(2, 0, i), device=dev)
        _sampled_rows_check(orc, x, "nvfp4_razer", seed=i)
        del x


@pytest.mark.parametrize("fmt", FMTS)
def test_llama3_70b_mlp_sampled(orc, dev, fmt):
    name, r, c = synthetic.LLAMA3_70B_MLP[2]
    x = synthetic.mlp_row_scaled(r, c, seed=3, device=dev)
    _sampled_rows_check(orc, x, fmt, nrows=16)


# ------------------------------------------------------------------ MXFP4 exponent without clipping

def check_mx_ceil(orc, x: torch.Tensor, rotate=False):
    """GPU MXFP4 with FP4Q_FLAG_MX_CEIL_SCALE against the oracle's "mxfp4_ceil"."""
    xb = bits(x)
    n = x.numel()
    codes, scales, _, mse = run_gpu(x, "mxfp4", rotate, extra_flags=fp4q.FLAG_MX_CEIL_SCALE)
    rc, rs, _, rsse = orc.quantize(xb, "mxfp4_ceil", rotate)
    if not rotate:
        assert np.array_equal(scales, rs) and np.array_equal(codes, rc)
        assert rel(mse, rsse / n) <= 1e-5 or (mse == 0.0 and rsse == 0.0)
        y = run_dequant(codes, scales, 0.0, x.shape[0], x.shape[1], "mxfp4", False, x.device)
        _, ry = orc.dequantize(rc, rs, 0.0, "mxfp4_ceil", False)
        assert np.array_equal(y, ry)
    else:
        assert rel(mse, rsse / n) <= 1e-3
        nib = np.stack([codes & 15, codes >> 4], -1).reshape(x.shape)
        rnib = np.stack([rc & 15, rc >> 4], -1).reshape(x.shape)
        bad = (nib != rnib) | np.repeat(scales != rs, 32, axis=1)
        assert bad.mean() <= 1e-4
    return codes, scales, mse


@pytest.mark.parametrize("rotate", [False, True])
def test_mxfp4_ceil_activation_t3(orc, dev, rotate):
    x = synthetic.activation_t3(2048, 4096, seed=31, device="cpu").to(dev)
    _, scales, mse_c = check_mx_ceil(orc, x, rotate)
    _, scales_f, _, _ = run_gpu(x, "mxfp4", rotate)
    assert np.all(scales >= scales_f) and np.any(scales > scales_f)


@pytest.mark.parametrize("shape", [(1, 32), (7, 160), (33, 224), (1, 4096 + 32)])
def test_mxfp4_ceil_small_shapes_and_extremes(orc, dev, shape):
    check_mx_ceil(orc, synthetic.llm_weight(*shape, seed=sum(shape), device="cpu").to(dev))
    rng = np.random.default_rng(9)
    big = rng.standard_normal((4, 64)) * 1e37
    big[1, 3] = 3.3895313892515355e38
    check_mx_ceil(orc, _bf(big).to(dev))
    sub = rng.integers(1, 128, size=(4, 64)) * 2.0 ** -133 * rng.choice([-1, 1], size=(4, 64))
    check_mx_ceil(orc, _bf(sub).to(dev))
    m = np.array([1.0, 1.5, 1.5078125, 1.75, 1.9921875])           # significands around 1.5
    blocks = np.repeat(m[:, None], 32, axis=1) * 0.01
    check_mx_ceil(orc, _bf(blocks.reshape(1, -1)).to(dev))


def test_mxfp4_ceil_batch_equals_per_tensor(dev):
    xs = [synthetic.activation_t3(r, c, seed=40 + r, device=dev) for r, c in ((64, 256), (300, 1024), (5, 4096))]
    got = fp4q.quantize_batch(xs, "mxfp4", False, mx_ceil=True)
    for x, g in zip(xs, got):
        w = fp4q.quantize(x, "mxfp4", False, mx_ceil=True)
        torch.cuda.synchronize()
        assert torch.equal(g.codes, w.codes) and torch.equal(g.scales, w.scales)
        assert abs(g.mse.item() - w.mse.item()) <= 1e-12 * w.mse.item()


def test_single_level_nvfp4_full_size_sampled(orc, dev):
    """Single-level NVFP4 (tensor scale 1): N(0, 0.02^2) weights take E4M3 subnormal
    block scales; a 14336 x 4096 tensor, sampled rows against the oracle."""
    name, r, c = synthetic.LLAMA3_8B_LAYER[4]
    x = synthetic.llm_weight(r, c, seed=synthetic.tensor_seed(2, 0, 4), device=dev)
    for fmt in ("nvfp4", "nvfp4_razer"):
        ts = torch.ones(1, dtype=torch.float32, device=dev)
        q = fp4q.quantize(x, fmt, tensor_scale=ts)
        torch.cuda.synchronize()
        pick = np.array([0, 1, 777, r // 2, r - 1])
        idx = torch.from_numpy(pick).to(dev)
        rc, rs, _, _ = orc.quantize(bits(x[idx]), fmt, False, tensor_scale=1.0, want_sse=False)
        assert np.array_equal(q.codes[idx].cpu().numpy(), rc) and np.array_equal(q.scales[idx].cpu().numpy(), rs)
        assert np.mean((rs & 0x7F) < 0x08) > 0.5                       # most block scales are E4M3 subnormals
        e = fp4q.error(x, q, fmt)
        torch.cuda.synchronize()
        assert rel(q.mse.item(), e.item()) <= 1e-6


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "nvfp4_razer_w"])
def test_rotated_nvfp4_full_size_sampled(orc, dev, fmt):
    """Rotated NVFP4 formats on a full 14336 x 4096 tensor: the tensor scale from the
    rotated absmax, and sampled rows against the oracle (rotated tolerance)."""
    name, r, c = synthetic.LLAMA3_8B_LAYER[5]
    x = synthetic.llm_weight(r, c, seed=synthetic.tensor_seed(2, 0, 5), device=dev)
    q = fp4q.quantize(x, fmt, rotate=True)
    torch.cuda.synchronize()
    amax = 0.0
    for r0 in range(0, r, 4096):
        amax = max(amax, orc.tensor_amax(bits(x[r0:r0 + 4096]), rotate=True))
    ts = orc.tensor_scale_from_amax(amax, fmt)
    assert rel(q.tensor_scale.item(), float(ts)) <= 1e-6
    pick = np.unique(np.concatenate([[0, r - 1], np.random.default_rng(5).choice(r, 48, replace=False)]))
    idx = torch.from_numpy(pick).to(dev)
    rc, rs, _, _ = orc.quantize(bits(x[idx]), fmt, True, tensor_scale=q.tensor_scale.item(), want_sse=False)
    codes, scales = q.codes[idx].cpu().numpy(), q.scales[idx].cpu().numpy()
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(len(pick), c)
    rnib = np.stack([rc & 15, rc >> 4], -1).reshape(len(pick), c)
    bad = (nib != rnib) | np.repeat(scales != rs, 16, axis=1)
    assert bad.mean() <= 1e-4
    e = fp4q.error(x, q, fmt, rotate=True)
    torch.cuda.synchronize()
    assert rel(q.mse.item(), e.item()) <= 1e-4


def test_rejected_calls_leave_no_cuda_error_pending(dev):
    """Calls rejected by validation return before any CUDA call, so nothing is left pending:
    a valid call right after them (whose launches check cudaGetLastError) succeeds and matches
    a clean run."""
    x = synthetic.llm_weight(64, 256, seed=50, device="cpu").to(dev)
    want = fp4q.quantize(x, "nvfp4_razer")
    q = fp4q.empty_like_quantized(x, "nvfp4_razer")
    ws = torch.empty(fp4q.fp4q_workspace_size(64, 256, 1, 0), dtype=torch.uint8, device=dev)
    args = dict(x=x, rows=64, cols=256, ldx=256, fmt=1, rotate=0, flags=0, codes=q.codes, scales=q.scales,
                tensor_scale=q.tensor_scale, mse=q.mse, workspace=ws, workspace_bytes=ws.numel())
    for kw in (dict(fmt=7), dict(cols=40, ldx=40), dict(ldx=260), dict(codes=None), dict(workspace_bytes=16),
               dict(rows=-1), dict(flags=8)):
        assert fp4q.fp4q_quantize(**{**args, **kw}) != 0, kw
    y = torch.empty_like(x)
    assert fp4q.fp4q_dequantize(q.codes, q.scales, q.tensor_scale, 64, 256, 9, 0, y, 256) != 0
    assert fp4q.fp4q_tensor_scale(x, 64, 256, 256, 2, 0, q.tensor_scale, ws, ws.numel()) != 0
    assert fp4q.fp4q_quantize(**args) == 0
    torch.cuda.synchronize()
    assert torch.equal(q.codes, want.codes) and torch.equal(q.scales, want.scales)
    assert q.tensor_scale.item() == want.tensor_scale.item()
    assert rel(q.mse.item(), want.mse.item()) <= 1e-12
