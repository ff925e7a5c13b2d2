"""Pins for the CPU oracle: checks against what the papers and the mathematics fix.

None of these compares the oracle with itself.  Each pin comes from the papers'
printed values (``tests/golden``), an exhaustive enumeration, exact rational
arithmetic, a library cast (``ml_dtypes``, ``scipy``), a closed form or an
invariant -- chosen so that a dropped term, a wrong sign, a wrong tie rule, a
swapped nibble or a mis-indexed scale fails at least one of them.
"""
from __future__ import annotations

import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import scipy.linalg

from tests import bruteforce as bf

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- E2M1 elements

def test_e2m1_value_set_is_the_papers_set(orc):
    page = sorted(float(r[0]) for r in bf.read_golden("e2m1_value_set.txt"))
    mine = sorted(orc.e2m1_value(c) for c in range(16))
    assert mine == page
    # sign-magnitude: code | 8 is the negation, -0 included
    for c in range(8):
        assert orc.e2m1_value(c | 8) == -orc.e2m1_value(c)
        assert math.copysign(1.0, orc.e2m1_value(c | 8)) == -1.0


def test_e2m1_decode_matches_bit_fields_and_ml_dtypes(orc):
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    for c in range(16):
        assert orc.e2m1_value(c) == bf.e2m1_from_bits(c) == float(lib[c])


def _e2m1_sweep():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    pts = set(grid)
    for a, b in zip(grid, grid[1:]):
        m = np.float32((a + b) / 2)
        pts.update([float(m), float(np.nextafter(m, np.float32(0))), float(np.nextafter(m, np.float32(9)))])
    for g in grid:
        g32 = np.float32(g)
        pts.update([float(np.nextafter(g32, np.float32(-1))), float(np.nextafter(g32, np.float32(9)))])
    pts.update([7.0, 100.0, 3.0e38, 1e-40, 2 ** -149, 0.2499999, 5.5, 4.5])
    rng = np.random.default_rng(11)
    pts.update(float(v) for v in rng.uniform(0, 8, 3000).astype(np.float32))
    vals = sorted(pts)
    return [v for v in vals] + [-v for v in vals]


def test_e2m1_encode_equals_exhaustive_argmin(orc):
    for v in _e2m1_sweep():
        assert orc.e2m1_encode(v) == bf.e2m1_nearest(v), v


def test_e2m1_encode_ties_follow_even_code():
    # the tie rule fixed for the oracle, checked against ml_dtypes' RNE cast
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    expect = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    got = ties.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)
    assert list(got) == expect


def test_e2m1_encode_agrees_with_ml_dtypes_cast(orc):
    sweep = np.array(_e2m1_sweep(), dtype=np.float32)
    lib = sweep.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)
    for v, l in zip(sweep, lib):
        mine = orc.e2m1_value(orc.e2m1_encode(float(v)))
        assert mine == l  # equal as values; -0 == +0 (the oracle canonicalises zero)
        if mine == 0:
            assert orc.e2m1_encode(float(v)) == 0


# ---------------------------------------------------------------- E4M3 scales

def test_e4m3_decode_all_bytes(orc):
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for b in range(256):
        if b & 0x7F == 0x7F:
            assert math.isnan(orc.e4m3_value(b))
            continue
        assert orc.e4m3_value(b) == bf.e4m3_from_bits(b) == lib[b], b
    assert orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x01) == 2.0 ** -9


def _e4m3_sweep():
    vals = [float(v) for v in bf.E4M3_POS]
    pts = set(vals)
    for a, b in zip(vals, vals[1:]):
        m = np.float32((a + b) / 2)
        pts.update([float(m), float(np.nextafter(m, np.float32(0))), float(np.nextafter(m, np.float32(1e9)))])
    rng = np.random.default_rng(12)
    pts.update(float(v) for v in rng.uniform(0, 460, 2000).astype(np.float32))
    pts.update(float(v) for v in np.exp2(rng.uniform(-12, 9, 2000)).astype(np.float32))
    pts.update([0.0, 448.0, 450.0, 464.0, 470.0, 1e6, 1e-30, 2 ** -10, 3 * 2 ** -11])
    return sorted(pts)


def test_e4m3_encode_equals_exhaustive_argmin(orc):
    for t in _e4m3_sweep():
        assert orc.e4m3_encode(t) == bf.e4m3_nearest(t), t


def test_e4m3_encode_saturates_and_matches_ml_dtypes_in_range(orc):
    sweep = np.array(_e4m3_sweep(), dtype=np.float32)
    inr = sweep[sweep <= 448]
    lib = inr.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    for t, b in zip(inr, lib):
        assert orc.e4m3_encode(float(t)) == int(b), t
    for t in sweep[sweep > 448]:
        assert orc.e4m3_encode(float(t)) == 0x7E


# ---------------------------------------------------------------- E8M0 / MXFP4 exponent

def test_e8m0_decode(orc):
    lib = np.arange(255, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    for b in range(255):
        assert orc.e8m0_value(b) == lib[b] == 2.0 ** (b - 127)
    assert math.isnan(orc.e8m0_value(255))


def test_mx_exponent_is_floor_log2_minus_two(orc):
    rng = np.random.default_rng(13)
    pts = [float(v) for v in np.exp2(rng.uniform(-140, 127, 3000)).astype(np.float32) if v > 0]
    for k in range(-149, 128):
        p = np.float32(2.0 ** k)
        pts += [float(p), float(np.nextafter(p, np.float32(0)))]
    pts = [p for p in pts if p > 0 and math.isfinite(p)]
    for a in pts:
        want = max(-127, min(127, bf.floor_log2(a) - 2))
        assert orc.mx_exponent(a) == want, a


# ---------------------------------------------------------------- bf16

def test_bf16_rounding_matches_ml_dtypes(orc):
    rng = np.random.default_rng(14)
    v = rng.standard_normal(4000).astype(np.float32) * np.float32(3.0)
    # exact ties: a bf16 value plus half of its last place
    base = v.astype(ml_dtypes.bfloat16).astype(np.float32)
    ties = (base.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    allv = np.concatenate([v, ties, np.float32([0.0, -0.0, 1e-40, -3e38])])
    want = allv.astype(ml_dtypes.bfloat16).view(np.uint16)
    got = orc.f32_to_bf16(allv)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- rotation

def test_hadamard_is_sylvester(orc):
    H = np.array([[orc.hadamard_entry(i, j) for j in range(32)] for i in range(32)])
    assert np.array_equal(H, scipy.linalg.hadamard(32))
    assert np.array_equal(H @ H.T, 32 * np.eye(32, dtype=H.dtype))


def test_wht_constant_is_rn_of_inverse_sqrt32(orc):
    c = np.float32(orc.wht_constant())
    # c is the binary32 nearest to 1/sqrt(32): compare squares exactly against 1/32
    lo, hi = np.nextafter(c, np.float32(0)), np.nextafter(c, np.float32(1))
    target = Fraction(1, 32)
    # the true value lies between the midpoints (lo+c)/2 and (c+hi)/2
    assert (Fraction(float(lo)) + Fraction(float(c))) ** 2 / 4 < target
    assert (Fraction(float(c)) + Fraction(float(hi))) ** 2 / 4 > target


def test_wht_closed_forms(orc):
    c = np.float32(orc.wht_constant())
    e0 = np.zeros(32, np.float32); e0[0] = 1
    assert np.all(orc.wht32(e0) == c)                               # delta -> flat
    y = orc.wht32(np.ones(32, np.float32))
    assert y[0] == np.float32(np.float32(32) * c) and np.all(y[1:] == 0)   # flat -> delta
    H = scipy.linalg.hadamard(32).astype(np.float32)
    for k in (1, 5, 17, 31):                                          # Walsh row k -> delta at k
        y = orc.wht32(H[k])
        assert y[k] == np.float32(np.float32(32) * c)
        assert np.count_nonzero(y) == 1


def test_wht_orthogonal_involution(orc):
    rng = np.random.default_rng(15)
    for _ in range(50):
        x = rng.standard_normal(32).astype(np.float32)
        y = orc.wht32(x)
        assert abs(np.linalg.norm(y.astype(np.float64)) / np.linalg.norm(x.astype(np.float64)) - 1) < 1e-6
        z = orc.wht32(y)
        ulp = np.spacing(np.abs(x).max())
        assert np.max(np.abs(z - x)) <= 2 * ulp


def test_wht_equals_exact_rational_transform(orc):
    rng = np.random.default_rng(16)
    H = bf.sylvester_hadamard(32)
    c = np.float32(orc.wht_constant())
    for _ in range(20):
        xb = (rng.standard_normal(32).astype(np.float32)).astype(ml_dtypes.bfloat16).astype(np.float32)
        got = orc.wht32(xb)
        for i in range(32):
            s = sum((int(H[i, j]) * Fraction(float(xb[j])) for j in range(32)), Fraction(0))
            assert got[i] == np.float32(bf.rn_f32(s) * c)


# ---------------------------------------------------------------- tensor scale (two-level NVFP4)

def test_tensor_scale_maps_amax_to_6x448(orc):
    for k in range(-20, 20):
        assert orc.tensor_scale_from_amax(2688.0 * 2.0 ** k) == 2.0 ** k


def test_tensor_amax_is_the_largest_magnitude(orc):
    x = (np.random.default_rng(21).standard_normal((300, 256)) * 0.02).astype(np.float32)
    x[123, 45] = -0.75
    xb = orc.f32_to_bf16(x)
    assert orc.tensor_amax(xb, False) == np.abs(bf.bits_to_f32(xb)).max() == 0.75


@pytest.mark.parametrize("fmt,c", [("nvfp4", 2688), ("nvfp4_razer_w", 180)])
def test_tensor_scale_is_the_rounded_quotient_and_monotone(orc, fmt, c):
    """s_t = RN(A / c): checked against the exact quotient rounded once, and monotone in A
    (what lets parts of a row-split tensor exchange their s_t instead of their absmax)."""
    rng = np.random.default_rng(22)
    a = np.sort(np.concatenate([rng.uniform(0, 50, 400), 10.0 ** rng.uniform(-30, 30, 400)]).astype(np.float32))
    a = np.concatenate([a, np.nextafter(a, np.float32(np.inf))])
    a.sort()
    st = [orc.tensor_scale_from_amax(float(v), fmt) for v in a]
    for v, s_ in zip(a, st):
        assert np.float32(s_) == bf.rn_f32(Fraction(float(v)) / c)
    assert all(x <= y for x, y in zip(st, st[1:]))


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer"])
def test_max_block_gets_scale_448(orc, fmt):
    rng = np.random.default_rng(17)
    x = (rng.standard_normal((4, 64)) * 0.02).astype(np.float32)
    x[2, 37] = 2688.0 * 2.0 ** -7   # tensor max, exactly 6 * 448 * 2^-7
    xb = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    codes, scales, ts, _ = orc.quantize(xb, fmt)
    assert ts == np.float32(2.0 ** -7)
    assert scales[2, 37 // 16] & 0x7F == 0x7E
    nib = bf.unpack_codes(codes, 64)
    assert nib[2, 37] == 7   # +6


# ---------------------------------------------------------------- brute force on tiny tensors

def _tiny_inputs():
    rng = np.random.default_rng(18)
    out = []
    x = (rng.standard_normal((3, 64)) * 0.02).astype(np.float32)
    x.ravel()[rng.choice(x.size, 3, replace=False)] *= 20
    out.append(x)
    t = rng.standard_t(3, size=(2, 64)).astype(np.float32) * np.exp(rng.standard_normal(64)).astype(np.float32)
    out.append(t)
    z = np.zeros((2, 32), np.float32); z[1, 5] = -3.0
    out.append(z)
    return [a.astype(ml_dtypes.bfloat16).view(np.uint16) for a in out]


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "mxfp4", "nvfp4_razer_w", "mxfp4_ceil"])
@pytest.mark.parametrize("rotate", [False, True])
def test_quantize_equals_bruteforce(orc, fmt, rotate):
    for xb in _tiny_inputs():
        codes, scales, ts, sse = orc.quantize(xb, fmt, rotate)
        bcodes, bscales, bts = bf.quantize_bruteforce(xb, fmt, rotate, pair2=orc.razer_w_pair())
        assert np.array_equal(codes, bcodes)
        assert np.array_equal(scales, bscales)
        if fmt != "mxfp4":
            assert ts == bts
        xhat = bf.dequantize_bruteforce(bcodes, bscales, bts, fmt, rotate, pair2=orc.razer_w_pair())
        exact = bf.sse_exact(xb, xhat)
        assert abs(sse - float(exact)) <= 1e-12 * max(1.0, float(exact))


def _tiny_magnitude_inputs():
    """bf16 tensors whose absmax lies between 2^-133 (the smallest bf16
    subnormal) and 6 * 2^-128, zeros included.  Their block scales
    den = RN(dec(sb) * s_t) fall below 2^-128, where RN(1 / den) overflows."""
    rng = np.random.default_rng(23)
    out = []
    k = rng.integers(-127, 128, size=(4, 32)).astype(np.float64)   # subnormal multiples of 2^-133
    k[rng.random(k.shape) < 0.25] = 0.0
    out.append(k * 2.0 ** -133)
    top = rng.uniform(-1.5, 1.5, size=(2, 64)) * 2.0 ** -126          # up to 6 * 2^-128
    top[0, :5] = 0.0
    top[1, 7] = 1.5 * 2.0 ** -126
    out.append(top)
    one = np.zeros((1, 32)); one[0, 3] = 2.0 ** -133; one[0, 20] = -2.0 ** -133
    out.append(one)
    return [a.astype(np.float32).astype(ml_dtypes.bfloat16).view(np.uint16) for a in out]


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "nvfp4_razer_w"])
@pytest.mark.parametrize("rotate", [False, True])
def test_overflowing_block_reciprocal_equals_bruteforce(orc, fmt, rotate):
    """Where RN(1 / den) is infinite the elements are scaled by exact division
    (rounded once), so each goes to its nearest code and zeros stay +0."""
    for xb in _tiny_magnitude_inputs():
        codes, scales, ts, sse = orc.quantize(xb, fmt, rotate)
        assert 0 < ts < 2.0 ** -120
        bcodes, bscales, bts = bf.quantize_bruteforce(xb, fmt, rotate, pair2=orc.razer_w_pair())
        assert np.array_equal(codes, bcodes)
        assert np.array_equal(scales, bscales)
        assert ts == bts
        nib = bf.unpack_codes(codes, xb.shape[1])
        if not rotate:
            assert np.all(nib[xb == 0] == 0)                 # zeros stay +0
            nz = bf.bits_to_f32(xb) != 0
            if nz.sum() > 8:                                  # not everything saturated to +-6
                assert not np.all(np.isin(nib[nz], (7, 15)))
        xhat = bf.dequantize_bruteforce(bcodes, bscales, bts, fmt, rotate, pair2=orc.razer_w_pair())
        exact = bf.sse_exact(xb, xhat)
        assert abs(sse - float(exact)) <= 1e-12 * max(float(exact), 2.0 ** -300)


def test_overflowing_reciprocal_codes_are_nearest_to_the_exact_quotient(orc):
    """Closed form, unrotated NVFP4: every code is the E2M1 value nearest to
    RN(y / den), with den = RN(dec(sb) * s_t) from the scale byte the oracle wrote."""
    for xb in _tiny_magnitude_inputs():
        codes, scales, ts, _ = orc.quantize(xb, "nvfp4")
        x = bf.bits_to_f32(xb)
        nib = bf.unpack_codes(codes, xb.shape[1])
        for r in range(x.shape[0]):
            for j in range(x.shape[1]):
                den = np.float32(np.float32(bf.E4M3_POS[int(scales[r, j // 16])]) * ts)
                if den == 0:
                    assert nib[r, j] == 0
                    continue
                assert np.isinf(np.float32(1.0) / den) or den >= 2.0 ** -128
                v = bf.rn_f32_exact(Fraction(float(x[r, j])) / Fraction(float(den)))
                assert nib[r, j] == bf.e2m1_nearest(float(v))


def test_e2m1_encoder_refuses_nan(orc):
    assert orc.e2m1_encode(float("nan")) == -1
    xb = np.zeros((1, 16), np.float32)
    xb[0, 3] = 1.0
    xb[0, 5] = np.nan
    with pytest.raises(FloatingPointError):
        orc.quantize(xb.astype(ml_dtypes.bfloat16).view(np.uint16), "nvfp4")


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "mxfp4", "nvfp4_razer_w", "mxfp4_ceil"])
@pytest.mark.parametrize("rotate", [False, True])
def test_dequantize_equals_bruteforce(orc, fmt, rotate):
    import torch
    from activation_quantization_block_b200 import synthetic
    codes, scales, ts = synthetic.random_packed(3, 64, fmt, seed=4)
    codes, scales = codes.numpy(), scales.numpy()
    ts = float(ts[0]) * 2.0 ** -6
    y32, y16 = orc.dequantize(codes, scales, ts, fmt, rotate)
    want = bf.dequantize_bruteforce(codes, scales, ts, fmt, rotate, pair2=orc.razer_w_pair())
    assert np.array_equal(y32.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(y16, want.astype(ml_dtypes.bfloat16).view(np.uint16))
    del torch


# ---------------------------------------------------------------- idempotence on representable inputs

def _representable(fmt, rows=4, cols=64, seed=19):
    """x = value(code) * scale exactly, with a +-6 (MXFP4: +-6 or +-4) in every block."""
    rng = np.random.default_rng(seed)
    B = 32 if fmt == "mxfp4" else 16
    nb = cols // B
    codes = rng.integers(0, 16, size=(rows, cols))
    codes[codes == 8] = 0
    for r in range(rows):
        for b in range(nb):
            codes[r, b * B + rng.integers(0, B)] = rng.choice([7, 15])
    x = np.zeros((rows, cols), np.float64)
    if fmt == "mxfp4":
        ex = rng.integers(-20, 20, size=(rows, nb))
        for r in range(rows):
            for j in range(cols):
                x[r, j] = bf.E2M1[codes[r, j]] * 2.0 ** ex[r, j // B]
    else:
        ts = 2.0 ** -9
        sb = rng.integers(0x20, 0x7F, size=(rows, nb))
        sb[0, 0] = 0x7E
        for r in range(rows):
            for b in range(nb):
                den = bf.e4m3_from_bits(int(sb[r, b])) * ts
                if fmt == "nvfp4_razer" and rng.random() < 0.7:
                    sign = rng.choice([1.0, -1.0])
                    j = b * B + (int(np.argmax(np.abs([bf.E2M1[c] for c in codes[r, b * B:(b + 1) * B]]))) + 1) % B
                    codes[r, j] = 8
                    x[r, j] = 5.0 * sign * den
                for j in range(b * B, (b + 1) * B):
                    if codes[r, j] != 8 or fmt != "nvfp4_razer":
                        x[r, j] = bf.E2M1[codes[r, j]] * den
    x32 = x.astype(np.float32)
    assert np.array_equal(x32.astype(np.float64), x)
    xb = x32.astype(ml_dtypes.bfloat16)
    assert np.array_equal(xb.astype(np.float64), x)   # exactly representable in bf16
    return xb.view(np.uint16)


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "mxfp4"])
def test_idempotent_on_representable_inputs(orc, fmt):
    xb = _representable(fmt)
    codes, scales, ts, sse = orc.quantize(xb, fmt)
    assert sse == 0.0
    y32, y16 = orc.dequantize(codes, scales, ts, fmt)
    assert np.array_equal(y16, xb)
    codes2, scales2, ts2, sse2 = orc.quantize(y16, fmt)
    assert np.array_equal(codes, codes2) and np.array_equal(scales, scales2) and ts == ts2
    if fmt == "nvfp4_razer":
        nib = bf.unpack_codes(codes, xb.shape[1])
        assert (nib == 8).any()      # the +-5 entries were used


# ---------------------------------------------------------------- RaZeR invariants and worked case

def test_razer_special_values_are_the_papers_pair(orc):
    pair = {int(r[0]): float(r[1]) for r in bf.read_golden("razer_special_values.txt")}
    ts = 1.0
    for sel, val in pair.items():
        codes = np.array([[0x08] + [0] * 7], np.uint8)        # element 0 = code 0b1000
        scales = np.array([[0x38 | (sel << 7)]], np.uint8)    # E4M3 1.0, selector bit
        y32, _ = orc.dequantize(codes, scales, ts, "nvfp4_razer")
        assert y32[0, 0] == val and val % 0.5 == 0


def test_razer_worked_block(orc):
    # one block [6d, 5d, 0, ...] with d = 448 * 2^-9: the 5d element is exactly the
    # special value +5, so RaZeR is lossless where NVFP4 must round 5 -> 4.
    d = 448 * 2.0 ** -9
    x = np.zeros((1, 16), np.float32); x[0, 0] = 6 * d; x[0, 1] = 5 * d
    xb = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    c_nv, s_nv, ts, sse_nv = orc.quantize(xb, "nvfp4")
    c_rz, s_rz, ts2, sse_rz = orc.quantize(xb, "nvfp4_razer")
    assert ts == ts2 == np.float32(2.0 ** -9)
    assert s_nv[0, 0] == 0x7E and s_rz[0, 0] == 0x7E     # +5 selected: bit 7 clear
    assert bf.unpack_codes(c_nv, 16)[0, 1] == 6          # 5 -> 4 (tie to even)
    assert bf.unpack_codes(c_rz, 16)[0, 1] == 8
    assert sse_rz == 0.0 and sse_nv == float((d) ** 2)
    # the negated block picks -5 through the scale's sign bit
    c_neg, s_neg, _, sse_neg = orc.quantize((-x).astype(ml_dtypes.bfloat16).view(np.uint16), "nvfp4_razer")
    assert s_neg[0, 0] == 0xFE and bf.unpack_codes(c_neg, 16)[0, 1] == 8 and sse_neg == 0.0


def test_razer_invariants_on_random_blocks(orc):
    from activation_quantization_block_b200 import synthetic
    xb = synthetic.bf16_bits(synthetic.llm_weight(64, 256, seed=20))
    c_nv, s_nv, ts, _ = orc.quantize(xb, "nvfp4", nthreads=2)
    c_rz, s_rz, ts2, _ = orc.quantize(xb, "nvfp4_razer", nthreads=2)
    assert ts == ts2
    assert np.array_equal(s_rz & 0x7F, s_nv)
    n_nv, n_rz = bf.unpack_codes(c_nv, 256), bf.unpack_codes(c_rz, 256)
    differ = n_nv != n_rz
    assert np.all(n_rz[differ] == 8)
    assert differ.any() and (s_rz & 0x80).any()
    # per-block squared error never grows
    y_nv, _ = orc.dequantize(c_nv, s_nv, ts, "nvfp4")
    y_rz, _ = orc.dequantize(c_rz, s_rz, ts, "nvfp4_razer")
    x = bf.bits_to_f32(xb).astype(np.float64)
    e_nv = ((x - y_nv) ** 2).reshape(64, 16, 16).sum(-1)
    e_rz = ((x - y_rz) ** 2).reshape(64, 16, 16).sum(-1)
    assert np.all(e_rz <= e_nv * (1 + 1e-12))
    assert e_rz.sum() < e_nv.sum()


def test_scale_rule_versus_best_scale_record(orc):
    """Record, not an equality: the absmax rule is never better than the best
    E4M3 scale found by enumerating all 126 nonzero scale bytes."""
    from activation_quantization_block_b200 import synthetic
    xb = synthetic.bf16_bits(synthetic.llm_weight(2, 32, seed=21))
    x = bf.bits_to_f32(xb)
    codes, scales, ts, _ = orc.quantize(xb, "nvfp4")
    y, _ = orc.dequantize(codes, scales, ts, "nvfp4")
    for b in range(4):
        r, c0 = divmod(b, 2)
        blk = x[r, c0 * 16:(c0 + 1) * 16].astype(np.float64)
        rule = float(((blk - y[r, c0 * 16:(c0 + 1) * 16]) ** 2).sum())
        best = min(
            float(((blk - np.array([bf.E2M1[bf.e2m1_nearest(float(v / (bf.e4m3_from_bits(sb) * ts)))]
                                      for v in blk]) * bf.e4m3_from_bits(sb) * ts) ** 2).sum())
            for sb in range(1, 0x7F))
        # the enumeration reconstructs in double, the rule in binary32: 1e-5 slack
        assert rule >= best * (1 - 1e-5)


# ---------------------------------------------------------------- statistics sanity (direction only)

def test_rotation_spreads_mxfp4_code_occupancy(orc):
    from activation_quantization_block_b200 import synthetic
    xb = synthetic.bf16_bits(synthetic.activation_t3(64, 512, seed=1))
    c0, _, _, sse0 = orc.quantize(xb, "mxfp4", False)
    c1, _, _, sse1 = orc.quantize(xb, "mxfp4", True)
    z0 = (bf.unpack_codes(c0, 512) & 7 == 0).mean()
    z1 = (bf.unpack_codes(c1, 512) & 7 == 0).mean()
    assert z1 < z0          # rotation leaves fewer elements quantized to zero
    assert sse1 < sse0


# ---------------------------------------------------------------- RaZeR weight mode (E3M3 scale, four specials)

def test_e3m3_decode(orc):
    """64 values: the normal ones are exactly the E4M3 values (ml_dtypes) whose
    exponent field is 4 higher (same 3-bit mantissa, bias 3 instead of 7), the
    subnormal ones the multiples of 2^-5 below the smallest normal 0.25."""
    vals = [orc.e3m3_value(b) for b in range(64)]
    assert vals == [bf.e3m3_from_bits(b) for b in range(64)]
    e4 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for b in range(64):
        e, m = b >> 3, b & 7
        if e:
            assert vals[b] == e4[((e + 4) << 3) | m]
        else:
            assert vals[b] == m * 2.0 ** -5
    assert vals[0x3F] == 30.0 and vals[8] == 0.25 and vals[1] == 2.0 ** -5
    assert all(a < b for a, b in zip(vals, vals[1:]))


def test_e3m3_encode_equals_exhaustive_argmin(orc):
    vals = sorted(set(bf.E3M3))
    probes = [0.0, 1e-9, 40.0, 30.0, 31.0, 1e30]
    for a, b in zip(vals, vals[1:]):
        mid = np.float32((a + b) / 2)
        probes += [a, b, float(mid), float(np.nextafter(mid, np.float32(0))), float(np.nextafter(mid, np.float32(99)))]
    for t in probes:
        assert orc.e3m3_encode(np.float32(t)) == bf.e3m3_nearest(min(float(np.float32(t)), 30.0)), t


def test_scale_widths_follow_the_paper(orc):
    """E3M3 codes fit the 6 bits the paper gives the weight scale, and the weight mode's
    selector lives exactly in the 8 - 6 = 2 bits that frees (tests/golden/scale_bits.txt)."""
    bits = {r[0]: int(r[1]) for r in bf.read_golden("scale_bits.txt")}
    assert bits == {"e4m3": 8, "e3m3": 6}
    free = bits["e4m3"] - bits["e3m3"]
    codes = [orc.e3m3_encode(np.float32(t)) for t in np.geomspace(1e-6, 1e6, 400)]
    assert max(codes) == (1 << bits["e3m3"]) - 1 and min(codes) >= 0
    assert all(orc.e4m3_encode(np.float32(t)) < (1 << (bits["e4m3"] - 1)) for t in np.geomspace(1e-6, 1e6, 400))
    rng = np.random.default_rng(31)
    x = orc.f32_to_bf16((rng.standard_normal((64, 256)) * 0.02).astype(np.float32))
    _, scales, _, _ = orc.quantize(x, "nvfp4_razer_w", want_sse=False)
    sel = scales >> bits["e3m3"]
    assert sel.max() < (1 << free) and len(np.unique(sel)) == 1 << free


def test_mxfp4_block_length_follows_the_paper(orc):
    """One shared exponent per 32 elements (tests/golden/block_sizes.txt): a row of two blocks
    whose magnitudes differ by 2^10 gets two scale bytes 10 apart, and every element of a block
    decodes with its own block's exponent."""
    B = {r[0]: int(r[1]) for r in bf.read_golden("block_sizes.txt")}["mxfp4"]
    assert orc.block_size("mxfp4") == B == 32
    v = np.concatenate([np.full(B, 1.0), np.full(B, 1024.0)]).astype(np.float32)[None, :]
    x = orc.f32_to_bf16(v)
    codes, scales, _, sse = orc.quantize(x, "mxfp4", False)
    assert scales.shape == (1, 2) and int(scales[0, 1]) - int(scales[0, 0]) == 10 and sse == 0.0
    _, y16 = orc.dequantize(codes, scales, 0.0, "mxfp4", False)
    assert np.array_equal(y16, x)


def test_weight_mode_tensor_scale_maps_amax_to_6x30(orc):
    for k in range(-20, 20):
        assert orc.tensor_scale_from_amax(180.0 * 2.0 ** k, "nvfp4_razer_w") == np.float32(2.0 ** k)
    assert orc.tensor_scale_from_amax(1.0, "nvfp4_razer_w") == np.float32(1.0) / np.float32(180.0)


def test_weight_mode_worked_blocks(orc):
    """[6d, 2.5d, 0...] is lossless with the second pair (selector 2, or 3 for the
    negated block); [6d, 5d, 0...] with the first (selector 0 / 1)."""
    d = 2.0 ** -4        # with A = 6d, s_t = A / 180, so the block scale is 30 (E3M3 0x3F)
    for special, sel in ((orc.razer_w_pair(), 2), (5.0, 0)):
        x = np.zeros((1, 16), np.float32); x[0, 0] = 6 * d; x[0, 3] = special * d
        for sign, s_sel in ((1.0, sel), (-1.0, sel + 1)):
            xb = (sign * x).astype(ml_dtypes.bfloat16).view(np.uint16)
            codes, scales, ts, sse = orc.quantize(xb, "nvfp4_razer_w")
            assert ts == np.float32(6 * d / 180.0)
            assert scales[0, 0] == (s_sel << 6) | 0x3F
            assert bf.unpack_codes(codes, 16)[0, 3] == 8 and sse == 0.0
            y32, _ = orc.dequantize(codes, scales, ts, "nvfp4_razer_w")
            assert np.array_equal(y32, (sign * x).astype(np.float32))


def test_weight_mode_invariants_on_random_blocks(orc):
    """Against NVFP4 with the same (E3M3-rounded) block scales, the weight mode
    only moves elements to code 0b1000 and never raises a block's error."""
    from activation_quantization_block_b200 import synthetic
    xb = synthetic.bf16_bits(synthetic.llm_weight(64, 256, seed=22))
    x = bf.bits_to_f32(xb).astype(np.float64)
    c_w, s_w, ts, _ = orc.quantize(xb, "nvfp4_razer_w", nthreads=2)
    y_w, _ = orc.dequantize(c_w, s_w, ts, "nvfp4_razer_w")
    n_w = bf.unpack_codes(c_w, 256)
    sels = (s_w >> 6) & 3
    assert {0, 1, 2, 3} <= set(np.unique(sels).tolist())
    # the same scales with every special code read as its regular E2M1 neighbour:
    # plain rounding of the scaled values, block by block
    for r in range(8):
        for b in range(16):
            sb = int(s_w[r, b]) & 0x3F
            den = np.float32(np.float32(bf.E3M3[sb]) * ts)
            rr = np.float32(np.float32(1) / den)
            blk = x[r, 16 * b:16 * b + 16].astype(np.float32)
            v = [np.float32(val * rr) for val in blk]
            q = [bf.e2m1_nearest(float(vi)) for vi in v]
            got = n_w[r, 16 * b:16 * b + 16]
            assert all(g == qi or g == 8 for g, qi in zip(got, q))
            plain = float(((blk.astype(np.float64) - np.array([bf.E2M1[qi] for qi in q]) * float(den)) ** 2).sum())
            mine = float(((blk.astype(np.float64) - y_w[r, 16 * b:16 * b + 16]) ** 2).sum())
            assert mine <= plain * (1 + 1e-6)


def test_weight_mode_second_pair_wins_a_reduced_search(orc):
    """The second pair is the minimum of the offline search; a smaller sample of
    the same synthetic weights gives the same winner."""
    from oracle import razer_weight_pair
    from activation_quantization_block_b200 import synthetic
    mats = [synthetic.bf16_bits(synthetic.llm_weight(256, 2048, seed=300 + k, device="cpu")) for k in range(2)]
    keep = orc.razer_w_pair()
    try:
        table = {s2: razer_weight_pair.total_sse(mats, s2) for s2 in razer_weight_pair.CANDIDATES}
    finally:
        orc.set_razer_w_pair(keep)
    assert min(table, key=table.get) == keep == 2.5
    assert all(keep % 0.5 == 0 for keep in table)


# ---------------------------------------------------------------- tensor-core operand form and W4A4 product

@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "nvfp4_razer_w"])
def test_mma_planes_sum_to_the_reconstruction(orc, fmt):
    """Decoded with the brute-force E2M1 table, the planes' values add up exactly to
    the element's value (special values included), and with the atom's scale and
    the tensor scale, rounded as a reconstruction is, give the brute-force
    dequantizer's value."""
    from activation_quantization_block_b200 import synthetic
    rows, cols = 40, 96
    xb = synthetic.bf16_bits(synthetic.llm_weight(rows, cols, seed=41))
    codes, scales, ts, _ = orc.quantize(xb, fmt, nthreads=2)
    planes, sf = orc.mma_pack(codes, scales, fmt)
    np_ = orc.mma_planes(fmt)
    assert np_ == (1 if fmt == "nvfp4" else 2) and planes.shape == (rows, np_ * cols // 2)
    ref = bf.dequantize_bruteforce(codes, scales, float(ts), fmt, False)
    n_special = 0
    for r in range(rows):
        q0 = bf.unpack_codes(planes[r:r + 1, :cols // 2], cols)[0]
        q1 = bf.unpack_codes(planes[r:r + 1, cols // 2:], cols)[0] if np_ == 2 else np.zeros(cols, int)
        for j in range(cols):
            byte = int(sf[orc.mma_sf_offset(r, j // 16, cols)])
            assert byte < 0x7F                                   # an E4M3 magnitude, bit 7 clear
            q = Fraction(bf.E2M1[q0[j]]) + Fraction(bf.E2M1[q1[j]])
            den = np.float32(np.float32(bf.e4m3_from_bits(byte)) * np.float32(ts))
            assert np.float32(np.float32(float(q)) * den) == ref[r][j]
            orig = bf.unpack_codes(codes[r:r + 1], cols)[0][j]
            if np_ == 2 and orig == 8:
                sb = int(scales[r, j // 16])
                s = ((-5.0 if sb & 0x80 else 5.0) if fmt == "nvfp4_razer"
                     else (5.0, -5.0, 2.5, -2.5)[(sb >> 6) & 3])
                assert q == Fraction(s)
                n_special += 1
            else:
                assert q == Fraction(bf.E2M1[orig]) and q1[j] == 0
    if fmt != "nvfp4":
        assert n_special > 0


def test_mma_plane_split_of_each_special_value(orc):
    """The split of every special value: base = the largest E2M1 magnitude below it."""
    for fmt, sbyte, s in (("nvfp4_razer", 0x38, 5.0), ("nvfp4_razer", 0xB8, -5.0),
                          ("nvfp4_razer_w", 0x00 | 0x20, 5.0), ("nvfp4_razer_w", 0x40 | 0x20, -5.0),
                          ("nvfp4_razer_w", 0x80 | 0x20, 2.5), ("nvfp4_razer_w", 0xC0 | 0x20, -2.5)):
        codes = np.full((1, 8), 0x08, np.uint8)                 # element 0 special, element 1 zero
        scales = np.full((1, 1), sbyte, np.uint8)
        planes, _ = orc.mma_pack(codes, scales, fmt)
        b = math.copysign(4.0 if abs(s) == 5.0 else 2.0, s)
        assert bf.E2M1[planes[0, 0] & 15] == b and bf.E2M1[planes[0, 8] & 15] == s - b
        assert bf.E2M1[planes[0, 0] >> 4] == 0 and bf.E2M1[planes[0, 8] >> 4] == 0


def test_mma_scale_bytes_are_exact_e4m3(orc):
    """Every E3M3 value is an E4M3 value; activation-mode scales lose only bit 7."""
    for c in range(64):
        b = orc.mma_scale_byte("nvfp4_razer_w", c | 0xC0)
        assert float(np.array([b], np.uint8).view(ml_dtypes.float8_e4m3fn)[0]) == bf.E3M3[c]
    for b in range(0x7F):
        assert orc.mma_scale_byte("nvfp4_razer", b | 0x80) == b == orc.mma_scale_byte("nvfp4", b)


def test_mma_scale_atoms_match_a_reshape(orc):
    """The atom order restated as numpy axes: [row block][block group][row % 32]
    [(row % 128) / 32][block % 4]; padding is zero."""
    rows, cols = 300, 16 * 37
    nb = cols // 16
    rng = np.random.default_rng(5)
    scales = rng.integers(1, 0x7F, size=(rows, nb), dtype=np.uint8)
    codes = np.zeros((rows, cols // 2), np.uint8)
    _, sf = orc.mma_pack(codes, scales, "nvfp4")
    rb, kb4 = -(-rows // 128), -(-nb // 4)
    pad = np.zeros((rb * 128, kb4 * 4), np.uint8)
    pad[:rows, :nb] = scales
    want = pad.reshape(rb, 4, 32, kb4, 4).transpose(0, 3, 2, 1, 4).ravel()
    assert sf.size == orc.mma_sf_bytes(rows, cols) == rb * kb4 * 512
    assert np.array_equal(sf, want)


def test_gemm_oracle_against_numpy_and_exact_integers(orc):
    rng = np.random.default_rng(6)
    a = rng.standard_normal((37, 200)).astype(np.float32)
    w = rng.standard_normal((23, 200)).astype(np.float32)
    y, yabs = orc.gemm(a, w, nthreads=3)
    ref = a.astype(np.float64) @ w.astype(np.float64).T
    assert np.all(np.abs(y - ref) <= 1e-12 * (np.abs(a).astype(np.float64) @ np.abs(w).astype(np.float64).T))
    assert np.allclose(yabs, np.abs(a).astype(np.float64) @ np.abs(w).astype(np.float64).T, rtol=1e-12)
    ai = rng.integers(-6, 7, size=(5, 64)).astype(np.float32)
    wi = rng.integers(-6, 7, size=(7, 64)).astype(np.float32)
    yi, _ = orc.gemm(ai, wi)
    assert np.array_equal(yi, ai.astype(np.int64) @ wi.astype(np.int64).T)


def test_gemm_of_one_hot_rows_returns_weight_columns(orc):
    """A one-hot activation row picks one column of the weight reconstruction."""
    from activation_quantization_block_b200 import synthetic
    xb = synthetic.bf16_bits(synthetic.llm_weight(24, 128, seed=43))
    codes, scales, ts, _ = orc.quantize(xb, "nvfp4_razer_w", nthreads=2)
    w, _ = orc.dequantize(codes, scales, ts, "nvfp4_razer_w")
    a = np.zeros((128, 128), np.float32)
    a[np.arange(128), np.arange(128)] = 1.0
    y, _ = orc.gemm(a, w)
    assert np.array_equal(y, w.T.astype(np.float64))


# ---------------------------------------------------------------- MXFP4 exponent without clipping

def _mx_ceil_points():
    pts = []
    for k in list(range(-149, -120)) + list(range(-20, 21)) + list(range(120, 128)):
        for m in (1.0, 1.25, 1.5, 1.75, 1.9990234375):
            v = np.float32(m * 2.0 ** k)
            if v > 0 and np.isfinite(v):
                pts += [v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(np.inf))]
    for e in range(-126, 126):          # 6 * 2^e and its neighbours
        v = np.float32(6.0 * 2.0 ** e)
        pts += [v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(np.inf))]
    return [p for p in pts if p > 0 and np.isfinite(p)]


def test_mx_exponent_ceil_equals_exhaustive_minimum(orc):
    """e = min{e in [-127, 125] : a <= 6 * 2^e} (125 if none), by enumeration with exact rationals."""
    for a in _mx_ceil_points():
        fa = Fraction(float(a))
        want = min((k for k in range(-127, 126) if fa <= 6 * Fraction(2) ** k), default=125)
        assert orc.mx_exponent_ceil(float(a)) == want, a


def test_mx_exponent_ceil_closed_forms(orc):
    assert orc.mx_exponent_ceil(6.0) == 0 and orc.mx_exponent_ceil(3.0) == -1 and orc.mx_exponent_ceil(4.0) == 0
    assert orc.mx_exponent_ceil(float(np.nextafter(np.float32(6), np.float32(7)))) == 1
    assert orc.mx_exponent_ceil(3.3895313892515355e38) == 125       # the clamp: 4 * 2^126 would overflow
    # differs from the floor rule exactly when the block maximum's mantissa exceeds 1.5
    for k in range(-30, 30):
        for m, up in ((1.0, 0), (1.5, 0), (1.5000001, 1), (1.75, 1), (1.99, 1)):
            a = float(np.float32(m * 2.0 ** k))
            assert orc.mx_exponent_ceil(a) - orc.mx_exponent(a) == up


def test_mxfp4_ceil_never_saturates_and_decodes_as_mxfp4(orc):
    from activation_quantization_block_b200 import synthetic
    xb = synthetic.bf16_bits(synthetic.activation_t3(64, 512, seed=44))
    x = bf.bits_to_f32(xb).astype(np.float64)
    c, s, _, sse_c = orc.quantize(xb, "mxfp4_ceil", nthreads=2)
    _, _, _, sse_f = orc.quantize(xb, "mxfp4", nthreads=2)
    y_c, _ = orc.dequantize(c, s, 0.0, "mxfp4_ceil")
    y_m, _ = orc.dequantize(c, s, 0.0, "mxfp4")
    assert np.array_equal(y_c, y_m)                     # the same stored format
    blocks = np.abs(x).reshape(64, 16, 32).max(-1)
    scale = 2.0 ** (s.astype(np.float64) - 127)
    assert np.all(blocks <= 6 * scale)                  # the block maximum fits: no element saturates
    assert sse_c != sse_f


# ---------------------------------------------------------------- sparse outlier separation

def _rn_fraction(v: Fraction, quantum: Fraction) -> Fraction:
    q = v / quantum
    r = math.floor(q)
    frac = q - r
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and r % 2):
        r += 1
    return r * quantum


def test_f64_to_bf16_is_exact_nearest_even(orc):
    rng = np.random.default_rng(50)
    vals = list(rng.standard_normal(300) * 10.0 ** rng.integers(-40, 38, 300))
    for e in (-130, -20, 0, 5):                        # ties and their neighbours
        for m in (1 + 1 / 256, 1 + 3 / 256, 1.5 + 1 / 256):
            t = m * 2.0 ** e
            vals += [t, np.nextafter(t, 0), np.nextafter(t, 10)]
    for v in vals:
        fv = Fraction(float(v))
        e = math.floor(math.log2(abs(float(v))))
        if Fraction(2) ** (e + 1) <= abs(fv):
            e += 1
        if Fraction(2) ** e > abs(fv):
            e -= 1
        want = _rn_fraction(abs(fv), Fraction(2) ** (-133 if e < -126 else e - 7))
        got = orc.f64_to_bf16(float(v))
        gv = float(np.array([got], np.uint16).view(ml_dtypes.bfloat16)[0])
        assert Fraction(abs(gv)) == want and (gv < 0) == (v < 0), v


def test_f32_to_f16_saturating_matches_numpy(orc):
    rng = np.random.default_rng(51)
    vals = np.concatenate([rng.standard_normal(2000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 5, 2000),
                           np.float32([65504, 65519.99, 65520, 7e4, -1e6, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                                       6.1e-5, -0.0, 0.0])])
    for v in vals:
        got = orc.f32_to_f16_sat(float(v))
        ref = np.float16(v) if abs(v) < 65520 else np.float16(np.sign(v) * 65504)
        assert got == int(np.array([ref]).view(np.uint16)[0]), v
        assert orc.f16_value(got) == float(ref)


def test_outlier_rule_follows_the_paper(orc):
    """The defaults and storage of the separation are the page's (tests/golden/outlier_rule.txt):
    k = 4, at most 2 % of a row, fp16 values, the row mean in the bulk."""
    rule = {r[0]: r[1] for r in bf.read_golden("outlier_rule.txt")}
    k, frac = float(rule["k"]), float(rule["max_frac"])
    assert rule["value_format"] == "fp16" and rule["bulk_fill"] == "group_mean"
    for cols in (8, 49, 50, 100, 1024, 4096, 14336):
        assert orc.outlier_capacity(cols) == orc.outlier_capacity(cols, frac) == int(np.floor(frac * cols + 1e-9))
    # one row: 250 zeros and a 0.5 spike; mean 0.5/251 and sigma about 0.0315, so the spike
    # is past 4 sigma and is the only outlier; its value comes back as the fp16 bits of 0.5
    row = np.zeros((1, 256), np.float32)
    row[0, 100] = 0.5
    x = orc.f32_to_bf16(row)
    bulk, oc, ov, cnt, mu, thr = orc.separate_outliers(x)
    mean = 0.5 / 256
    sigma = np.sqrt(((row[0].astype(np.float64) - mean) ** 2).mean())
    assert cnt[0] == 1 and oc[0, 0] == 100 and abs(mu[0] - mean) < 1e-15
    assert abs(thr[0] - k * sigma) <= 1e-12 * k * sigma
    assert ov[0, 0] == np.float16(0.5).view(np.uint16)
    assert bulk[0, 100] == orc.f64_to_bf16(mean) and (np.delete(bulk[0], 100) == 0).all()


def test_outliers_closed_form_rows(orc):
    """Rows of n - m zeros and m spikes of height h: mu = m h / n, sigma = h sqrt(m (n - m)) / n,
    and the spikes are outliers exactly when (n - m) / sqrt(m (n - m)) > k."""
    n = 256
    rows = []
    for m in (1, 3, 8, 16, 40):
        row = np.zeros(n, np.float32)
        row[np.arange(m) * 5 + 2] = 0.5
        rows.append(row)
    x = np.array(rows).astype(ml_dtypes.bfloat16).view(np.uint16)
    bulk, oc, ov, cnt, mu, thr = orc.separate_outliers(x, k=4.0, max_frac=0.02)
    cap = orc.outlier_capacity(n, 0.02)
    assert cap == 5
    for i, m in enumerate((1, 3, 8, 16, 40)):
        assert mu[i] == m * 0.5 / n
        is_out = (n - m) / math.sqrt(m * (n - m)) > 4.0
        expect = min(m, cap) if is_out else 0
        assert cnt[i] == expect, (m, cnt[i])
        cols = oc[i, :cnt[i]]
        assert list(cols) == list((np.arange(m) * 5 + 2)[:expect])    # ties: the lowest columns
        assert all(orc.f16_value(v) == 0.5 for v in ov[i, :cnt[i]])
        b = bulk[i].view(ml_dtypes.bfloat16).astype(np.float64)
        assert np.all(b[cols] == float(np.array([orc.f64_to_bf16(mu[i])], np.uint16).view(ml_dtypes.bfloat16)[0]))


def test_outliers_against_numpy_statistics(orc):
    """Random LLM-weight rows (with x20 outliers) and rows where the 2 % cap binds:
    the outlier set equals one built from numpy's mean / std and a sort."""
    from activation_quantization_block_b200 import synthetic
    w = synthetic.llm_weight(48, 1024, seed=52).float().numpy()
    rng = np.random.default_rng(53)
    w[40:] *= np.where(rng.random((8, 1024)) < 0.1, 20.0, 1.0)      # 10 % spikes: the cap binds
    x = w.astype(ml_dtypes.bfloat16).view(np.uint16)
    xf = x.view(ml_dtypes.bfloat16).astype(np.float64)
    bulk, oc, ov, cnt, mu, thr = orc.separate_outliers(x, k=4.0, max_frac=0.02)
    cap = orc.outlier_capacity(1024, 0.02)
    bound = 0
    for r in range(48):
        m, s = np.mean(xf[r]), np.std(xf[r])
        assert abs(m - mu[r]) <= 1e-12 * np.abs(xf[r]).max() and abs(4 * s - thr[r]) <= 1e-12 * thr[r]
        d = np.abs(xf[r] - m)
        cand = np.nonzero(d > 4 * s)[0]
        if len(cand) > cap:
            bound += 1
            order = sorted(cand, key=lambda j: (-d[j], j))
            cand = np.sort(order[:cap])
        assert list(oc[r, :cnt[r]]) == list(cand)
        assert np.array_equal(ov[r, :cnt[r]], xf[r, cand].astype(np.float16).view(np.uint16))
        keep = np.ones(1024, bool)
        keep[cand] = False
        assert np.array_equal(bulk[r, keep], x[r, keep])
    assert bound >= 4                                              # rows where the cap binds


# ---------------------------------------------------------------- negation symmetry and constants

def _special_gains(blk_x, sb, ts, fmt):
    """Exact gains (Fractions) of each special value for one 16-block, from the
    block's scaled values as the encoder forms them."""
    wmode = fmt == "nvfp4_razer_w"
    sval = bf.E3M3[sb & 0x3F] if wmode else bf.e4m3_from_bits(sb & 0x7F)
    den = np.float32(np.float32(sval) * np.float32(ts))
    r = np.float32(np.float32(1) / den)
    v = [np.float32(np.float32(x) * r) for x in blk_x]
    specials = (5.0, -5.0, 2.5, -2.5) if wmode else (5.0, -5.0)
    gains = []
    for sp in specials:
        g = Fraction(0)
        for vi in v:
            fv = Fraction(float(vi))
            q = Fraction(bf.E2M1[bf.e2m1_nearest(float(vi))])
            if abs(fv - sp) < abs(fv - q):
                g += (fv - q) ** 2 - (fv - sp) ** 2
        gains.append(g)
    return gains


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp4_razer", "nvfp4_razer_w", "mxfp4", "mxfp4_ceil"])
def test_negating_the_input_negates_the_encoding(orc, fmt):
    """quantize(-x): the same block scale magnitudes and error; nonzero codes flip
    their sign bit; RaZeR selectors flip their sign (activation bit 7; weight bit 6,
    so +5 <-> -5 and +2.5 <-> -2.5) -- except in blocks where the best gains of a
    special value and its negation tie, which both encodings resolve to the
    positive one (the lower selector): those are checked to be exact ties."""
    from activation_quantization_block_b200 import synthetic
    x = synthetic.llm_weight(32, 256, seed=45)
    xb = synthetic.bf16_bits(x)
    nb = synthetic.bf16_bits(-x)
    xf = bf.bits_to_f32(xb)
    c, s, ts, sse = orc.quantize(xb, fmt, nthreads=2)
    cn, sn, tsn, ssen = orc.quantize(nb, fmt, nthreads=2)
    assert ts == tsn
    B = 32 if fmt.startswith("mxfp4") else 16
    q = bf.unpack_codes(c, 256).reshape(32, 256 // B, B)
    qn = bf.unpack_codes(cn, 256).reshape(32, 256 // B, B)
    mag_mask = {"nvfp4": 0xFF, "nvfp4_razer": 0x7F, "nvfp4_razer_w": 0x3F}.get(fmt, 0xFF)
    assert np.array_equal(s & mag_mask, sn & mag_mask)
    ties = 0
    for r in range(32):
        for b in range(256 // B):
            a, an = q[r, b], qn[r, b]
            sel_flip = {"nvfp4_razer": 0x80, "nvfp4_razer_w": 0x40}.get(fmt, 0)
            special = a == 8
            mirrored = (np.array_equal(an[(a & 7) != 0], a[(a & 7) != 0] ^ 8) and
                        np.array_equal(an[(a & 7) == 0], a[(a & 7) == 0]))
            if fmt in ("nvfp4_razer", "nvfp4_razer_w") and special.any():
                mirrored = mirrored and int(sn[r, b]) == int(s[r, b]) ^ sel_flip
            elif fmt in ("nvfp4_razer", "nvfp4_razer_w"):
                mirrored = mirrored and int(sn[r, b]) == int(s[r, b])
            if not mirrored:
                assert fmt in ("nvfp4_razer", "nvfp4_razer_w"), (r, b)
                g = _special_gains(xf[r, 16 * b:16 * b + 16], int(s[r, b]), ts, fmt)
                best = max(g)
                pos_neg = [(g[i], g[i + 1]) for i in range(0, len(g), 2)]
                assert any(gp == gn == best for gp, gn in pos_neg), (r, b, g)
                ties += 1
    if fmt in ("nvfp4", "mxfp4", "mxfp4_ceil"):
        assert sse == ssen and ties == 0


def test_the_kernels_second_pair_is_the_oracles():
    """The weight mode's second special-value pair is one constant on each side (they
    share no code): the CUDA source's value equals the oracle's default."""
    import os
    import re
    import oracle
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = open(os.path.join(root, "activation_quantization_block_b200", "csrc", "fp4q_common.cuh")).read()
    m = re.search(r"constexpr float kRazerWPair = ([0-9.]+)f;", src)
    assert m and float(m.group(1)) == oracle.razer_w_pair() == 2.5
