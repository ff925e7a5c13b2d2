"""Independent brute-force restatements used to pin the oracle (tests only).

Each helper reaches its answer by a different route from the oracle's C code:
exhaustive enumeration of every code or scale byte, exact rational arithmetic
(``fractions.Fraction``), or a library (``ml_dtypes``, ``scipy``).  Nothing
here imports the oracle or the CUDA library.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> list[list[str]]:
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---- element and scale formats from their bit fields --------------------------

def e2m1_from_bits(code: int) -> float:
    """E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if s else mag


def e4m3_from_bits(byte: int) -> float:
    """E4M3 (fn variant): bias 7, exponent 0 subnormal, 0x7F/0xFF NaN, no infinities."""
    s, e, m = (byte >> 7) & 1, (byte >> 3) & 15, byte & 7
    if e == 15 and m == 7:
        return float("nan")
    mag = m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


def e3m3_from_bits(byte6: int) -> float:
    """E3M3 (6 bits, unsigned): bias 3, exponent 0 subnormal, no NaN."""
    e, m = (byte6 >> 3) & 7, byte6 & 7
    return m * 2.0 ** -5 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 3)


E2M1 = [e2m1_from_bits(c) for c in range(16)]
E4M3_POS = [e4m3_from_bits(b) for b in range(0x7F)]  # 0x00 .. 0x7E, increasing
E3M3 = [e3m3_from_bits(b) for b in range(64)]        # increasing


def e2m1_nearest(v: float) -> int:
    """Argmin over all 16 codes of |v - value|; ties go to the even magnitude
    index; a zero result is +0 (code 0)."""
    best = None
    for code in range(16):
        d = abs(Fraction(v) - Fraction(E2M1[code]))
        key = (d, (code & 7) & 1, code >> 3)  # distance, odd index, sign bit
        if best is None or key < best[0]:
            best = (key, code)
    code = best[1]
    return 0 if (code & 7) == 0 else code


def e4m3_nearest(t: float) -> int:
    """Argmin over the 127 non-negative finite E4M3 bytes; ties to the even byte."""
    best = None
    ft = Fraction(t)
    for b, val in enumerate(E4M3_POS):
        key = (abs(ft - Fraction(val)), b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return best[1]


def e3m3_nearest(t: float) -> int:
    """Argmin over the 64 E3M3 values; ties to the even byte."""
    best = None
    ft = Fraction(t)
    for b, val in enumerate(E3M3):
        key = (abs(ft - Fraction(val)), b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return best[1]


def razer_pick(v, q, specials):
    """Exact per-block special-value choice: for each candidate, elements strictly
    closer to it than to their regular value move to it; the candidate with the
    lowest total squared error wins (ties: the earlier candidate).  Returns
    (index, codes)."""
    best = None
    for idx, sv in enumerate(specials):
        tot = Fraction(0)
        ch = []
        for vi, qi in zip(v, q):
            er = (Fraction(float(vi)) - Fraction(E2M1[qi])) ** 2
            es = (Fraction(float(vi)) - Fraction(sv)) ** 2
            if es < er:
                tot += es
                ch.append(8)
            else:
                tot += er
                ch.append(qi)
        if best is None or tot < best[0]:
            best = (tot, idx, ch)
    return best[1], best[2]


def floor_log2(a: float) -> int:
    """Largest k with 2**k <= a, for a > 0, by exact comparison."""
    fa = Fraction(a)
    k = 0
    while Fraction(2) ** k > fa:
        k -= 1
    while Fraction(2) ** (k + 1) <= fa:
        k += 1
    return k


# ---- fp32 / bf16 -------------------------------------------------------------

def f32(x) -> np.float32:
    return np.float32(x)


def bits_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rn_f32(fr: Fraction) -> np.float32:
    """Round an exact rational to binary32, nearest even (via double; exact
    whenever the rational fits in 53 bits, which holds for every sum here)."""
    return np.float32(float(fr))


def rn_f32_exact(fr: Fraction) -> np.float32:
    """Round an exact rational to binary32, nearest even, subnormals included,
    by integer arithmetic on its significand (no intermediate rounding)."""
    if fr == 0:
        return np.float32(0.0)
    neg = fr < 0
    a = -fr if neg else fr
    e = a.numerator.bit_length() - a.denominator.bit_length()   # 2^e <= a < 2^(e+2)
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    qexp = max(e, -126) - 23                                       # the binary32 quantum at a
    scaled = a / Fraction(2) ** qexp
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    val = Fraction(n) * Fraction(2) ** qexp
    out = np.float32(np.inf) if val >= Fraction(2) ** 128 else np.float32(float(val))
    return -out if neg else out


def sylvester_hadamard(n: int = 32) -> np.ndarray:
    h = np.array([[1]], dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


# ---- full brute-force quantizer for tiny tensors --------------------------------

def unpack_codes(codes: np.ndarray, cols: int) -> np.ndarray:
    """[rows, cols/2] bytes -> [rows, cols] nibbles, element 2k in the low nibble."""
    out = np.zeros((codes.shape[0], cols), dtype=np.int64)
    out[:, 0::2] = codes & 0x0F
    out[:, 1::2] = codes >> 4
    return out


def quantize_bruteforce(xbits: np.ndarray, fmt: str, rotate: bool, pair2: float = 2.5):
    """Quantize by enumeration: every scale byte and every element code is the
    argmin of its own exhaustive search; rotation sums are exact rationals.
    ``pair2``: the second special-value pair of the weight mode."""
    x = bits_to_f32(xbits).astype(np.float32)
    rows, cols = x.shape
    y = x.copy()
    c = np.float32(1 / np.sqrt(np.float64(32)))
    if rotate:
        H = sylvester_hadamard(32)
        for r in range(rows):
            for g in range(0, cols, 32):
                seg = [Fraction(float(v)) for v in x[r, g:g + 32]]
                for i in range(32):
                    s = sum((H[i, j] * seg[j] for j in range(32)), Fraction(0))
                    y[r, g + i] = np.float32(rn_f32(s) * c)
    mx = fmt in ("mxfp4", "mxfp4_ceil")
    B = 32 if mx else 16
    codes = np.zeros((rows, cols), dtype=np.int64)
    scales = np.zeros((rows, cols // B), dtype=np.int64)
    ts = np.float32(0)
    wmode = fmt == "nvfp4_razer_w"
    if not mx:
        A = np.float32(np.max(np.abs(y))) if y.size else np.float32(0)
        ts = np.float32(A / np.float32(180 if wmode else 2688))
    for r in range(rows):
        for b in range(cols // B):
            blk = y[r, b * B:(b + 1) * B]
            a = np.float32(np.max(np.abs(blk)))
            if mx:
                if a == 0:
                    continue
                if fmt == "mxfp4_ceil":   # the smallest exponent whose 6 * 2^e holds the block maximum
                    e = min((k for k in range(-127, 126) if Fraction(float(a)) <= 6 * Fraction(2) ** k),
                            default=125)
                else:
                    e = max(-127, min(127, floor_log2(float(a)) - 2))
                scales[r, b] = e + 127
                v = [np.float32(val * np.float32(2.0 ** -e)) for val in blk]
            else:
                six = np.float32(np.float32(6) * ts)
                t = np.float32(a / six) if six > 0 else np.float32(0)
                sb = e3m3_nearest(float(t)) if wmode else e4m3_nearest(float(t))
                den = np.float32(np.float32(E3M3[sb] if wmode else E4M3_POS[sb]) * ts)
                scales[r, b] = sb
                if sb == 0 or den == 0:
                    continue
                with np.errstate(over="ignore"):
                    rr = np.float32(np.float32(1) / den)
                if np.isinf(rr):   # the reciprocal overflows: scale by exact division, rounded once
                    v = [rn_f32_exact(Fraction(float(val)) / Fraction(float(den))) for val in blk]
                else:
                    v = [np.float32(val * rr) for val in blk]
            q = [e2m1_nearest(float(vi)) for vi in v]
            if fmt == "nvfp4_razer":
                idx, q = razer_pick(v, q, (5.0, -5.0))
                scales[r, b] |= idx << 7
            elif wmode:
                idx, q = razer_pick(v, q, (5.0, -5.0, pair2, -pair2))
                scales[r, b] |= idx << 6
            codes[r, b * B:(b + 1) * B] = q
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, scales.astype(np.uint8), ts


def dequantize_bruteforce(codes: np.ndarray, scales: np.ndarray, ts: float, fmt: str,
                          rotate: bool, pair2: float = 2.5) -> np.ndarray:
    """fp32 reconstruction from the bit-field definitions (exact rationals for rotation)."""
    rows, cols = codes.shape[0], codes.shape[1] * 2
    nib = unpack_codes(codes, cols)
    mx = fmt in ("mxfp4", "mxfp4_ceil")
    B = 32 if mx else 16
    out = np.zeros((rows, cols), dtype=np.float32)
    for r in range(rows):
        for j in range(cols):
            sb = int(scales[r, j // B])
            code = int(nib[r, j])
            if mx:
                out[r, j] = np.float32(E2M1[code] * 2.0 ** (sb - 127))
            else:
                if fmt == "nvfp4_razer_w":
                    sval = e3m3_from_bits(sb & 0x3F)
                else:
                    sval = e4m3_from_bits(sb & 0x7F if fmt == "nvfp4_razer" else sb)
                den = np.float32(np.float32(sval) * np.float32(ts))
                if fmt == "nvfp4_razer" and code == 8:
                    qv = -5.0 if sb & 0x80 else 5.0
                elif fmt == "nvfp4_razer_w" and code == 8:
                    qv = (5.0, -5.0, pair2, -pair2)[(sb >> 6) & 3]
                else:
                    qv = E2M1[code]
                out[r, j] = np.float32(np.float32(qv) * den)
    if rotate:
        H = sylvester_hadamard(32)
        c = np.float32(1 / np.sqrt(np.float64(32)))
        res = out.copy()
        for r in range(rows):
            for g in range(0, cols, 32):
                seg = [Fraction(float(v)) for v in out[r, g:g + 32]]
                for i in range(32):
                    s = sum((H[i, j] * seg[j] for j in range(32)), Fraction(0))
                    res[r, g + i] = np.float32(rn_f32(s) * c)
        out = res
    return out


def sse_exact(xbits: np.ndarray, xhat: np.ndarray) -> Fraction:
    x = bits_to_f32(xbits)
    tot = Fraction(0)
    for a, b in zip(x.ravel(), xhat.ravel()):
        d = Fraction(float(a)) - Fraction(float(b))
        tot += d * d
    return tot
