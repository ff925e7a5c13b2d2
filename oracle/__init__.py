"""fp4q oracle: the plain CPU restatement of block-scaled 4-bit quantization.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg and reference arm of ``bench.py`` may import this package.  The CUDA library
and its Python binding never import, link or call it, and it imports nothing
from them.

The arithmetic lives in ``fp4q_oracle.c`` (scalar loops, IEEE binary32 /
binary64, no fast-math); this module is a numpy/ctypes wrapper around it.  The
header comment of the C file lists the page passages it follows and the
readings it takes where the cited papers are silent.  Functions whose result is not
pinned by an independent check are marked "parity unpinned" in their
docstring; at present every function is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

NVFP4, NVFP4_RAZER, MXFP4, NVFP4_RAZER_W, MXFP4_CEIL = 0, 1, 2, 3, 4
# "mxfp4_ceil": MXFP4 whose block exponent maps the block maximum onto 6 without clipping
# (the encoder's choice only: stored and decoded exactly as MXFP4)
FORMAT_NAMES = {"nvfp4": NVFP4, "nvfp4_razer": NVFP4_RAZER, "mxfp4": MXFP4, "nvfp4_razer_w": NVFP4_RAZER_W,
                "mxfp4_ceil": MXFP4_CEIL}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4q_oracle.c")
_LIB = os.path.join(_HERE, "libfp4q_oracle.so")
CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC", "-pthread"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library in place (gcc) and return its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        vp = ctypes.c_void_p
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]; L.orc_bf16_to_f32.restype = f32
        L.orc_f32_to_bf16.argtypes = [f32]; L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_e2m1_value.argtypes = [i32]; L.orc_e2m1_value.restype = f64
        L.orc_e2m1_encode.argtypes = [f32]; L.orc_e2m1_encode.restype = i32
        L.orc_e4m3_value.argtypes = [i32]; L.orc_e4m3_value.restype = f64
        L.orc_e4m3_encode.argtypes = [f32]; L.orc_e4m3_encode.restype = i32
        L.orc_e3m3_value.argtypes = [i32]; L.orc_e3m3_value.restype = f64
        L.orc_e3m3_encode.argtypes = [f32]; L.orc_e3m3_encode.restype = i32
        L.orc_set_razer_w_pair.argtypes = [f64]; L.orc_set_razer_w_pair.restype = None
        L.orc_razer_w_pair.argtypes = []; L.orc_razer_w_pair.restype = f64
        L.orc_tensor_scale_from_amax_w.argtypes = [f32]; L.orc_tensor_scale_from_amax_w.restype = f32
        L.orc_e8m0_value.argtypes = [i32]; L.orc_e8m0_value.restype = f64
        L.orc_mx_exponent.argtypes = [f32]; L.orc_mx_exponent.restype = i32
        L.orc_mx_exponent_ceil.argtypes = [f32]; L.orc_mx_exponent_ceil.restype = i32
        L.orc_hadamard_entry.argtypes = [i32, i32]; L.orc_hadamard_entry.restype = i32
        L.orc_wht_constant.argtypes = []; L.orc_wht_constant.restype = f32
        L.orc_wht32.argtypes = [vp, vp]; L.orc_wht32.restype = None
        L.orc_tensor_amax.argtypes = [vp, i64, i64, i64, i32, i32]; L.orc_tensor_amax.restype = f32
        L.orc_tensor_scale_from_amax.argtypes = [f32]; L.orc_tensor_scale_from_amax.restype = f32
        L.orc_quantize.argtypes = [vp, i64, i64, i64, i32, i32, i32, vp, vp, vp, vp, i32]
        L.orc_quantize.restype = i32
        L.orc_dequantize.argtypes = [vp, vp, f32, i64, i64, i32, i32, vp, vp, i64, i32]
        L.orc_dequantize.restype = i32
        L.orc_error.argtypes = [vp, i64, vp, vp, f32, i64, i64, i32, i32, vp, i32]
        L.orc_error.restype = i32
        L.orc_mma_planes.argtypes = [i32]; L.orc_mma_planes.restype = i32
        L.orc_mma_sf_bytes.argtypes = [i64, i64]; L.orc_mma_sf_bytes.restype = i64
        L.orc_mma_sf_offset.argtypes = [i64, i64, i64]; L.orc_mma_sf_offset.restype = i64
        L.orc_mma_scale_byte.argtypes = [i32, i32]; L.orc_mma_scale_byte.restype = i32
        L.orc_mma_pack.argtypes = [vp, vp, i64, i64, i32, vp, vp]; L.orc_mma_pack.restype = i32
        L.orc_gemm.argtypes = [vp, vp, i64, i64, i64, vp, vp, i32]; L.orc_gemm.restype = i32
        L.orc_f64_to_bf16.argtypes = [f64]; L.orc_f64_to_bf16.restype = ctypes.c_uint16
        L.orc_f32_to_f16_sat.argtypes = [f32]; L.orc_f32_to_f16_sat.restype = ctypes.c_uint16
        L.orc_f16_value.argtypes = [ctypes.c_uint16]; L.orc_f16_value.restype = f64
        L.orc_outlier_capacity.argtypes = [i64, f64]; L.orc_outlier_capacity.restype = i64
        L.orc_separate_outliers.argtypes = [vp, i64, i64, i64, f64, i64, vp, vp, vp, vp, vp, vp]
        L.orc_separate_outliers.restype = i32
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _fmt(fmt) -> int:
    return FORMAT_NAMES[fmt] if isinstance(fmt, str) else int(fmt)


def block_size(fmt) -> int:
    return 32 if _fmt(fmt) in (MXFP4, MXFP4_CEIL) else 16


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


# ---- scalar format helpers (each pinned by enumeration in the tests) --------

def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(float(v))


def e4m3_value(byte: int) -> float:
    return lib().orc_e4m3_value(int(byte))


def e4m3_encode(t: float) -> int:
    return lib().orc_e4m3_encode(float(t))


def e3m3_value(byte6: int) -> float:
    return lib().orc_e3m3_value(int(byte6))


def e3m3_encode(t: float) -> int:
    return lib().orc_e3m3_encode(float(t))


def razer_w_pair() -> float:
    """The second special-value pair (+-s2) of the RaZeR weight mode."""
    return lib().orc_razer_w_pair()


def set_razer_w_pair(s2: float) -> None:
    """Change the weight mode's second pair (the offline search only)."""
    lib().orc_set_razer_w_pair(float(s2))


def e8m0_value(byte: int) -> float:
    return lib().orc_e8m0_value(int(byte))


def mx_exponent(a: float) -> int:
    return lib().orc_mx_exponent(float(a))


def mx_exponent_ceil(a: float) -> int:
    """Smallest e with a <= 6 * 2^e, clamped to [-127, 125] (the no-clipping block exponent)."""
    return lib().orc_mx_exponent_ceil(float(a))


def hadamard_entry(i: int, j: int) -> int:
    return lib().orc_hadamard_entry(int(i), int(j))


def wht_constant() -> float:
    return lib().orc_wht_constant()


def wht32(x) -> np.ndarray:
    """Rotated 32-group, RN_f32(RN_f32(H x) * c)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32).reshape(32))
    out = np.empty(32, dtype=np.float32)
    lib().orc_wht32(_ptr(a), _ptr(out))
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float32).ravel()
    L = lib()
    return np.array([L.orc_f32_to_bf16(float(v)) for v in a], dtype=np.uint16).reshape(np.shape(x))


# ---- tensor entry points ------------------------------------------------------

def _as_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    if x.ndim != 2:
        raise ValueError("expected a 2-D matrix")
    if x.strides[1] != 2:
        raise ValueError("rows must be contiguous")
    return x


def tensor_amax(x: np.ndarray, rotate: bool = False, nthreads: int | None = None) -> float:
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    return lib().orc_tensor_amax(_ptr(x), rows, cols, x.strides[0] // 2, int(rotate),
                                 nthreads or default_threads())


def tensor_scale_from_amax(amax: float, fmt="nvfp4") -> float:
    if _fmt(fmt) == NVFP4_RAZER_W:
        return lib().orc_tensor_scale_from_amax_w(float(amax))
    return lib().orc_tensor_scale_from_amax(float(amax))


def quantize(x: np.ndarray, fmt, rotate: bool = False, tensor_scale: float | None = None,
             want_sse: bool = True, nthreads: int | None = None):
    """Quantize a bf16 matrix (uint16 bit patterns, rows contiguous).

    Returns ``(codes[rows, cols/2] u8, scales[rows, cols/B] u8, tensor_scale
    f32, sse f64 or None)``.  ``tensor_scale`` given means the NVFP4 tensor
    scale is an input (no absmax pass); it is ignored for MXFP4.
    """
    x = _as_bf16_bits(x)
    f = _fmt(fmt)
    rows, cols = x.shape
    B = block_size(f)
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // B), dtype=np.uint8)
    ts = np.array([tensor_scale if tensor_scale is not None else 0.0], dtype=np.float32)
    sse = np.zeros(1, dtype=np.float64)
    rc = lib().orc_quantize(_ptr(x), rows, cols, x.strides[0] // 2, f, int(rotate),
                            int(tensor_scale is not None), _ptr(ts), _ptr(codes), _ptr(scales),
                            _ptr(sse) if want_sse else None, nthreads or default_threads())
    if rc == -2:
        raise FloatingPointError("oracle: an element reached the E2M1 encoder as NaN (non-finite input)")
    if rc != 0:
        raise ValueError(f"oracle rejected shape {x.shape} for format {fmt} rotate={rotate}")
    return codes, scales, np.float32(ts[0]), (float(sse[0]) if want_sse else None)


def dequantize(codes: np.ndarray, scales: np.ndarray, tensor_scale: float, fmt,
               rotate: bool = False, nthreads: int | None = None):
    """Return ``(y_f32, y_bf16_bits)``, the reconstruction before and after bf16 rounding."""
    f = _fmt(fmt)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    y32 = np.empty((rows, cols), dtype=np.float32)
    y16 = np.empty((rows, cols), dtype=np.uint16)
    rc = lib().orc_dequantize(_ptr(codes), _ptr(scales), float(tensor_scale), rows, cols, f,
                              int(rotate), _ptr(y32), _ptr(y16), cols,
                              nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected shape")
    return y32, y16


def error(x: np.ndarray, codes: np.ndarray, scales: np.ndarray, tensor_scale: float, fmt,
          rotate: bool = False, nthreads: int | None = None) -> float:
    """Sum of squared errors of the reconstruction against ``x`` (original domain)."""
    x = _as_bf16_bits(x)
    f = _fmt(fmt)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = x.shape
    sse = np.zeros(1, dtype=np.float64)
    rc = lib().orc_error(_ptr(x), x.strides[0] // 2, _ptr(codes), _ptr(scales),
                         float(tensor_scale), rows, cols, f, int(rotate), _ptr(sse),
                         nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected shape")
    return float(sse[0])


# ---------------------------------------------------------------- tensor-core operand form, W4A4 product

def mma_planes(fmt) -> int:
    """Code planes of a format's tensor-core operand form (1 for NVFP4, 2 for RaZeR)."""
    return lib().orc_mma_planes(_fmt(fmt))


def mma_sf_bytes(rows: int, cols: int) -> int:
    return lib().orc_mma_sf_bytes(int(rows), int(cols))


def mma_sf_offset(r: int, kb: int, cols: int) -> int:
    return lib().orc_mma_sf_offset(int(r), int(kb), int(cols))


def mma_scale_byte(fmt, sbyte: int) -> int:
    return lib().orc_mma_scale_byte(_fmt(fmt), int(sbyte))


def mma_pack(codes: np.ndarray, scales: np.ndarray, fmt):
    """Return ``(planes, sf)``: planes uint8 [rows][planes * cols/2], sf uint8 [mma_sf_bytes]."""
    f = _fmt(fmt)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    np_ = mma_planes(f)
    planes = np.empty((rows, np_ * cols // 2), dtype=np.uint8)
    sf = np.empty(mma_sf_bytes(rows, cols), dtype=np.uint8)
    if lib().orc_mma_pack(_ptr(codes), _ptr(scales), rows, cols, f, _ptr(planes), _ptr(sf)) != 0:
        raise ValueError("oracle rejected format or shape")
    return planes, sf


def gemm(a: np.ndarray, w: np.ndarray, nthreads: int | None = None):
    """Return ``(y, yabs)``: y = a w^T and yabs = |a| |w|^T in binary64 (a: M x K, w: N x K fp32)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    (M, K), (N, K2) = a.shape, w.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    y = np.empty((M, N), dtype=np.float64)
    yabs = np.empty((M, N), dtype=np.float64)
    lib().orc_gemm(_ptr(a), _ptr(w), M, N, K, _ptr(y), _ptr(yabs), nthreads or default_threads())
    return y, yabs


# ---------------------------------------------------------------- sparse outlier separation

def f64_to_bf16(v: float) -> int:
    return lib().orc_f64_to_bf16(float(v))


def f32_to_f16_sat(v: float) -> int:
    return lib().orc_f32_to_f16_sat(float(v))


def f16_value(h: int) -> float:
    return lib().orc_f16_value(int(h))


def outlier_capacity(cols: int, max_frac: float = 0.02) -> int:
    return lib().orc_outlier_capacity(int(cols), float(max_frac))


def separate_outliers(x: np.ndarray, k: float = 4.0, max_frac: float = 0.02):
    """Return ``(bulk u16 [rows, cols], cols u16 [rows, cap], vals f16-bits u16 [rows, cap],
    count i32 [rows], mu f64 [rows], thr f64 [rows])``."""
    x = _as_bf16_bits(x)
    rows, cols = x.shape
    cap = outlier_capacity(cols, max_frac)
    bulk = np.empty((rows, cols), dtype=np.uint16)
    oc = np.zeros((rows, max(cap, 1)), dtype=np.uint16)
    ov = np.zeros((rows, max(cap, 1)), dtype=np.uint16)
    cnt = np.zeros(rows, dtype=np.int32)
    mu = np.zeros(rows, dtype=np.float64)
    thr = np.zeros(rows, dtype=np.float64)
    if lib().orc_separate_outliers(_ptr(x), rows, cols, x.strides[0] // 2, float(k), cap, _ptr(bulk), _ptr(oc),
                                   _ptr(ov), _ptr(cnt), _ptr(mu), _ptr(thr)) != 0:
        raise ValueError("oracle rejected shape")
    return bulk, oc[:, :cap], ov[:, :cap], cnt, mu, thr
