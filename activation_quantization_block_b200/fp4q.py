"""Python binding of the fp4q C ABI (``include/fp4q.h``).

The functions named ``fp4q_*`` mirror the C entry points one to one: they only
marshal arguments (torch tensors become device pointers, the stream becomes a
``cudaStream_t``) and return the C status code.  The convenience wrappers
``quantize`` / ``dequantize`` / ``error`` allocate outputs with torch, pass the
current torch stream and raise ``Fp4qError`` on a non-success status.  Every
step of the computation runs in the CUDA library; there is no CPU path, and a
missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple

import torch

from . import _build

NVFP4, NVFP4_RAZER, MXFP4, NVFP4_RAZER_W = 0, 1, 2, 3
FORMATS = {"nvfp4": NVFP4, "nvfp4_razer": NVFP4_RAZER, "mxfp4": MXFP4, "nvfp4_razer_w": NVFP4_RAZER_W}
FLAG_TENSOR_SCALE_GIVEN = 0x1
FLAG_MX_CEIL_SCALE = 0x2

SUCCESS = 0
STATUS_NAMES = {
    0: "FP4Q_SUCCESS", 1: "FP4Q_ERROR_INVALID_VALUE", 2: "FP4Q_ERROR_SHAPE", 3: "FP4Q_ERROR_MISALIGNED",
    4: "FP4Q_ERROR_WORKSPACE", 5: "FP4Q_ERROR_UNSUPPORTED_DEVICE", 6: "FP4Q_ERROR_CUDA",
}

# Names the C header declares; the tests check that the library exports each one.
ABI_SYMBOLS = ("fp4q_abi_version", "fp4q_status_string", "fp4q_workspace_size",
               "fp4q_quantize", "fp4q_dequantize", "fp4q_error", "fp4q_quantize_noalloc",
               "fp4q_device_errors", "fp4q_batch_workspace_size", "fp4q_quantize_batch",
               "fp4q_mma_planes", "fp4q_mma_sf_bytes", "fp4q_mma_pack", "fp4q_gemm",
               "fp4q_outlier_capacity", "fp4q_separate_outliers", "fp4q_scatter_outliers",
               "fp4q_selftest_timeout", "fp4q_tensor_scale", "fp4q_device_error_site", "fp4q_debug_build")


class TensorDesc(ctypes.Structure):
    """fp4q_tensor_desc_t: one tensor of a batch (device pointers)."""
    _fields_ = [("x", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("ldx", ctypes.c_int64), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("mse", ctypes.c_void_p)]


class Fp4qError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({fp4q_status_string(status)})")


_lib = None


# FP4Q_DEBUG_LIBRARY=1 in the environment loads the bounds-checking build
# (libfp4q_debug.so) in place of libfp4q.so.
DEBUG_ENV = "FP4Q_DEBUG_LIBRARY"


def _want_debug() -> bool:
    return os.environ.get(DEBUG_ENV, "") not in ("", "0")


def library_path() -> str:
    return _build.DEBUG_LIB if _want_debug() else _build.LIB


def lib() -> ctypes.CDLL:
    """Load (building first if the sources are newer) the in-tree libfp4q.so, or with
    FP4Q_DEBUG_LIBRARY=1 the bounds-checking libfp4q_debug.so."""
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build_debug() if _want_debug() else _build.build())
        vp, i64, i32, u32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32, ctypes.c_size_t
        L.fp4q_abi_version.argtypes = []
        L.fp4q_abi_version.restype = i32
        L.fp4q_status_string.argtypes = [i32]
        L.fp4q_status_string.restype = ctypes.c_char_p
        L.fp4q_workspace_size.argtypes = [i64, i64, i32, i32]
        L.fp4q_workspace_size.restype = sz
        L.fp4q_quantize.argtypes = [vp, i64, i64, i64, i32, i32, u32, vp, vp, vp, vp, vp, sz, vp]
        L.fp4q_quantize.restype = i32
        L.fp4q_dequantize.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp, i64, vp]
        L.fp4q_dequantize.restype = i32
        L.fp4q_error.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, i32, vp, vp, sz, vp]
        L.fp4q_error.restype = i32
        L.fp4q_quantize_noalloc.argtypes = [vp, i64, i64, i64, i32, i32, u32, vp, vp, vp, vp, vp]
        L.fp4q_quantize_noalloc.restype = i32
        L.fp4q_device_error_site.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint64)]
        L.fp4q_device_error_site.restype = i32
        L.fp4q_debug_build.argtypes = []
        L.fp4q_debug_build.restype = i32
        L.fp4q_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
        L.fp4q_device_errors.restype = i32
        L.fp4q_batch_workspace_size.argtypes = [i32, ctypes.POINTER(TensorDesc), i32, i32]
        L.fp4q_batch_workspace_size.restype = sz
        L.fp4q_quantize_batch.argtypes = [i32, ctypes.POINTER(TensorDesc), i32, i32, u32, vp, sz, vp]
        L.fp4q_quantize_batch.restype = i32
        L.fp4q_mma_planes.argtypes = [i32]
        L.fp4q_mma_planes.restype = i32
        L.fp4q_mma_sf_bytes.argtypes = [i64, i64]
        L.fp4q_mma_sf_bytes.restype = sz
        L.fp4q_mma_pack.argtypes = [vp, vp, i64, i64, i32, vp, vp, vp]
        L.fp4q_mma_pack.restype = i32
        L.fp4q_gemm.argtypes = [vp, vp, i32, vp, vp, vp, i32, vp, i64, i64, i64, vp, i64, vp]
        L.fp4q_gemm.restype = i32
        f64 = ctypes.c_double
        L.fp4q_outlier_capacity.argtypes = [i64, f64]
        L.fp4q_outlier_capacity.restype = i64
        L.fp4q_separate_outliers.argtypes = [vp, i64, i64, i64, f64, f64, vp, i64, vp, vp, vp, vp]
        L.fp4q_separate_outliers.restype = i32
        L.fp4q_scatter_outliers.argtypes = [vp, vp, vp, i64, i64, i64, vp, i64, vp]
        L.fp4q_scatter_outliers.restype = i32
        L.fp4q_selftest_timeout.argtypes = [vp]
        L.fp4q_selftest_timeout.restype = i32
        L.fp4q_tensor_scale.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp, sz, vp]
        L.fp4q_tensor_scale.restype = i32
        _lib = L
    return _lib


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


# ---- the C entry points, same names --------------------------------------------

def fp4q_abi_version() -> int:
    return lib().fp4q_abi_version()


def fp4q_status_string(status: int) -> str:
    return lib().fp4q_status_string(int(status)).decode()


def fp4q_workspace_size(rows: int, cols: int, fmt, rotate: int) -> int:
    return lib().fp4q_workspace_size(rows, cols, _fmt(fmt), int(rotate))


def fp4q_quantize(x, rows, cols, ldx, fmt, rotate, flags, codes, scales, tensor_scale, mse,
                  workspace, workspace_bytes, stream=None) -> int:
    return lib().fp4q_quantize(_ptr(x), rows, cols, ldx, _fmt(fmt), int(rotate), flags, _ptr(codes),
                               _ptr(scales), _ptr(tensor_scale), _ptr(mse), _ptr(workspace),
                               workspace_bytes, _stream(stream))


def fp4q_dequantize(codes, scales, tensor_scale, rows, cols, fmt, rotate, y, ldy, stream=None) -> int:
    return lib().fp4q_dequantize(_ptr(codes), _ptr(scales), _ptr(tensor_scale), rows, cols, _fmt(fmt),
                                 int(rotate), _ptr(y), ldy, _stream(stream))


def fp4q_error(x, ldx, codes, scales, tensor_scale, rows, cols, fmt, rotate, mse, workspace,
               workspace_bytes, stream=None) -> int:
    return lib().fp4q_error(_ptr(x), ldx, _ptr(codes), _ptr(scales), _ptr(tensor_scale), rows, cols,
                            _fmt(fmt), int(rotate), _ptr(mse), _ptr(workspace), workspace_bytes,
                            _stream(stream))


def fp4q_tensor_scale(x, rows, cols, ldx, fmt, rotate, tensor_scale, workspace, workspace_bytes,
                      stream=None) -> int:
    return lib().fp4q_tensor_scale(_ptr(x), rows, cols, ldx, _fmt(fmt), int(rotate), _ptr(tensor_scale),
                                   _ptr(workspace), workspace_bytes, _stream(stream))


def fp4q_quantize_noalloc(x, rows, cols, ldx, fmt, rotate, flags, codes, scales, tensor_scale, mse,
                          stream=None) -> int:
    """fp4q_quantize with the library's static scratch: for callers that cannot allocate."""
    return lib().fp4q_quantize_noalloc(_ptr(x), rows, cols, ldx, _fmt(fmt), int(rotate), flags, _ptr(codes),
                                       _ptr(scales), _ptr(tensor_scale), _ptr(mse), _stream(stream))


def fp4q_device_errors(clear: bool = False) -> tuple[int, int]:
    """(status, error bits) of the current device; synchronous."""
    v = ctypes.c_uint32(0)
    st = lib().fp4q_device_errors(ctypes.byref(v), int(clear))
    return st, v.value


def fp4q_device_error_site() -> tuple[int, int, int]:
    """(status, site, byte offset) of the first out-of-bounds access a debug build found."""
    site, off = ctypes.c_uint32(0), ctypes.c_uint64(0)
    st = lib().fp4q_device_error_site(ctypes.byref(site), ctypes.byref(off))
    return st, site.value, off.value


def fp4q_debug_build() -> int:
    """1 when the loaded library is the bounds-checking build."""
    return lib().fp4q_debug_build()


def _descs(descs):
    if isinstance(descs, ctypes.Array):
        return descs
    arr = (TensorDesc * max(1, len(descs)))()
    for i, d in enumerate(descs):
        arr[i] = d
    return arr


def fp4q_batch_workspace_size(count, descs, fmt, rotate) -> int:
    return lib().fp4q_batch_workspace_size(count, _descs(descs), _fmt(fmt), int(rotate))


def fp4q_quantize_batch(count, descs, fmt, rotate, flags, workspace, workspace_bytes, stream=None) -> int:
    return lib().fp4q_quantize_batch(count, _descs(descs), _fmt(fmt), int(rotate), flags, _ptr(workspace),
                                     workspace_bytes, _stream(stream))


def fp4q_mma_planes(fmt) -> int:
    return lib().fp4q_mma_planes(_fmt(fmt))


def fp4q_mma_sf_bytes(rows: int, cols: int) -> int:
    return lib().fp4q_mma_sf_bytes(rows, cols)


def fp4q_mma_pack(codes, scales, rows, cols, fmt, planes, sf, stream=None) -> int:
    return lib().fp4q_mma_pack(_ptr(codes), _ptr(scales), rows, cols, _fmt(fmt), _ptr(planes), _ptr(sf),
                               _stream(stream))


def fp4q_gemm(a_planes, a_sf, a_np, a_scale, w_planes, w_sf, w_np, w_scale, M, N, K, y, ldy, stream=None) -> int:
    return lib().fp4q_gemm(_ptr(a_planes), _ptr(a_sf), a_np, _ptr(a_scale), _ptr(w_planes), _ptr(w_sf), w_np,
                           _ptr(w_scale), M, N, K, _ptr(y), ldy, _stream(stream))


def fp4q_selftest_timeout(stream=None) -> int:
    return lib().fp4q_selftest_timeout(_stream(stream))


def fp4q_outlier_capacity(cols: int, max_frac: float) -> int:
    return lib().fp4q_outlier_capacity(cols, max_frac)


def fp4q_separate_outliers(x, rows, cols, ldx, k, max_frac, bulk, ldb, out_cols, out_vals, out_count,
                           stream=None) -> int:
    return lib().fp4q_separate_outliers(_ptr(x), rows, cols, ldx, k, max_frac, _ptr(bulk), ldb, _ptr(out_cols),
                                        _ptr(out_vals), _ptr(out_count), _stream(stream))


def fp4q_scatter_outliers(out_cols, out_vals, out_count, rows, cols, cap, y, ldy, stream=None) -> int:
    return lib().fp4q_scatter_outliers(_ptr(out_cols), _ptr(out_vals), _ptr(out_count), rows, cols, cap, _ptr(y),
                                       ldy, _stream(stream))


def tensor_desc(x, q: "Quantized") -> TensorDesc:
    """Descriptor of bf16 matrix x and its outputs q (torch tensors)."""
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    return TensorDesc(x.data_ptr(), rows, cols, ld, q.codes.data_ptr(), q.scales.data_ptr(),
                      q.tensor_scale.data_ptr() if q.tensor_scale is not None else None,
                      q.mse.data_ptr() if q.mse is not None else None)


# ---- torch-level wrappers -------------------------------------------------------

class Quantized(NamedTuple):
    codes: torch.Tensor          # uint8 [rows, cols/2]
    scales: torch.Tensor         # uint8 [rows, cols/16] or [rows, cols/32]
    tensor_scale: torch.Tensor   # float32 [1] (zero and unused for MXFP4)
    mse: torch.Tensor | None     # float64 [1] or None


def block_size(fmt) -> int:
    return 32 if _fmt(fmt) == MXFP4 else 16


def _check(status: int, what: str):
    if status != SUCCESS:
        raise Fp4qError(status, what)


_workspaces: dict = {}


def workspace_for(device: torch.device, stream=None) -> torch.Tensor:
    """A cached workspace tensor per (device, stream); calls on one stream are ordered."""
    key = (device, _stream(stream))
    ws = _workspaces.get(key)
    if ws is None:
        n = lib().fp4q_workspace_size(0, 0, 0, 0)
        ws = torch.empty(n, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def _rows_cols_ld(x: torch.Tensor):
    if x.dim() != 2:
        raise ValueError("expected a 2-D tensor")
    if x.stride(1) != 1:
        raise ValueError("rows must be contiguous (stride(1) == 1)")
    return x.shape[0], x.shape[1], x.stride(0) if x.shape[0] > 1 else x.shape[1]


def _device(*tensors) -> torch.device:
    """The one CUDA device every given tensor (None skipped) lives on.  The C ABI takes device
    pointers only and cannot tell a host address from a device one, so a host tensor, or a
    tensor of another device, is rejected here before its address reaches a kernel."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise TypeError("fp4q takes CUDA tensors only")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on two devices: {dev} and {t.device}")
    if dev is None:
        raise TypeError("no tensor given")
    return dev


def _bf16(*tensors):
    for t in tensors:
        if t is not None and t.dtype != torch.bfloat16:
            raise TypeError("expected bf16 tensors")


def quantize(x: torch.Tensor, fmt="nvfp4_razer", rotate: bool = False, tensor_scale: torch.Tensor | None = None,
             want_mse: bool = True, out: Quantized | None = None, workspace: torch.Tensor | None = None,
             stream=None, mx_ceil: bool = False) -> Quantized:
    """Quantize a bf16 CUDA matrix; returns codes, scales, tensor scale and (optionally) the MSE.

    mx_ceil (MXFP4): block exponent without clipping (FP4Q_FLAG_MX_CEIL_SCALE)."""
    dev = _device(x, tensor_scale, workspace, *(out or ()))
    _bf16(x)
    rows, cols, ld = _rows_cols_ld(x)
    f = _fmt(fmt)
    B = block_size(f)
    with torch.cuda.device(dev):
        if out is None:
            codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
            scales = torch.empty(rows, cols // B, dtype=torch.uint8, device=dev)
            ts = torch.zeros(1, dtype=torch.float32, device=dev) if tensor_scale is None else tensor_scale
            mse = torch.empty(1, dtype=torch.float64, device=dev) if want_mse else None
        else:
            codes, scales, ts, mse = out
            if tensor_scale is not None:
                ts = tensor_scale
        ws = workspace if workspace is not None else workspace_for(dev, stream)
        flags = (FLAG_TENSOR_SCALE_GIVEN if tensor_scale is not None else 0) | (FLAG_MX_CEIL_SCALE if mx_ceil else 0)
        st = fp4q_quantize(x, rows, cols, ld, f, rotate, flags, codes, scales, ts, mse, ws, ws.numel(), stream)
    _check(st, "fp4q_quantize")
    return Quantized(codes, scales, ts, mse)


def tensor_scale(x: torch.Tensor, fmt="nvfp4_razer", rotate: bool = False, out: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The tensor scale s_t of an NVFP4 format alone (float32 [1] on x's device): the value quantize
    computes when no tensor_scale is given."""
    dev = _device(x, out, workspace)
    _bf16(x)
    rows, cols, ld = _rows_cols_ld(x)
    with torch.cuda.device(dev):
        ts = out if out is not None else torch.empty(1, dtype=torch.float32, device=dev)
        ws = workspace if workspace is not None else workspace_for(dev, stream)
        st = fp4q_tensor_scale(x, rows, cols, ld, fmt, rotate, ts, ws, ws.numel(), stream)
    _check(st, "fp4q_tensor_scale")
    return ts


def empty_like_quantized(x: torch.Tensor, fmt, want_mse: bool = True) -> Quantized:
    rows, cols = x.shape
    B = block_size(fmt)
    return Quantized(torch.empty(rows, cols // 2, dtype=torch.uint8, device=x.device),
                     torch.empty(rows, cols // B, dtype=torch.uint8, device=x.device),
                     torch.zeros(1, dtype=torch.float32, device=x.device),
                     torch.empty(1, dtype=torch.float64, device=x.device) if want_mse else None)


def quantize_batch(xs, fmt="nvfp4_razer", rotate: bool = False, outs=None, scale_given: bool = False,
                   want_mse: bool = True, workspace: torch.Tensor | None = None, stream=None,
                   mx_ceil: bool = False) -> list:
    """Quantize a list of bf16 CUDA matrices with one fp4q_quantize_batch call.

    With scale_given, each out's tensor_scale holds the input scale."""
    if not xs:
        return []
    dev = _device(*xs, workspace, *(t for q in (outs or ()) for t in q))
    _bf16(*xs)
    with torch.cuda.device(dev):
        if outs is None:
            outs = [empty_like_quantized(x, fmt, want_mse) for x in xs]
        descs = _descs([tensor_desc(x, q) for x, q in zip(xs, outs)])
        need = fp4q_batch_workspace_size(len(xs), descs, fmt, rotate)
        ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=dev)
        flags = (FLAG_TENSOR_SCALE_GIVEN if scale_given else 0) | (FLAG_MX_CEIL_SCALE if mx_ceil else 0)
        st = fp4q_quantize_batch(len(xs), descs, fmt, rotate, flags, ws, ws.numel(), stream)
    _check(st, "fp4q_quantize_batch")
    return outs


def dequantize(q: Quantized, fmt="nvfp4_razer", rotate: bool = False, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """bf16 reconstruction of a quantized matrix."""
    dev = _device(*q, out)
    _bf16(out)
    rows, cols = q.codes.shape[0], q.codes.shape[1] * 2
    with torch.cuda.device(dev):
        y = out if out is not None else torch.empty(rows, cols, dtype=torch.bfloat16, device=dev)
        ldy = y.stride(0) if rows > 1 else cols
        st = fp4q_dequantize(q.codes, q.scales, q.tensor_scale, rows, cols, _fmt(fmt), rotate, y, ldy, stream)
    _check(st, "fp4q_dequantize")
    return y


def error(x: torch.Tensor, q: Quantized, fmt="nvfp4_razer", rotate: bool = False,
          workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """MSE (fp64 [1] on the device) of the reconstruction against x."""
    dev = _device(x, *q, workspace)
    _bf16(x)
    rows, cols, ld = _rows_cols_ld(x)
    with torch.cuda.device(dev):
        mse = torch.empty(1, dtype=torch.float64, device=dev)
        ws = workspace if workspace is not None else workspace_for(dev, stream)
        st = fp4q_error(x, ld, q.codes, q.scales, q.tensor_scale, rows, cols, _fmt(fmt), rotate, mse, ws,
                        ws.numel(), stream)
    _check(st, "fp4q_error")
    return mse


class MmaOperand(NamedTuple):
    planes: torch.Tensor         # uint8 [rows, planes * cols/2]
    sf: torch.Tensor             # uint8 [fp4q_mma_sf_bytes(rows, cols)]
    tensor_scale: torch.Tensor   # float32 [1]
    nplanes: int


def mma_operand(q: Quantized, fmt, stream=None) -> MmaOperand:
    """Tensor-core operand form of a quantized NVFP4-family matrix."""
    dev = _device(*q)
    rows, cols = q.codes.shape[0], q.codes.shape[1] * 2
    npl = fp4q_mma_planes(fmt)
    if npl == 0:
        raise Fp4qError(1, "no operand form for this format")
    with torch.cuda.device(dev):
        planes = torch.empty(rows, npl * cols // 2, dtype=torch.uint8, device=dev)
        sf = torch.empty(max(1, fp4q_mma_sf_bytes(rows, cols)), dtype=torch.uint8, device=dev)
        st = fp4q_mma_pack(q.codes, q.scales, rows, cols, fmt, planes, sf, stream)
    _check(st, "fp4q_mma_pack")
    return MmaOperand(planes, sf, q.tensor_scale, npl)


def gemm(a: MmaOperand, w: MmaOperand, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bf16 y = A^ W^T of two operands in tensor-core form (A: M x K, W: N x K)."""
    dev = _device(a.planes, a.sf, a.tensor_scale, w.planes, w.sf, w.tensor_scale, out)
    _bf16(out)
    M, N = a.planes.shape[0], w.planes.shape[0]
    K = a.planes.shape[1] * 2 // a.nplanes
    if w.planes.shape[1] * 2 // w.nplanes != K:
        raise ValueError("inner dimensions differ")
    with torch.cuda.device(dev):
        y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ldy = y.stride(0) if M > 1 else N
        st = fp4q_gemm(a.planes, a.sf, a.nplanes, a.tensor_scale, w.planes, w.sf, w.nplanes, w.tensor_scale, M, N,
                       K, y, ldy, stream)
    _check(st, "fp4q_gemm")
    return y


class Outliers(NamedTuple):
    bulk: torch.Tensor       # bf16 [rows, cols]: x with the row mean at every outlier
    cols: torch.Tensor       # int16 (uint16 bit patterns) [rows, cap]
    vals: torch.Tensor       # float16 [rows, cap]
    count: torch.Tensor      # int32 [rows]


def separate_outliers(x: torch.Tensor, k: float = 4.0, max_frac: float = 0.02, stream=None) -> Outliers:
    """Sparse outlier separation of a bf16 CUDA matrix (rows are the groups)."""
    dev = _device(x)
    _bf16(x)
    rows, cols, ld = _rows_cols_ld(x)
    cap = fp4q_outlier_capacity(cols, max_frac)
    with torch.cuda.device(dev):
        o = Outliers(torch.empty(rows, cols, dtype=torch.bfloat16, device=dev),
                     torch.zeros(rows, max(cap, 1), dtype=torch.int16, device=dev),
                     torch.zeros(rows, max(cap, 1), dtype=torch.float16, device=dev),
                     torch.zeros(rows, dtype=torch.int32, device=dev))
        st = fp4q_separate_outliers(x, rows, cols, ld, k, max_frac, o.bulk, cols, o.cols, o.vals, o.count, stream)
    _check(st, "fp4q_separate_outliers")
    return o


def scatter_outliers(o: Outliers, y: torch.Tensor, max_frac: float = 0.02, stream=None) -> torch.Tensor:
    """Put the outliers of o back into the bf16 reconstruction y (in place)."""
    dev = _device(*o, y)
    _bf16(y)
    rows, cols = y.shape
    cap = fp4q_outlier_capacity(cols, max_frac)
    ldy = y.stride(0) if rows > 1 else cols
    with torch.cuda.device(dev):
        st = fp4q_scatter_outliers(o.cols, o.vals, o.count, rows, cols, cap, y, ldy, stream)
    _check(st, "fp4q_scatter_outliers")
    return y
