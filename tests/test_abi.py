"""C ABI checks that need no GPU: the library builds and loads, exports every
symbol include/fp4q.h declares, and rejects bad arguments on the host before
touching the device.  Pointers here are fake addresses: every call below fails
validation (or the device check) before any pointer is dereferenced."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from activation_quantization_block_b200 import fp4q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp4q.h")

ST = {name: code for code, name in fp4q.STATUS_NAMES.items()}
A = 1 << 20          # a 16-byte-aligned fake address
WS = fp4q.fp4q_workspace_size(0, 0, 0, 0)


def declared_symbols() -> list[str]:
    text = open(HEADER).read()
    return re.findall(r"FP4Q_API\s+[\w\s\*]+?\b(fp4q_\w+)\s*\(", text)


def test_header_declares_what_the_binding_knows():
    assert sorted(declared_symbols()) == sorted(fp4q.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(fp4q.library_path() if os.path.exists(fp4q.library_path()) else fp4q.lib()._name)
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_version_status_strings_workspace():
    assert fp4q.fp4q_abi_version() == 4
    for code in range(7):
        assert fp4q.fp4q_status_string(code)
    assert fp4q.fp4q_status_string(99) == "unknown status"
    assert WS >= 4096 * 12


def q(**kw):
    args = dict(x=A, rows=4, cols=64, ldx=64, fmt=0, rotate=0, flags=0, codes=A, scales=A, tensor_scale=A,
                mse=None, workspace=A, workspace_bytes=WS, stream=0)
    args.update(kw)
    return fp4q.fp4q_quantize(**args)


@pytest.mark.parametrize("kw,expect", [
    (dict(fmt=4), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(fmt=-1), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(fmt=3, cols=40, ldx=40), "FP4Q_ERROR_SHAPE"),          # weight mode: blocks of 16
    (dict(fmt=3, tensor_scale=None), "FP4Q_ERROR_INVALID_VALUE"),  # weight mode needs it
    (dict(rotate=2), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(flags=2), "FP4Q_ERROR_INVALID_VALUE"),                # the MX exponent flag needs MXFP4
    (dict(flags=4), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(rows=-1), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(cols=40, ldx=40), "FP4Q_ERROR_SHAPE"),                 # not a multiple of 16
    (dict(fmt=2, cols=48, ldx=48), "FP4Q_ERROR_SHAPE"),          # MXFP4 needs 32
    (dict(rotate=1, cols=48, ldx=48), "FP4Q_ERROR_SHAPE"),       # rotation needs 32
    (dict(ldx=32), "FP4Q_ERROR_SHAPE"),                          # ld < cols
    (dict(rows=1 << 40, cols=1 << 30, ldx=1 << 30), "FP4Q_ERROR_SHAPE"),   # size overflow
    (dict(x=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(codes=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(scales=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(tensor_scale=None), "FP4Q_ERROR_INVALID_VALUE"),       # NVFP4 needs it
    (dict(x=A + 8), "FP4Q_ERROR_MISALIGNED"),
    (dict(ldx=68), "FP4Q_ERROR_MISALIGNED"),
    (dict(codes=A + 4), "FP4Q_ERROR_MISALIGNED"),
    (dict(scales=A + 1), "FP4Q_ERROR_MISALIGNED"),
    (dict(tensor_scale=A + 2), "FP4Q_ERROR_MISALIGNED"),
    (dict(mse=A + 4), "FP4Q_ERROR_MISALIGNED"),
    (dict(workspace=None), "FP4Q_ERROR_WORKSPACE"),
    (dict(workspace=A + 8), "FP4Q_ERROR_WORKSPACE"),
    (dict(workspace_bytes=WS - 1), "FP4Q_ERROR_WORKSPACE"),
])
def test_quantize_rejects_bad_arguments_before_launch(kw, expect):
    assert q(**kw) == ST[expect]


def test_quantize_argument_rules_that_relax():
    # MXFP4 needs no tensor scale; a given tensor scale and no mse need no workspace.
    ok_then_device = {ST["FP4Q_ERROR_CUDA"], ST["FP4Q_ERROR_UNSUPPORTED_DEVICE"], ST["FP4Q_SUCCESS"]}
    if not _no_gpu():
        pytest.skip("these calls would launch on a real device")
    assert q(fmt=2, tensor_scale=None) in ok_then_device
    assert q(flags=1, workspace=None, workspace_bytes=0) in ok_then_device
    assert q(fmt=3, cols=48, ldx=48) in ok_then_device           # weight mode: 16-element blocks
    assert q(fmt=2, flags=2, tensor_scale=None) in ok_then_device  # MXFP4 with the ceil exponent


def _no_gpu() -> bool:
    import torch
    return not torch.cuda.is_available()


def test_no_cpu_fallback_without_a_device():
    """On a machine with no GPU a valid call reports a CUDA error; nothing runs on the CPU."""
    if not _no_gpu():
        pytest.skip("a device is present")
    assert q() == ST["FP4Q_ERROR_CUDA"]


@pytest.mark.parametrize("kw,expect", [
    (dict(fmt=5), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(cols=24), "FP4Q_ERROR_SHAPE"),
    (dict(y=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(y=A + 2), "FP4Q_ERROR_MISALIGNED"),
    (dict(ldy=60), "FP4Q_ERROR_SHAPE"),
    (dict(tensor_scale=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(codes=A + 8), "FP4Q_ERROR_MISALIGNED"),
])
def test_dequantize_rejects_bad_arguments(kw, expect):
    args = dict(codes=A, scales=A, tensor_scale=A, rows=4, cols=64, fmt=1, rotate=0, y=A, ldy=64, stream=0)
    args.update(kw)
    assert fp4q.fp4q_dequantize(**args) == ST[expect]


@pytest.mark.parametrize("kw,expect", [
    (dict(mse=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(mse=A + 4), "FP4Q_ERROR_MISALIGNED"),
    (dict(workspace=None), "FP4Q_ERROR_WORKSPACE"),
    (dict(workspace_bytes=16), "FP4Q_ERROR_WORKSPACE"),
    (dict(rotate=1, cols=16), "FP4Q_ERROR_SHAPE"),
    (dict(x=A + 16, ldx=12), "FP4Q_ERROR_SHAPE"),
])
def test_error_rejects_bad_arguments(kw, expect):
    args = dict(x=A, ldx=64, codes=A, scales=A, tensor_scale=A, rows=4, cols=64, fmt=0, rotate=0, mse=A,
                workspace=A, workspace_bytes=WS, stream=0)
    args.update(kw)
    assert fp4q.fp4q_error(**args) == ST[expect]


def test_binding_has_no_oracle_or_cpu_path():
    """The product package never imports the oracle."""
    pkg = os.path.join(ROOT, "activation_quantization_block_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "fp4q_oracle" not in text, f


def _desc(**kw):
    d = dict(x=A, rows=4, cols=64, ldx=64, codes=A, scales=A, tensor_scale=A, mse=None)
    d.update(kw)
    return fp4q.TensorDesc(**d)


def test_batch_workspace_size_is_fixed():
    one = fp4q.fp4q_batch_workspace_size(1, [_desc(rows=128, cols=8192, ldx=8192)], 1, 0)
    two = fp4q.fp4q_batch_workspace_size(2, [_desc(rows=128, cols=8192, ldx=8192)] * 2, 1, 0)
    assert one == two == 3 * 4096 * (4 + 8)     # three slots of per-CTA partials


@pytest.mark.parametrize("descs,kw,expect", [
    ([_desc()], dict(count=-1), "FP4Q_ERROR_INVALID_VALUE"),
    ([_desc()], dict(flags=4), "FP4Q_ERROR_INVALID_VALUE"),
    ([_desc(), _desc(cols=40, ldx=40)], {}, "FP4Q_ERROR_SHAPE"),
    ([_desc(), _desc(x=A + 8)], {}, "FP4Q_ERROR_MISALIGNED"),
    ([_desc(tensor_scale=None)], {}, "FP4Q_ERROR_INVALID_VALUE"),
    ([_desc(codes=None)], {}, "FP4Q_ERROR_INVALID_VALUE"),
    ([_desc()], dict(workspace=None), "FP4Q_ERROR_WORKSPACE"),
    ([_desc()], dict(workspace_bytes=100), "FP4Q_ERROR_WORKSPACE"),
])
def test_batch_rejects_bad_arguments(descs, kw, expect):
    args = dict(count=len(descs), descs=descs, fmt=0, rotate=0, flags=0, workspace=A, workspace_bytes=1 << 20,
                stream=0)
    args.update(kw)
    assert fp4q.fp4q_quantize_batch(**args) == ST[expect]


def test_batch_of_nothing_is_a_no_op():
    assert fp4q.fp4q_quantize_batch(0, [], 0, 0, 0, None, 0, 0) == ST["FP4Q_SUCCESS"]


def test_mma_planes_and_sf_bytes():
    assert [fp4q.fp4q_mma_planes(f) for f in (0, 1, 2, 3, 7)] == [1, 2, 0, 2, 0]
    assert fp4q.fp4q_mma_sf_bytes(300, 4096) == 3 * 64 * 512
    assert fp4q.fp4q_mma_sf_bytes(1, 16) == 512 and fp4q.fp4q_mma_sf_bytes(-1, 16) == 0


@pytest.mark.parametrize("kw,expect", [
    (dict(fmt=2), "FP4Q_ERROR_INVALID_VALUE"),                 # MXFP4 has no operand form
    (dict(fmt=9), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(rows=-1), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(cols=40), "FP4Q_ERROR_SHAPE"),
    (dict(planes=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(sf=A + 4), "FP4Q_ERROR_MISALIGNED"),
])
def test_mma_pack_rejects_bad_arguments(kw, expect):
    args = dict(codes=A, scales=A, rows=4, cols=64, fmt=1, planes=A, sf=A, stream=0)
    args.update(kw)
    assert fp4q.fp4q_mma_pack(**args) == ST[expect]


@pytest.mark.parametrize("kw,expect", [
    (dict(a_np=3), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(w_np=0), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(M=-1), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(K=128), "FP4Q_ERROR_SHAPE"),                         # K a multiple of 256
    (dict(K=0), "FP4Q_ERROR_SHAPE"),
    (dict(N=12, ldy=16), "FP4Q_ERROR_SHAPE"),                  # N a multiple of 8
    (dict(ldy=8), "FP4Q_ERROR_SHAPE"),                         # ldy >= N
    (dict(ldy=68), "FP4Q_ERROR_MISALIGNED"),
    (dict(y=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(w_scale=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(a_planes=A + 8), "FP4Q_ERROR_MISALIGNED"),
    (dict(a_scale=A + 2), "FP4Q_ERROR_MISALIGNED"),
])
def test_gemm_rejects_bad_arguments(kw, expect):
    args = dict(a_planes=A, a_sf=A, a_np=2, a_scale=A, w_planes=A, w_sf=A, w_np=1, w_scale=A, M=4, N=64, K=256,
                y=A, ldy=64, stream=0)
    args.update(kw)
    assert fp4q.fp4q_gemm(**args) == ST[expect]


def test_gemm_of_nothing_is_a_no_op():
    assert fp4q.fp4q_gemm(A, A, 1, A, A, A, 1, A, 0, 64, 256, A, 64, 0) == ST["FP4Q_SUCCESS"]


def test_outlier_capacity():
    assert fp4q.fp4q_outlier_capacity(4096, 0.02) == 81
    assert fp4q.fp4q_outlier_capacity(4096, 0.0) == 0 and fp4q.fp4q_outlier_capacity(4096, 1.5) == 0


@pytest.mark.parametrize("kw,expect", [
    (dict(k=0.0), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(max_frac=-0.1), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(rows=-1), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(cols=12, ldx=16, ldb=16), "FP4Q_ERROR_SHAPE"),       # cols a multiple of 8
    (dict(cols=65544, ldx=65544, ldb=65544), "FP4Q_ERROR_SHAPE"),
    (dict(bulk=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(out_count=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(x=A + 8), "FP4Q_ERROR_MISALIGNED"),
    (dict(ldb=60), "FP4Q_ERROR_SHAPE"),
])
def test_separate_outliers_rejects_bad_arguments(kw, expect):
    args = dict(x=A, rows=4, cols=64, ldx=64, k=4.0, max_frac=0.05, bulk=A, ldb=64, out_cols=A, out_vals=A,
                out_count=A, stream=0)
    args.update(kw)
    assert fp4q.fp4q_separate_outliers(**args) == ST[expect]


@pytest.mark.parametrize("kw,expect", [
    (dict(cap=65), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(y=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(ldy=32), "FP4Q_ERROR_SHAPE"),
    (dict(out_count=A + 2), "FP4Q_ERROR_MISALIGNED"),
])
def test_scatter_outliers_rejects_bad_arguments(kw, expect):
    args = dict(out_cols=A, out_vals=A, out_count=A, rows=4, cols=64, cap=3, y=A, ldy=64, stream=0)
    args.update(kw)
    assert fp4q.fp4q_scatter_outliers(**args) == ST[expect]


@pytest.mark.parametrize("kw,expect", [
    (dict(fmt=2), "FP4Q_ERROR_INVALID_VALUE"),                   # MXFP4 has no tensor scale
    (dict(fmt=4), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(rotate=2), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(rows=-1), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(tensor_scale=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(tensor_scale=A + 2), "FP4Q_ERROR_MISALIGNED"),
    (dict(cols=40, ldx=40), "FP4Q_ERROR_SHAPE"),
    (dict(rotate=1, cols=48, ldx=48), "FP4Q_ERROR_SHAPE"),
    (dict(ldx=32), "FP4Q_ERROR_SHAPE"),
    (dict(x=None), "FP4Q_ERROR_INVALID_VALUE"),
    (dict(x=A + 8), "FP4Q_ERROR_MISALIGNED"),
    (dict(ldx=68), "FP4Q_ERROR_MISALIGNED"),
    (dict(workspace=None), "FP4Q_ERROR_WORKSPACE"),
    (dict(workspace=A + 8), "FP4Q_ERROR_WORKSPACE"),
    (dict(workspace_bytes=WS - 1), "FP4Q_ERROR_WORKSPACE"),
])
def test_tensor_scale_rejects_bad_arguments(kw, expect):
    args = dict(x=A, rows=4, cols=64, ldx=64, fmt=1, rotate=0, tensor_scale=A, workspace=A, workspace_bytes=WS,
                stream=0)
    args.update(kw)
    assert fp4q.fp4q_tensor_scale(**args) == ST[expect]


def test_build_entry_expects_the_header_abi_version():
    """__graft_entry__.build() checks the loaded library's ABI version against a literal."""
    ver = re.search(r"#define FP4Q_ABI_VERSION (\d+)", open(HEADER).read()).group(1)
    entry = open(os.path.join(ROOT, "__graft_entry__.py")).read()
    assert f"fp4q_abi_version() == {ver}" in entry
    assert fp4q.fp4q_abi_version() == int(ver)


# ---- the torch-level wrappers reject host tensors before any address reaches the library

def _cpu_quantized(rows=4, cols=64):
    import torch
    return fp4q.Quantized(torch.zeros(rows, cols // 2, dtype=torch.uint8), torch.zeros(rows, cols // 16, dtype=torch.uint8),
                          torch.zeros(1), torch.zeros(1, dtype=torch.float64))


@pytest.mark.parametrize("call", [
    lambda x, q: fp4q.quantize(x),
    lambda x, q: fp4q.tensor_scale(x),
    lambda x, q: fp4q.quantize_batch([x]),
    lambda x, q: fp4q.dequantize(q),
    lambda x, q: fp4q.error(x, q),
    lambda x, q: fp4q.mma_operand(q, "nvfp4"),
    lambda x, q: fp4q.separate_outliers(x),
    lambda x, q: fp4q.scatter_outliers(fp4q.Outliers(x, q.codes, q.codes, q.codes), x),
])
def test_wrappers_reject_host_tensors(call):
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="CUDA tensors only"):
        call(x, _cpu_quantized())


def test_gemm_rejects_host_operands():
    import torch
    op = fp4q.MmaOperand(torch.zeros(128, 128, dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8),
                         torch.ones(1), 1)
    with pytest.raises(TypeError, match="CUDA tensors only"):
        fp4q.gemm(op, op)


def test_device_of_mixed_tensors():
    import torch
    with pytest.raises(TypeError):
        fp4q._device(None, None)
    with pytest.raises(TypeError):
        fp4q._device(torch.zeros(1, device="meta"))
    with pytest.raises(TypeError, match="bf16"):
        fp4q._bf16(torch.zeros(1))
    fp4q._bf16(None, torch.zeros(1, dtype=torch.bfloat16))


C_CLIENT = r"""
#include <stdio.h>
#include <stdint.h>
#include "fp4q.h"

int main(void)
{
    /* a plain C caller: version, status strings and host-side validation (no device needed) */
    if (fp4q_abi_version() != FP4Q_ABI_VERSION) return 1;
    if (fp4q_status_string(FP4Q_ERROR_SHAPE)[0] == 0) return 2;
    uintptr_t a = (uintptr_t)1 << 20;                      /* fake 16-byte-aligned addresses */
    size_t ws = fp4q_workspace_size(4, 64, FP4Q_NVFP4_RAZER, 0);
    fp4q_status_t s = fp4q_quantize((const void*)a, 4, 40, 40, FP4Q_NVFP4_RAZER, 0, 0, (uint8_t*)a, (uint8_t*)a,
                                    (float*)a, NULL, (void*)a, ws, NULL);
    if (s != FP4Q_ERROR_SHAPE) return 3;
    s = fp4q_tensor_scale((const void*)a, 4, 64, 64, FP4Q_MXFP4, 0, (float*)a, (void*)a, ws, NULL);
    if (s != FP4Q_ERROR_INVALID_VALUE) return 4;
    s = fp4q_gemm((const uint8_t*)a, (const uint8_t*)a, 3, (const float*)a, (const uint8_t*)a, (const uint8_t*)a, 1,
                  (const float*)a, 8, 8, 256, (void*)a, 8, NULL);
    if (s != FP4Q_ERROR_INVALID_VALUE) return 5;
    if (fp4q_mma_planes(FP4Q_NVFP4_RAZER) != 2 || fp4q_mma_planes(FP4Q_NVFP4) != 1) return 6;
    printf("ok\n");
    return 0;
}
"""


def test_a_plain_c_program_links_and_calls_the_abi(tmp_path):
    """The boundary is a C ABI: a C11 program compiles against include/fp4q.h alone, links
    libfp4q.so and gets the documented statuses from host-side validation."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = fp4q.lib()._name
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                    lib, f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_the_bounds_checking_twin_loads_and_says_so():
    """libfp4q_debug.so (FP4Q_DEBUG=1) exports the same C ABI and reports the debug build; the
    release library does not.  Loading needs no GPU."""
    import ctypes

    from activation_quantization_block_b200 import _build
    dbg = ctypes.CDLL(_build.build_debug())
    rel = ctypes.CDLL(_build.build())
    for L in (dbg, rel):
        L.fp4q_debug_build.restype = ctypes.c_int
        L.fp4q_abi_version.restype = ctypes.c_int
        assert L.fp4q_abi_version() == 4
        for name in fp4q.ABI_SYMBOLS:
            assert hasattr(L, name), name
    assert dbg.fp4q_debug_build() == 1 and rel.fp4q_debug_build() == 0
