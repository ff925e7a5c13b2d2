"""Time one fp4q operation on one seeded tensor.

    python -m activation_quantization_block_b200.kernel_bench --op quantize --fmt nvfp4_razer \\
        --rows 14336 --cols 4096 [--rotate] [--no-mse] [--scale-given] [--iters 20]
    python -m activation_quantization_block_b200.kernel_bench --op gemm --a-fmt nvfp4_razer \\
        --w-fmt nvfp4_razer_w --M 8192 --N 8192 --K 8192

Each iteration is one C-ABI call on the current stream, timed with CUDA events;
between iterations a 512 MB buffer is overwritten so that no input stays in
L2 (--no-flush keeps them).  Prints one JSON line: median and minimum time
per call, elements/s and the call's algorithmic bytes per second
(quantize: 2 B read + codes and scales written, plus 2 B for the absmax read
when the tensor scale is computed; dequantize: codes and scales read + 2 B
written; error: 2 B + codes and scales read; tensor_scale: 2 B read, the absmax
pass alone).

--op gemm times fp4q_gemm on the operand forms of a seeded activation-like A
(M x K, --a-fmt) and LLM-weight W (N x K, --w-fmt) and reports TFLOP/s: useful
(2 M N K) and on the tensor cores (times the plane passes), and their fraction
of the dense FP4 peak, taken as the measured bf16 peak of MEASURED_PEAKS.json
times 4 (the nominal FP4 / bf16 ratio, 9 / 2.25 PFLOP/s).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics

import torch

from . import fp4q, synthetic


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--op", choices=["quantize", "dequantize", "error", "tensor_scale", "gemm", "outliers"],
                   default="quantize")
    p.add_argument("--fmt", choices=list(fp4q.FORMATS), default="nvfp4_razer")
    p.add_argument("--rows", type=int, default=14336)
    p.add_argument("--cols", type=int, default=4096)
    p.add_argument("--rotate", action="store_true")
    p.add_argument("--no-mse", action="store_true")
    p.add_argument("--scale-given", action="store_true")
    p.add_argument("--mx-ceil", action="store_true", help="MXFP4 block exponent without clipping")
    p.add_argument("--data", choices=["weight", "activation", "mlp"], default="weight")
    p.add_argument("--seed", type=int, default=2)
    p.add_argument("--iters", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--no-flush", action="store_true")
    p.add_argument("--a-fmt", choices=["nvfp4", "nvfp4_razer", "nvfp4_razer_w"], default="nvfp4_razer")
    p.add_argument("--w-fmt", choices=["nvfp4", "nvfp4_razer", "nvfp4_razer_w"], default="nvfp4_razer_w")
    p.add_argument("--M", type=int, default=8192)
    p.add_argument("--N", type=int, default=8192)
    p.add_argument("--K", type=int, default=8192)
    a = p.parse_args(argv)
    if a.op == "gemm":
        return gemm_main(a)
    if a.op == "outliers":
        return outliers_main(a)

    dev = torch.device("cuda", torch.cuda.current_device())
    gen = {"weight": synthetic.llm_weight, "activation": synthetic.activation_t3,
           "mlp": synthetic.mlp_row_scaled}[a.data]
    x = gen(a.rows, a.cols, seed=a.seed, device=dev)
    n = x.numel()
    B = fp4q.block_size(a.fmt)
    q = fp4q.quantize(x, a.fmt, a.rotate, want_mse=True)
    y = torch.empty_like(x)
    ws = torch.zeros(fp4q.fp4q_workspace_size(a.rows, a.cols, a.fmt, int(a.rotate)), dtype=torch.uint8, device=dev)
    mse = torch.empty(1, dtype=torch.float64, device=dev)
    flush = None if a.no_flush else torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    packed = n // 2 + n // B
    if a.op == "quantize":
        flags = (fp4q.FLAG_TENSOR_SCALE_GIVEN if a.scale_given else 0) | (fp4q.FLAG_MX_CEIL_SCALE if a.mx_ceil else 0)
        nbytes = 2 * n + packed + (0 if a.scale_given or a.fmt == "mxfp4" else 2 * n)

        def call():
            return fp4q.fp4q_quantize(x, a.rows, a.cols, a.cols, a.fmt, int(a.rotate), flags, q.codes, q.scales,
                                      q.tensor_scale, None if a.no_mse else mse, ws, ws.numel())
    elif a.op == "tensor_scale":
        nbytes = 2 * n   # the absmax pass reads x once
        ts = torch.empty(1, dtype=torch.float32, device=dev)

        def call():
            return fp4q.fp4q_tensor_scale(x, a.rows, a.cols, a.cols, a.fmt, int(a.rotate), ts, ws, ws.numel())
    elif a.op == "dequantize":
        nbytes = packed + 2 * n

        def call():
            return fp4q.fp4q_dequantize(q.codes, q.scales, q.tensor_scale, a.rows, a.cols, a.fmt, int(a.rotate),
                                        y, a.cols)
    else:
        nbytes = 2 * n + packed

        def call():
            return fp4q.fp4q_error(x, a.cols, q.codes, q.scales, q.tensor_scale, a.rows, a.cols, a.fmt,
                                   int(a.rotate), mse, ws, ws.numel())

    for _ in range(a.warmup):
        assert call() == 0
    torch.cuda.synchronize()
    times = []
    for _ in range(a.iters):
        if flush is not None:
            flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        st = call()
        e1.record()
        assert st == 0, fp4q.fp4q_status_string(st)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    med, best = statistics.median(times), min(times)
    mse_value = None
    if a.op == "quantize" and not a.no_mse:
        mse_value = mse.item()
    elif a.op == "error":
        mse_value = mse.item()
    print(json.dumps({
        "op": a.op, "fmt": a.fmt, "rotate": a.rotate, "mse": not a.no_mse, "scale_given": a.scale_given,
        "mse_value": mse_value,
        "mx_ceil": a.mx_ceil,
        "rows": a.rows, "cols": a.cols, "data": a.data, "l2_flushed": flush is not None,
        "ms_median": med, "ms_min": best, "elements_per_s": n / (med / 1e3),
        "algorithmic_bytes": nbytes, "gbs_median": nbytes / (med / 1e3) / 1e9, "gbs_best": nbytes / (best / 1e3) / 1e9,
    }), flush=True)


def fp4_peak_tflops():
    """Dense FP4 peak: measured bf16 burst peak x 4, else the pool's fallback bf16 figure x 4."""
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return 4.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 x 4"
    except (OSError, ValueError, KeyError):
        return 4.0 * 1590.0, "fallback bf16 x 4"


def outliers_main(a):
    """fp4q_separate_outliers on one seeded tensor (algorithmic bytes: x read, bulk written, outlier
    slots written); also the reconstruction error of the separated pipeline against direct quantization."""
    dev = torch.device("cuda", torch.cuda.current_device())
    gen = {"weight": synthetic.llm_weight, "activation": synthetic.activation_t3,
           "mlp": synthetic.mlp_row_scaled}[a.data]
    x = gen(a.rows, a.cols, seed=a.seed, device=dev)
    n = x.numel()
    o = fp4q.separate_outliers(x)
    cap = fp4q.fp4q_outlier_capacity(a.cols, 0.02)
    nbytes = 4 * n + a.rows * (4 * cap + 4)
    flush = None if a.no_flush else torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)

    def call():
        return fp4q.fp4q_separate_outliers(x, a.rows, a.cols, a.cols, 4.0, 0.02, o.bulk, a.cols, o.cols, o.vals,
                                           o.count)

    for _ in range(a.warmup):
        assert call() == 0
    torch.cuda.synchronize()
    times = []
    for _ in range(a.iters):
        if flush is not None:
            flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        st = call()
        e1.record()
        assert st == 0, fp4q.fp4q_status_string(st)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    med = statistics.median(times)
    y = fp4q.scatter_outliers(o, fp4q.dequantize(fp4q.quantize(o.bulk, a.fmt), a.fmt))
    yx = fp4q.dequantize(fp4q.quantize(x, a.fmt), a.fmt)
    err_sep = ((y.double() - x.double()) ** 2).mean().item()
    err_dir = ((yx.double() - x.double()) ** 2).mean().item()
    print(json.dumps({
        "op": "outliers", "fmt": a.fmt, "rows": a.rows, "cols": a.cols, "data": a.data,
        "l2_flushed": flush is not None, "ms_median": med, "ms_min": min(times),
        "algorithmic_bytes": nbytes, "gbs_median": nbytes / (med / 1e3) / 1e9,
        "outlier_fraction": o.count.sum().item() / n, "mse_separated": err_sep, "mse_direct": err_dir,
    }), flush=True)
    return 0


def gemm_main(a):
    dev = torch.device("cuda", torch.cuda.current_device())
    xa = synthetic.activation_t3(a.M, a.K, seed=a.seed, device=dev)
    xw = synthetic.llm_weight(a.N, a.K, seed=a.seed + 1, device=dev)
    oa = fp4q.mma_operand(fp4q.quantize(xa, a.a_fmt, want_mse=False), a.a_fmt)
    ow = fp4q.mma_operand(fp4q.quantize(xw, a.w_fmt, want_mse=False), a.w_fmt)
    del xa, xw
    y = torch.empty(a.M, a.N, dtype=torch.bfloat16, device=dev)
    flush = None if a.no_flush else torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    for _ in range(a.warmup):
        fp4q.gemm(oa, ow, out=y)
    torch.cuda.synchronize()
    times = []
    for _ in range(a.iters):
        if flush is not None:
            flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fp4q.gemm(oa, ow, out=y)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    med = statistics.median(times)
    passes = oa.nplanes * ow.nplanes
    useful = 2.0 * a.M * a.N * a.K / (med / 1e3) / 1e12
    peak, kind = fp4_peak_tflops()
    print(json.dumps({
        "op": "gemm", "a_fmt": a.a_fmt, "w_fmt": a.w_fmt, "M": a.M, "N": a.N, "K": a.K, "passes": passes,
        "l2_flushed": flush is not None, "ms_median": med, "ms_min": min(times),
        "useful_tflops": useful, "tensor_tflops": useful * passes, "fp4_peak_tflops": peak, "peak_kind": kind,
        "tensor_frac": useful * passes / peak,
    }), flush=True)
    return 0


if __name__ == "__main__":
    main()
