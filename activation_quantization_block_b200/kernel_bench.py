"""Time one fp4q operation on one seeded tensor.

    python -m activation_quantization_block_b200.kernel_bench --op quantize --fmt nvfp4_razer \\
        --rows 14336 --cols 4096 [--rotate] [--no-mse] [--scale-given] [--iters 20]

Each iteration is one C-ABI call on the current stream, timed with CUDA events;
between iterations a 512 MB buffer is overwritten so that no input stays in
L2 (--no-flush keeps them).  Prints one JSON line: median and minimum time
per call, elements/s and the call's algorithmic bytes per second
(quantize: 2 B read + codes and scales written, plus 2 B for the absmax read
when the tensor scale is computed; dequantize: codes and scales read + 2 B
written; error: 2 B + codes and scales read).
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

from . import fp4q, synthetic


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--op", choices=["quantize", "dequantize", "error"], default="quantize")
    p.add_argument("--fmt", choices=list(fp4q.FORMATS), default="nvfp4_razer")
    p.add_argument("--rows", type=int, default=14336)
    p.add_argument("--cols", type=int, default=4096)
    p.add_argument("--rotate", action="store_true")
    p.add_argument("--no-mse", action="store_true")
    p.add_argument("--scale-given", action="store_true")
    p.add_argument("--data", choices=["weight", "activation", "mlp"], default="weight")
    p.add_argument("--seed", type=int, default=2)
    p.add_argument("--iters", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--no-flush", action="store_true")
    a = p.parse_args(argv)

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
        flags = fp4q.FLAG_TENSOR_SCALE_GIVEN if a.scale_given else 0
        nbytes = 2 * n + packed + (0 if a.scale_given or a.fmt == "mxfp4" else 2 * n)

        def call():
            return fp4q.fp4q_quantize(x, a.rows, a.cols, a.cols, a.fmt, int(a.rotate), flags, q.codes, q.scales,
                                      q.tensor_scale, None if a.no_mse else mse, ws, ws.numel())
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
    print(json.dumps({
        "op": a.op, "fmt": a.fmt, "rotate": a.rotate, "mse": not a.no_mse, "scale_given": a.scale_given,
        "rows": a.rows, "cols": a.cols, "data": a.data, "l2_flushed": flush is not None,
        "ms_median": med, "ms_min": best, "elements_per_s": n / (med / 1e3),
        "algorithmic_bytes": nbytes, "gbs_median": nbytes / (med / 1e3) / 1e9, "gbs_best": nbytes / (best / 1e3) / 1e9,
    }), flush=True)


if __name__ == "__main__":
    main()
