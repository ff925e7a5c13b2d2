"""Throughput of block-scaled 4-bit quantization on B200.

One step quantizes a Llama-3-8B-shaped weight set -- 32 layers x {q 4096x4096,
k 1024x4096, v 1024x4096, o 4096x4096, gate 14336x4096, up 14336x4096,
down 4096x14336}, bf16 N(0, 0.02^2) with 0.1 % outliers x20 -- to NVFP4 with
RaZeR remapping (no rotation), each tensor with its own computed tensor scale
and its MSE, through the C ABI, back to back on one stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fp4q|reference]

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on the
host cores on a bounded row sample of the same workload instead.  With N > 1
(launched by torch.distributed.run) every rank quantizes its own weight set
(weak scaling, no collective on the data path); the time is the maximum over
ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantize+pack elements/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "elements/s"
FMT = "nvfp4_razer"
BYTES_PER_ELEMENT = 4.5625       # computed tensor scale: absmax read 2 + read 2 + codes 0.5 + scales 1/16
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
WORKLOAD = ("llama3-8b weight set: 32 layers x {q 4096x4096, k 1024x4096, v 1024x4096, o 4096x4096, "
            "gate 14336x4096, up 14336x4096, down 4096x14336} bf16 N(0,0.02^2) + 0.1% outliers x20, seed 2; "
            "NVFP4_RAZER, rotate 0, per-tensor computed scale, fused MSE")


def set_format(fmt: str):
    """Run the same workload in another NVFP4 format (the default is the headline's)."""
    global FMT, WORKLOAD
    if fmt != FMT:
        WORKLOAD = WORKLOAD.replace(FMT.upper(), fmt.upper())
        FMT = fmt


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["fp4q", "reference"], default="fp4q")
    p.add_argument("--layers", type=int, default=32, help="layers in the weight set (32 = the full 8B model)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workloads (2048^2 weight, activations, 70B MLP, dequantize sweep)")
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--fmt", choices=["nvfp4_razer", "nvfp4", "nvfp4_razer_w"], default=FMT,
                   help="format of the run (all three read 4.5625 B/element with the computed tensor scale)")
    p.add_argument("--mode", choices=["batch", "per-call"], default="batch",
                   help="batch: fp4q_quantize_batch over 16 layers (112 tensors) per call; "
                        "per-call: one fp4q_quantize per tensor")
    return p.parse_args()


def layer_shapes():
    from activation_quantization_block_b200 import synthetic
    return synthetic.LLAMA3_8B_LAYER


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# The translation units the measured kernels are built from: a traffic record
# stays valid until one of these files changes.
TRAFFIC_SOURCES = {
    "quantize_batch": ("fp4q_batch.cu", "fp4q_launch.cuh", "fp4q_common.cuh", "fp4q_device.cuh", "fp4q_tma.cuh",
                       "fp4q_internal.h"),
    "quantize": ("fp4q_kernels.cu", "fp4q_launch.cuh", "fp4q_common.cuh", "fp4q_device.cuh", "fp4q_tma.cuh",
                 "fp4q_internal.h"),
}


def kernel_source_sha256(kernel_key: str) -> str:
    from activation_quantization_block_b200 import _build
    import hashlib
    files = TRAFFIC_SOURCES["quantize_batch" if kernel_key.startswith("quantize_batch") else "quantize"]
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(_build.CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_record(kernel_key: str):
    """DRAM bytes per element from the committed ncu capture, if it was taken on the kernel's current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(kernel_key)
    if not entry or entry.get("source_sha256") != kernel_source_sha256(kernel_key):
        return None
    return float(entry["dram_bytes_per_element"])


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="fp4q_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return summarize_clock_lines(lines)


def summarize_clock_lines(lines):
    """Median SM clock, the largest max clock and every throttle reason seen Active, from
    nvidia-smi CSV lines in ClockSampler.FIELDS order."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) >= 9:
            rows.append(parts)
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
    mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle legs

def oracle_sample(layer: int, frac_rows: int = 32):
    """Host bf16 row slices (1/frac_rows of the rows of every tensor of one layer)."""
    from activation_quantization_block_b200 import synthetic
    out = []
    for i, (name, r, c) in enumerate(layer_shapes()):
        rows = max(1, r // frac_rows)
        x = synthetic.llm_weight(r, c, seed=synthetic.tensor_seed(2, layer, i), device="cpu")
        out.append(synthetic.bf16_bits(x[:rows]))
    return out


def time_oracle(samples, nthreads):
    import oracle
    t0 = time.perf_counter()
    n = 0
    for xb in samples:
        oracle.quantize(xb, FMT, False, want_sse=True, nthreads=nthreads)
        n += xb.size
    return n, time.perf_counter() - t0


def cpu_baseline_leg(layer0=None):
    """The oracle as it stands, on every host core, over one full layer (218 M elements).

    ``layer0``: the GPU's own layer-0 inputs and results, copied to the host after the
    timed region, as (x bf16 bits, codes, scales, tensor scale, mse) per tensor.  The
    oracle then quantizes exactly those input bytes, and its results are compared
    with the GPU's: codes, scales and tensor scales bit for bit, the MSE to its
    relative difference.  Returns (cpu_baseline, parity or None)."""
    import numpy as np
    import oracle
    from activation_quantization_block_b200 import synthetic
    nthreads = oracle.default_threads()
    if layer0 is None:
        layer0 = [(synthetic.bf16_bits(synthetic.llm_weight(r, c, seed=synthetic.tensor_seed(2, 0, i))),)
                  for i, (name, r, c) in enumerate(layer_shapes())]
    n, results = 0, []
    t0 = time.perf_counter()
    for item in layer0:
        results.append(oracle.quantize(item[0], FMT, False, want_sse=True, nthreads=nthreads))
        n += item[0].size
    dt = time.perf_counter() - t0
    base = {"value": n / dt, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": f"one full layer of the weight set (7 tensors, {n} elements), {dt:.2f} s wall, "
                      f"computed tensor scale + MSE, {nthreads} threads"
                      + (", on the GPU's own input bytes" if len(layer0[0]) > 1 else "")}
    if len(layer0[0]) == 1:
        return base, None
    codes_ok, scales_ok, ts_ok, mse_rel = True, True, True, 0.0
    for (xb, codes, scales, ts, mse), (rc, rs, rts, rsse) in zip(layer0, results):
        codes_ok = codes_ok and bool(np.array_equal(codes, rc))
        scales_ok = scales_ok and bool(np.array_equal(scales, rs))
        ts_ok = ts_ok and bool(np.float32(ts) == np.float32(rts))
        ref = rsse / xb.size
        mse_rel = max(mse_rel, abs(mse - ref) / ref if ref > 0 else abs(mse))
    parity = {"layer0_codes_scales_equal": codes_ok and scales_ok, "codes_equal": codes_ok,
              "scales_equal": scales_ok, "tensor_scales_equal": ts_ok, "mse_max_rel": mse_rel,
              "mse_tolerance": 1e-5, "tensors": len(layer0), "elements": n,
              "how": "the oracle on the GPU's layer-0 input bytes (copied from the device after the timed "
                     "region); codes, scales and tensor scales compared bit for bit, the MSE relatively"}
    return base, parity


# ---------------------------------------------------------------- multi-rank host logic

def rank_layer_seed(layer: int, rank: int, layers: int) -> int:
    """Layer index used for the seeds of rank `rank`'s copy of the weight set: every rank
    quantizes its own set (weak scaling), disjoint from the others'."""
    return layer + rank * layers


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The job's time: the maximum of the ranks' device-timed values (all_reduce MAX)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(elements_per_rank: int, world: int, steps: int, ms: float) -> float:
    """Whole-job elements/s: the units all ranks processed over the (max-over-ranks) time."""
    return elements_per_rank * world * steps / (ms / 1e3)


def sha256_of(tensors) -> str:
    """SHA-256 over the bytes of the given tensors in order (copied to the host); a failure is
    reported in the string instead of ending the run."""
    import hashlib

    import torch
    try:
        h = hashlib.sha256()
        for t in tensors:
            flat = t.detach().contiguous().reshape(-1)
            h.update(flat.view(torch.uint8).cpu().numpy().tobytes())
        return h.hexdigest()
    except Exception as e:  # the digest is a label, not a measurement
        return f"unavailable: {type(e).__name__}: {e}"


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    nthreads = oracle.default_threads()
    # each step: 1/8 of the rows of every tensor of one layer (about 27 M elements)
    pool = [oracle_sample(0, frac_rows=8)]
    for s in range(args.warmup):
        time_oracle(pool[s % len(pool)], nthreads)
    tot_n, tot_t = 0, 0.0
    for s in range(args.steps):
        n, dt = time_oracle(pool[s % len(pool)], nthreads)
        tot_n += n
        tot_t += dt
    value = tot_n / tot_t
    per_step = tot_n / args.steps
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": "1/8 of the rows of each tensor of layer 0 per step",
                   "elements_per_step": per_step},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": f"{per_step:.0f} elements per step (1/8 of every tensor's rows of layer 0), "
                                   f"{nthreads} threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- the other workloads

CONFIG_REPEATS = 20
FLUSH_BYTES = 256 << 20     # written before every timed call: more than the 126 MB L2


def time_device(fn, flush, repeats=CONFIG_REPEATS, warmup=3):
    """Median and minimum device time (us) of fn() over `repeats` calls, each preceded by a
    write of a buffer larger than L2 (outside the timed pair of events).  The flush also
    keeps the GPU busy while the host enqueues the call, so the events time the device."""
    import torch
    for _ in range(warmup):
        fn()
    ts = []
    for _ in range(repeats):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    us = sorted(1e3 * a.elapsed_time(b) for a, b in ts)
    return statistics.median(us), us[0]


def oracle_rates(xb, fmt, rotate, op="quantize", packed=None):
    """The oracle's elements/s on host bf16 bits (quantize) or packed inputs (dequantize), on one
    thread and on every core."""
    import oracle
    out = {}
    for label, nt in (("oracle_1t", 1), ("oracle_nt", oracle.default_threads())):
        t0 = time.perf_counter()
        if op == "quantize":
            oracle.quantize(xb, fmt, rotate, want_sse=True, nthreads=nt)
            n = xb.size
        else:
            codes, scales, ts = packed
            oracle.dequantize(codes, scales, ts, fmt, rotate, nthreads=nt)
            n = codes.size * 2
        out[label] = {"elements_per_s": n / (time.perf_counter() - t0), "threads": nt, "elements": n}
    return out


def measure_configs(dev, peak, with_oracle=True):
    """Every other workload of the benchmark suite, each call timed alone (median of 20, L2
    flushed before each): throughput, algorithmic GB/s and its fraction of the copy
    bandwidth, the MSE, and the oracle's rates on the host cores (one thread on a row
    slice, all cores on the stated slice).  The two small workloads also report the fixed
    cost of a call (the same call on a 128 x 64 tensor) and its share of their time."""
    import torch
    from activation_quantization_block_b200 import fp4q, synthetic
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = []

    def quant_entry(name, x, fmt, rotate, slice_rows, tiny_us=None):
        rows, cols = x.shape
        q = fp4q.empty_like_quantized(x, fmt)
        ws = torch.zeros(fp4q.fp4q_workspace_size(rows, cols, fmt, rotate), dtype=torch.uint8, device=dev)

        def call():
            st = fp4q.fp4q_quantize(x, rows, cols, cols, fmt, rotate, 0, q.codes, q.scales, q.tensor_scale,
                                    q.mse, ws, ws.numel())
            if st != 0:
                raise fp4q.Fp4qError(st, "fp4q_quantize")
        med, best = time_device(call, flush)
        n = x.numel()
        B = fp4q.block_size(fmt)
        nbytes = 2 * n + n // 2 + n // B + (2 * n if fmt != "mxfp4" else 0)
        e = {"workload": name, "op": "quantize", "format": fmt, "rotate": rotate, "shape": [rows, cols],
             "elements": n, "us_median": med, "us_min": best, "elements_per_s": n / (med / 1e6),
             "alg_bytes": nbytes, "gbs": nbytes / (med / 1e6) / 1e9, "frac": nbytes / (med / 1e6) / 1e9 / peak,
             "mse": float(q.mse.item())}
        if tiny_us is not None:
            e["call_overhead_us"] = tiny_us
            e["call_overhead_share"] = min(1.0, tiny_us / med)
        if with_oracle:
            xb = synthetic.bf16_bits(x[:slice_rows])
            e.update(oracle_rates(xb, fmt, bool(rotate)))
            e["oracle_slice_rows"] = slice_rows
        out.append(e)

    def tiny_call_us(fmt, rotate):
        x = synthetic.llm_weight(128, 64, seed=9, device=dev)
        q = fp4q.empty_like_quantized(x, fmt)
        ws = torch.zeros(fp4q.fp4q_workspace_size(128, 64, fmt, rotate), dtype=torch.uint8, device=dev)
        return time_device(lambda: fp4q.fp4q_quantize(x, 128, 64, 64, fmt, rotate, 0, q.codes, q.scales,
                                                      q.tensor_scale, q.mse, ws, ws.numel()), flush)[0]

    # 2048 x 2048 LLM weight, NVFP4 and NVFP4_RAZER
    x = synthetic.llm_weight(2048, 2048, seed=0, device=dev)
    for fmt in ("nvfp4", "nvfp4_razer"):
        quant_entry("2048x2048 llm weight N(0,0.02^2)+0.1% outliers x20, seed 0", x, fmt, 0, 2048,
                    tiny_us=tiny_call_us(fmt, 0))
    # 8192 x 4096 activations, MXFP4 with and without rotation
    x = synthetic.activation_t3(8192, 4096, seed=1, device=dev)
    for rot in (0, 1):
        quant_entry("8192x4096 activations, column LogNormal(0,1) x Student-t(3), seed 1", x, "mxfp4", rot,
                    512 if rot else 8192, tiny_us=tiny_call_us("mxfp4", rot))
    del x
    # 70B MLP block, NVFP4 / NVFP4_RAZER / MXFP4 + rotation
    for i, (pname, r, c) in enumerate(synthetic.LLAMA3_70B_MLP):
        x = synthetic.mlp_row_scaled(r, c, seed=synthetic.tensor_seed(3, 0, i), device=dev)
        for fmt, rot in (("nvfp4", 0), ("nvfp4_razer", 0), ("mxfp4", 1)):
            quant_entry(f"70B MLP {pname} {r}x{c}, row LogNormal(0,0.5) x N(0,0.015^2), seed 3", x, fmt, rot,
                        256 if rot else 1024)
        del x
    torch.cuda.empty_cache()
    # dequantize sweep 8192 x N
    for N in (4096, 14336, 28672, 57344):
        for fmt in ("nvfp4_razer", "mxfp4"):
            codes, scales, ts = synthetic.random_packed(8192, N, fmt, seed=4, device=dev)
            y = torch.empty(8192, N, dtype=torch.bfloat16, device=dev)

            def call():
                st = fp4q.fp4q_dequantize(codes, scales, ts, 8192, N, fmt, 0, y, N)
                if st != 0:
                    raise fp4q.Fp4qError(st, "fp4q_dequantize")
            med, best = time_device(call, flush)
            n = 8192 * N
            nbytes = n // 2 + n // fp4q.block_size(fmt) + 2 * n
            e = {"workload": f"dequantize sweep 8192x{N}, random codes and valid scales, seed 4", "op": "dequantize",
                 "format": fmt, "rotate": 0, "shape": [8192, N], "elements": n, "us_median": med, "us_min": best,
                 "elements_per_s": n / (med / 1e6), "alg_bytes": nbytes, "gbs": nbytes / (med / 1e6) / 1e9,
                 "frac": nbytes / (med / 1e6) / 1e9 / peak}
            if with_oracle and N == 4096:
                e.update(oracle_rates(None, fmt, False, op="dequantize",
                                      packed=(codes[:1024].cpu().numpy(), scales[:1024].cpu().numpy(), 1.0)))
                e["oracle_slice_rows"] = 1024
            out.append(e)
            del codes, scales, y
    del flush
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- GPU arm

def main():
    args = parse()
    set_format(args.fmt)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from activation_quantization_block_b200 import fp4q, synthetic

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    # ---- workload, resident in HBM -------------------------------------------------
    tensors = []
    for layer in range(args.layers):
        for i, (name, r, c) in enumerate(layer_shapes()):
            seed = synthetic.tensor_seed(2, rank_layer_seed(layer, rank, args.layers), i)
            x = synthetic.llm_weight(r, c, seed=seed, device=dev)
            q = fp4q.Quantized(torch.empty(r, c // 2, dtype=torch.uint8, device=dev),
                               torch.empty(r, c // 16, dtype=torch.uint8, device=dev),
                               torch.zeros(1, dtype=torch.float32, device=dev),
                               torch.zeros(1, dtype=torch.float64, device=dev))
            tensors.append((name, x, q))
    torch.cuda.synchronize()
    elements = sum(x.numel() for _, x, _ in tensors)
    layer0 = len(layer_shapes())
    inputs_sha = sha256_of([x for _, x, _ in tensors[:layer0]])
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    ws = torch.zeros(fp4q.fp4q_workspace_size(0, 0, FMT, 0), dtype=torch.uint8, device=dev)
    L = fp4q.lib()
    fmt = fp4q.FORMATS[FMT]
    if args.mode == "per-call":
        calls = [(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), q.codes.data_ptr(), q.scales.data_ptr(),
                  q.tensor_scale.data_ptr(), q.mse.data_ptr(), x.numel()) for _, x, q in tensors]
        launches_per_call = 3   # absmax, quantize, mse finaliser
        call_elements = [c[-1] for c in calls]
        kernel_desc = "fp4q_quantize call: absmax pass + quantize pass + mse finaliser"

        def one_call(k):
            xp, r, c, ld, cp, sp, tp, mp, n = calls[k]
            st = L.fp4q_quantize(xp, r, c, ld, fmt, 0, 0, cp, sp, tp, mp, ws.data_ptr(), ws.numel(), sh)
            if st != 0:
                raise fp4q.Fp4qError(st, "fp4q_quantize")
    else:
        groups = [tensors]                      # the whole weight set in one call
        descs = [fp4q._descs([fp4q.tensor_desc(x, q) for _, x, q in g]) for g in groups]
        ws_need = max(fp4q.fp4q_batch_workspace_size(len(g), d, FMT, 0) for g, d in zip(groups, descs))
        bws = torch.empty(ws_need, dtype=torch.uint8, device=dev)
        calls = list(range(len(groups)))
        launches_per_call = len(tensors) + 2    # one chained kernel per tensor, plus the first and last
        call_elements = [sum(x.numel() for _, x, _ in g) for g in groups]
        kernel_desc = ("fp4q_quantize_batch over the weight set: chain of persistent kernels, each the absmax "
                       "pass of one tensor interleaved with the quantize pass of the previous (PDL-chained); "
                       "per-launch figures = call totals / launches")

        def one_call(k):
            st = L.fp4q_quantize_batch(len(groups[k]), descs[k], fmt, 0, 0, bws.data_ptr(), bws.numel(), sh)
            if st != 0:
                raise fp4q.Fp4qError(st, "fp4q_quantize_batch")

    def step(events=None):
        for k in range(len(calls)):
            if events is not None:
                events[2 * k].record(stream)
            one_call(k)
            if events is not None:
                events[2 * k + 1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(calls))] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for s in range(args.steps):
        step(ev[s])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    ms_per_step = ms / args.steps
    value = job_throughput(elements, world, args.steps, ms)

    # per-call durations -> roofline of the call (its launches run back to back on the stream)
    call_ms = [ev[s][2 * k].elapsed_time(ev[s][2 * k + 1]) for s in range(args.steps) for k in range(len(calls))]
    avg_call_ms = statistics.mean(call_ms)
    avg_call_bytes = BYTES_PER_ELEMENT * statistics.mean(call_elements)
    peak, peak_kind = peaks()
    achieved = avg_call_bytes / (avg_call_ms / 1e3) / 1e9
    dram_bpe = traffic_record(f"quantize_batch_{FMT}_sse" if args.mode == "batch" else f"quantize_{FMT}_sse")
    roofline = {"bound": "hbm", "kernel": kernel_desc,
                "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "peak_kind": f"{peak_kind} copy bandwidth",
                "traffic": (dram_bpe * statistics.mean(call_elements)) if dram_bpe else None,
                "algorithmic_bytes_per_launch": avg_call_bytes, "avg_launch_ms": avg_call_ms}

    # ---- check a result, outside the timed region ---------------------------------
    mses = torch.cat([q.mse for _, _, q in tensors]).cpu()
    outputs_sha = sha256_of([t for _, _, q in tensors[:layer0] for t in (q.codes, q.scales)])
    assert torch.isfinite(mses).all() and (mses > 0).all()
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    host_layer0 = None
    if want_cpu:   # the GPU's own layer-0 bytes and results, for the oracle leg
        host_layer0 = [(synthetic.bf16_bits(x), q.codes.cpu().numpy(), q.scales.cpu().numpy(),
                        float(q.tensor_scale.item()), float(q.mse.item())) for _, x, q in tensors[:layer0]]

    # ---- end to end from pinned host memory -------------------------------------------
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, tensors, fmt, L, dev, world)

    del tensors
    torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "elements_per_step": elements * world, "layers": args.layers,
                   "api": "fp4q_quantize_batch, one call per step" if args.mode == "batch" else
                          "fp4q_quantize, one call per tensor",
                   "parallelism": f"dp{world} (independent weight sets, no collective)" if world > 1 else "1 GPU",
                   "l2": f"no flush: each step reads {elements * 2 / 1e9:.2f} GB of inputs (> 126 MB L2)",
                   "inputs_sha256": f"layer 0 of rank 0, 7 bf16 tensors in order: {inputs_sha}"},
        "outputs_sha256": f"layer 0 of rank 0, codes then scales of each tensor: {outputs_sha}",
        "achieved_gbs": BYTES_PER_ELEMENT * elements * world / (ms_per_step / 1e3) / 1e9,
        "pct_of_nominal_8tbs": 100 * BYTES_PER_ELEMENT * elements / (ms_per_step / 1e3) / 1e9 / NOMINAL_HBM_GBS,
        "roofline": roofline,
        "clocks": clocks,
        "gpu_launches": launches_per_call * len(calls) * args.steps,
        "e2e": e2e,
    }
    if want_cpu:
        line["cpu_baseline"], line["parity"] = cpu_baseline_leg(host_layer0)
    if rank == 0 and world == 1 and not args.no_configs:
        line["configs"] = measure_configs(dev, peak, with_oracle=not args.no_cpu_baseline)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, tensors, fmt, L, dev, world=1):
    """Same metric from pinned host buffers: every step copies each group of
    tensors in (one layer in batch mode, one tensor per call otherwise),
    quantizes it and copies codes, scales, tensor scales and MSEs back; copies
    of one group overlap the kernels of the other (two buffer sets, 3 streams).
    With several ranks the job's value is all ranks' elements over the slowest
    rank's time, and the bytes are all ranks' copies."""
    import torch
    from activation_quantization_block_b200 import fp4q
    per = len(layer_shapes()) if args.mode == "batch" else 1
    groups = [list(range(i, min(i + per, len(tensors)))) for i in range(0, len(tensors), per)]
    host_in = []
    for _, x, _ in tensors:
        h = torch.empty(x.shape, dtype=torch.bfloat16, pin_memory=True)
        h.copy_(x)
        host_in.append(h)
    host_out = [fp4q.Quantized(torch.empty(q.codes.shape, dtype=torch.uint8, pin_memory=True),
                               torch.empty(q.scales.shape, dtype=torch.uint8, pin_memory=True),
                               torch.empty(1, dtype=torch.float32, pin_memory=True),
                               torch.empty(1, dtype=torch.float64, pin_memory=True)) for _, _, q in tensors]
    # two buffer sets, each holding one group's inputs and outputs (by position in the group)
    shapes = [[tensors[k][1].shape for k in g] for g in groups]
    biggest = max(range(len(groups)), key=lambda i: sum(s[0] * s[1] for s in shapes[i]))
    bufs = []
    for _ in range(2):
        xs = [torch.empty(sh, dtype=torch.bfloat16, device=dev) for sh in shapes[biggest]]
        qs = [fp4q.empty_like_quantized(x, FMT) for x in xs]
        bufs.append((xs, qs))
    ws_bytes = max(fp4q.fp4q_batch_workspace_size(len(g), [fp4q.tensor_desc(x, q) for x, q in zip(*bufs[0])][:len(g)],
                                                  FMT, 0) for g in groups)
    ws_bytes = max(ws_bytes, fp4q.fp4q_workspace_size(0, 0, FMT, 0))
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    h2d, comp, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_free = [torch.cuda.Event() for _ in range(2)]
    for e in out_free:
        e.record(d2h)
    for e in comp_done:
        e.record(comp)

    def step():
        for gi, g in enumerate(groups):
            b = gi & 1
            xs, qs = bufs[b]
            h2d.wait_event(comp_done[b])          # buffer set b no longer read by an earlier call
            with torch.cuda.stream(h2d):
                for j, k in enumerate(g):
                    xs[j].copy_(host_in[k], non_blocking=True)
                in_ready[b].record(h2d)
            comp.wait_event(in_ready[b])
            comp.wait_event(out_free[b])          # outputs of set b copied out by an earlier D2H
            if args.mode == "batch":
                d = fp4q._descs([fp4q.tensor_desc(xs[j], qs[j]) for j in range(len(g))])
                st = L.fp4q_quantize_batch(len(g), d, fmt, 0, 0, ws.data_ptr(), ws.numel(), comp.cuda_stream)
            else:
                x, q = xs[0], qs[0]
                st = L.fp4q_quantize(x.data_ptr(), x.shape[0], x.shape[1], x.shape[1], fmt, 0, 0, q.codes.data_ptr(),
                                     q.scales.data_ptr(), q.tensor_scale.data_ptr(), q.mse.data_ptr(), ws.data_ptr(),
                                     ws.numel(), comp.cuda_stream)
            if st != 0:
                raise fp4q.Fp4qError(st, "quantize")
            comp_done[b].record(comp)
            d2h.wait_event(comp_done[b])
            with torch.cuda.stream(d2h):
                for j, k in enumerate(g):
                    ho = host_out[k]
                    ho.codes.copy_(qs[j].codes, non_blocking=True)
                    ho.scales.copy_(qs[j].scales, non_blocking=True)
                    ho.tensor_scale.copy_(qs[j].tensor_scale, non_blocking=True)
                    ho.mse.copy_(qs[j].mse, non_blocking=True)
                out_free[b].record(d2h)

    step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(h2d)
    for _ in range(args.e2e_steps):
        step()
    t1.record(d2h)     # the last D2H is ordered after every copy and kernel of the steps
    torch.cuda.synchronize()
    dt = max_over_ranks(t0.elapsed_time(t1), world, dev) / 1e3 / args.e2e_steps
    elements = sum(h.numel() for h in host_in) * world
    h2d_bytes = 2 * elements
    d2h_bytes = sum(o.codes.numel() + o.scales.numel() + 4 + 8 for o in host_out) * world
    # the host copies equal the device results
    ok = all(torch.equal(host_out[k].codes, tensors[k][2].codes.cpu()) for k in (0, len(tensors) - 1))
    return {"value": elements / dt, "unit": UNIT, "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes, "ms_per_step": dt * 1e3, "steps": args.e2e_steps,
            "path": ("pinned host bf16 -> H2D -> fp4q_quantize_batch per layer" if args.mode == "batch" else
                     "pinned host bf16 -> H2D -> fp4q_quantize per tensor") +
                    " -> D2H codes/scales/scale/mse; two buffer sets, 3 streams",
            "matches_device_results": bool(ok)}


if __name__ == "__main__":
    sys.exit(main())
