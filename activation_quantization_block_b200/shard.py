"""One tensor split by rows over the ranks of a process group.

Blocks and rotation groups run along rows, so the rows of a tensor quantize
independently except for two quantities of the whole tensor: the tensor scale
s_t of the NVFP4 formats (from the tensor's absolute maximum, RaZeR sect. 1)
and the mean squared error.  ``quantize_row_sharded`` exchanges exactly those:

1. each rank computes the s_t of its own rows (``fp4q_tensor_scale``), and an
   all-reduce(MAX) gives the whole tensor's s_t -- s_t is a correctly rounded
   division of the absmax by a positive constant, hence monotone, so the
   largest per-rank s_t is the s_t of the largest absmax;
2. each rank quantizes its rows with that scale given: its codes and scales are
   the rows of the whole tensor quantized on one device, bit for bit;
3. an all-reduce(SUM) of (squared-error sum, element count) gives the MSE, equal
   to the single-device MSE up to the fp64 rounding of the partial sums.

The collectives run on the tensors' device (NCCL on GPUs); everything else is
the C ABI.  A rank whose local call fails still takes part in every exchange
and reports the failure inside the reduced tensor, so every rank raises after
the last exchange instead of one rank leaving the others waiting.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import fp4q


def _world(group) -> int:
    if not (dist.is_available() and dist.is_initialized()):
        return 1
    return dist.get_world_size(group)


def quantize_row_sharded(x_local: torch.Tensor, fmt="nvfp4_razer", rotate: bool = False, want_mse: bool = True,
                         group=None) -> fp4q.Quantized:
    """Quantize this rank's rows of a tensor split by rows over ``group``.

    Every rank of the group calls this with its own rows (any count, zero
    included; the same cols, fmt and rotate everywhere).  Returns this rank's
    codes and scales, the whole tensor's s_t (float32 [1]; zero for MXFP4) and,
    with want_mse, the whole tensor's MSE (float64 [1]); the same s_t and MSE on
    every rank.  Raises on every rank if the local call failed on any rank."""
    f = fp4q._fmt(fmt)
    exchange = _world(group) > 1
    dev = x_local.device
    local_error = None

    # Step 1: s_t of the whole tensor.
    ts = torch.zeros(1, dtype=torch.float32, device=dev)
    if f != fp4q.MXFP4:
        try:
            fp4q.tensor_scale(x_local, f, rotate, out=ts)
        except Exception as e:  # reported to the group in step 3
            local_error = e
        if exchange:
            dist.all_reduce(ts, op=dist.ReduceOp.MAX, group=group)

    # Step 2: this rank's rows with the scale given.
    q = None
    if local_error is None:
        try:
            q = fp4q.quantize(x_local, f, rotate, tensor_scale=ts if f != fp4q.MXFP4 else None, want_mse=want_mse)
        except Exception as e:
            local_error = e

    # Step 3: error sum, element count and failed ranks, summed over the group.
    tail = torch.zeros(3, dtype=torch.float64, device=dev)
    n_local = x_local.shape[0] * x_local.shape[1] if x_local.dim() == 2 else 0
    if q is not None and q.mse is not None:
        tail[0:1] = q.mse * float(n_local)
    tail[1] = float(n_local)
    tail[2] = 0.0 if local_error is None else 1.0
    if exchange:
        dist.all_reduce(tail, op=dist.ReduceOp.SUM, group=group)
    sse, count, n_failed = tail.tolist()
    if local_error is not None:
        raise RuntimeError("quantize_row_sharded: the local call failed") from local_error
    if n_failed:
        raise RuntimeError(f"quantize_row_sharded: the local call failed on {int(n_failed)} other rank(s)")
    mse = None
    if want_mse:
        mse = torch.full((1,), sse / count if count > 0 else 0.0, dtype=torch.float64, device=dev)
    return fp4q.Quantized(q.codes, q.scales, ts, mse)
