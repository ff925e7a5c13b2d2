"""Offline choice of the second special-value pair of the RaZeR weight mode.

"RaZeR: Pushing the Limits of NVFP4 Quantization with Redundant Zero
Remapping", technical summary sect. 2.2: with the two bits an E3M3 block scale
frees, weights choose per block among four special values -- two pairs fixed
offline, each a multiple of 0.5; the pair +-5 is the best single pair.  The
paper does not name the second pair.  This script finds it the way the paper
describes: over every multiple of 0.5 that is not already an E2M1 value (nor 5)
up to 8, it quantizes a set of seeded synthetic LLM weight matrices in the
weight mode with {+-5, +-s2} and keeps the s2 with the lowest total squared
error.  It uses only the oracle.

    python -m oracle.razer_weight_pair
"""
from __future__ import annotations

import numpy as np

from activation_quantization_block_b200 import synthetic

from . import quantize, razer_w_pair, set_razer_w_pair

CANDIDATES = (2.5, 3.5, 4.5, 5.5, 6.5, 7.0, 7.5, 8.0)


def workload():
    """Seeded weight matrices of the two kinds the synthetic recipe defines."""
    mats = []
    for seed in range(4):
        mats.append(synthetic.llm_weight(1024, 4096, seed=100 + seed, device="cpu"))
    for seed in range(2):
        mats.append(synthetic.mlp_row_scaled(1024, 8192, seed=200 + seed, device="cpu"))
    return [synthetic.bf16_bits(m) for m in mats]


def total_sse(mats, s2: float) -> float:
    set_razer_w_pair(s2)
    return sum(quantize(x, "nvfp4_razer_w")[3] for x in mats)


def search() -> tuple[float, dict]:
    keep = razer_w_pair()
    mats = workload()
    try:
        table = {s2: total_sse(mats, s2) for s2 in CANDIDATES}
    finally:
        set_razer_w_pair(keep)
    best = min(table, key=table.get)
    return best, table


if __name__ == "__main__":
    best, table = search()
    for s2, e in table.items():
        print(f"s2 = {s2:4.1f}  total squared error {e:.6e}{'  <- best' if s2 == best else ''}")
