"""fp4q: block-scaled 4-bit quantization (NVFP4, NVFP4 with RaZeR in its
activation and weight modes, MXFP4, optional 32-point Walsh-Hadamard rotation)
of bf16 matrices on NVIDIA B200 (sm_100a).

``fp4q`` holds the binding of the C ABI in ``include/fp4q.h``; ``shard``
quantizes one tensor split by rows over the ranks of a process group;
``synthetic`` holds seeded input generators.
"""
from .fp4q import (  # noqa: F401
    ABI_SYMBOLS, FORMATS, MXFP4, NVFP4, NVFP4_RAZER, NVFP4_RAZER_W, Fp4qError, Quantized, block_size, dequantize,
    error,
    fp4q_abi_version, fp4q_dequantize, fp4q_error, fp4q_quantize, fp4q_status_string, fp4q_workspace_size,
    lib, library_path, quantize, quantize_batch, fp4q_quantize_batch, fp4q_batch_workspace_size,
    MmaOperand, mma_operand, gemm, fp4q_mma_planes, fp4q_mma_sf_bytes, fp4q_mma_pack, fp4q_gemm,
    tensor_scale, fp4q_tensor_scale,
)
from .shard import quantize_row_sharded  # noqa: F401
