"""fp4q: block-scaled 4-bit quantization (NVFP4, NVFP4 with RaZeR, MXFP4) for B200."""
