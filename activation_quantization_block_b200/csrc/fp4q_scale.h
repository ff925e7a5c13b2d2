// Interface of fp4q_scale.cu to the C ABI layer (fp4q_api.cu).  Not installed;
// not part of the ABI.
#pragma once

#include <cuda_runtime.h>

namespace fp4q {

// One-CTA kernel: *tensor_scale = s_t of an NVFP4 format (fmt 0, 1 or 3) from
// the n per-CTA maxima written by launch_amax, the same reduction and division
// as the quantize kernel.  Launched with programmatic dependent launch after
// the absmax pass; it waits for that pass before reading the maxima.
cudaError_t launch_tensor_scale(const float* partials, int n, int fmt, float* tensor_scale, cudaStream_t st);

}  // namespace fp4q
