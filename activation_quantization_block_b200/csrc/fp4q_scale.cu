// The tensor scale of an NVFP4 format on its own (fp4q_tensor_scale).
//
// fp4q_quantize computes s_t inside its quantize pass, from the per-CTA maxima
// of the absmax pass.  A tensor split by rows over several devices needs s_t
// before any part is quantized: each part runs the absmax pass, this kernel
// reduces the part's maxima to its s_t, the parts exchange the maximum, and
// each part quantizes with the scale given.  The reduction and the division
// are the quantize kernel's own (block_max over the same partials, then
// tensor_scale_of), so a part that is the whole tensor gets the same s_t bits
// that fp4q_quantize writes.
//
// Method reference: "RaZeR: Pushing the Limits of NVFP4 Quantization with
// Redundant Zero Remapping", sect. 1 (scales derived from the tensors'
// absolute maxima).
#include <cuda_runtime.h>

#include <cstdint>

#include "fp4q_launch.cuh"
#include "fp4q_scale.h"

namespace fp4q {

namespace {

// One CTA: s_t from the n per-CTA maxima the absmax pass wrote.
template <int FMT>
__global__ void __launch_bounds__(kThreads) tensor_scale_kernel(const float* partials, int n, float* tensor_scale,
                                                                unsigned* err)
{
    __shared__ float sh[32];
    pdl_wait();
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += kThreads)
        if (in_bounds(4 * (int64_t)i, 4, 4 * (int64_t)kMaxPartials, kSiteAmaxPartialLoad, err))
            m = fmaxf(m, partials[i]);
    m = block_max(m, sh);
    if (threadIdx.x == 0) *tensor_scale = tensor_scale_of<FMT>(m);
}

}  // namespace

cudaError_t launch_tensor_scale(const float* partials, int n, int fmt, float* tensor_scale, cudaStream_t st)
{
    unsigned* err = device_error_words();
    if (err == nullptr) return cudaErrorInvalidSymbol;
    switch (fmt) {
        case kNV: return launch(tensor_scale_kernel<kNV>, 1, 0, true, st, partials, n, tensor_scale, err);
        case kRZ: return launch(tensor_scale_kernel<kRZ>, 1, 0, true, st, partials, n, tensor_scale, err);
        case kRW: return launch(tensor_scale_kernel<kRW>, 1, 0, true, st, partials, n, tensor_scale, err);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fp4q
