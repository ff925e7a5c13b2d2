// fp4q_quantize_noalloc: fp4q_quantize with its scratch memory inside the library.
//
// fp4q_quantize needs 48 KB of device scratch (per-CTA partial maxima and
// partial squared-error sums) and takes it from the caller as a workspace.
// Some callers cannot provide one: code that runs where it must not call
// cudaMalloc or any other allocator -- a plugin or extension inside a host
// program that owns all device memory (a serving engine that reserved the GPU
// up front, where a stray cudaMalloc fails or fragments the pool), or a
// latency-critical path that cannot afford the device-wide synchronisation a
// cudaMalloc / cudaFree can imply.  This entry point serves them: its scratch
// is a file-scope device array that the CUDA module loader places on every
// GPU that loads this library, so the call itself allocates nothing.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp4q.h"
#include "fp4q_internal.h"

namespace {

// The scratch: FP4Q_NOALLOC_SCRATCH_BYTES bytes on every device that loads the
// library, held until the process exits.  Nothing in it needs to start at zero:
// every call writes each partial slot before any thread reads it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FP4Q_NOALLOC_SCRATCH_BYTES];

static_assert(FP4Q_NOALLOC_SCRATCH_BYTES >= fp4q::kWorkspaceBytes,
              "the static scratch must hold the quantize workspace");

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];   // device address of g_noalloc_scratch, per device

// Host code cannot pass g_noalloc_scratch to a kernel: on the host that name is
// a stand-in, not a device address.  Look the address up once per device, with
// that device current.
fp4q_status_t scratch_address(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return FP4Q_ERROR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return FP4Q_ERROR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return FP4Q_ERROR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FP4Q_SUCCESS;
}

}  // namespace

extern "C" fp4q_status_t fp4q_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                               fp4q_format_t fmt, int rotate, uint32_t flags,
                                               uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                               double* mse, fp4q_stream_t stream)
{
    if (fp4q_workspace_size(rows, cols, fmt, rotate) > sizeof(g_noalloc_scratch))
        return FP4Q_ERROR_WORKSPACE;   // this shape needs more scratch than the static array holds
    void* scratch = nullptr;
    fp4q_status_t s = scratch_address(&scratch);
    if (s != FP4Q_SUCCESS) return s;
    return fp4q_quantize(x, rows, cols, ldx, fmt, rotate, flags, codes, scales, tensor_scale, mse,
                         scratch, sizeof(g_noalloc_scratch), stream);
}
