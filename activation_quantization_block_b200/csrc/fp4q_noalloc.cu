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
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
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

// Driver calls that name the current CUDA context: its handle, and its ID,
// which is unique for the life of the process (a handle can be reused after a
// context is destroyed, an ID cannot).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct Driver {
    CtxGetCurrentFn get_current = nullptr;
    CtxGetIdFn get_id = nullptr;
};

const Driver& driver()
{
    static Driver d;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            d.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            d.get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    return d;
}

// ID of the calling thread's current context; false when there is none yet or
// the driver cannot say.
bool current_context_id(unsigned long long* id)
{
    const Driver& d = driver();
    CUcontext ctx = nullptr;
    if (d.get_current == nullptr || d.get_id == nullptr) return false;
    if (d.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return d.get_id(ctx, id) == CUDA_SUCCESS;
}

std::mutex g_mu;
std::map<unsigned long long, void*> g_scratch_addr;   // device address of g_noalloc_scratch, per context

// Host code cannot pass g_noalloc_scratch to a kernel: on the host that name is
// a stand-in, not a device address, and the device address belongs to one CUDA
// context.  So the address is looked up with cudaGetSymbolAddress in the
// calling thread's current context, the first time a call runs in that
// context, and cached under the context's ID: a later context (after
// cudaDeviceReset, or one the caller created itself) gets its own lookup.
fp4q_status_t scratch_address(void** out)
{
    unsigned long long id = 0;
    bool have_id = current_context_id(&id);
    if (have_id) {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_scratch_addr.find(id);
        if (it != g_scratch_addr.end()) {
            *out = it->second;
            return FP4Q_SUCCESS;
        }
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return FP4Q_ERROR_CUDA;
    }
    // the lookup made the device's primary context current if none was
    if (have_id || current_context_id(&id)) {
        std::lock_guard<std::mutex> lk(g_mu);
        g_scratch_addr[id] = p;
    }
    *out = p;
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
