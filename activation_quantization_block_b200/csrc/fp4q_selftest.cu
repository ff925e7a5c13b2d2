// Self-test of the failure path: a kernel whose bounded wait runs out.
//
// Every wait of the library's kernels on a pipeline barrier gives up after
// kWaitLimitNs of the global timer, records kErrPipelineTimeout in the device
// error word and returns, so that a stuck pipeline ends as a status the host
// reads instead of a hang.  This kernel exercises exactly that path: one
// thread arms an mbarrier with a transaction count that no copy will ever
// deliver and waits on it with the same bounded wait.  Nothing faults, traps or
// spins without a bound; the context stays usable.
#include <cuda_runtime.h>

#include <cstdint>

#include "fp4q_common.cuh"

namespace fp4q {

namespace {

__global__ void timeout_selftest_kernel(unsigned* err)
{
    __shared__ uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        mbar_init_fence();
        mbar_arm(b, 16u);                  // 16 bytes expected; no copy is issued
        if (!mbar_wait(b, 0u)) atomicOr(err, kErrPipelineTimeout);
    }
}

}  // namespace

cudaError_t launch_timeout_selftest(cudaStream_t st)
{
    unsigned* err = device_error_words();
    if (err == nullptr) return cudaErrorInvalidSymbol;
    timeout_selftest_kernel<<<1, 32, 0, st>>>(err);
    return cudaGetLastError();
}

}  // namespace fp4q
