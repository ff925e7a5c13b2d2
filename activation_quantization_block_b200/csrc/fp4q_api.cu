// C ABI of fp4q (declared in include/fp4q.h): argument validation, workspace
// carving and kernel dispatch.  Validation happens on the host before any
// launch; a rejected call enqueues nothing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <vector>

#include "fp4q.h"
#include "fp4q_internal.h"
#include "fp4q_scale.h"

using namespace fp4q;

#ifndef FP4Q_DEBUG
#define FP4Q_DEBUG 0
#endif

// The one set of device error words of the library (see device_error_words).
__device__ unsigned int g_fp4q_error_words[kErrorWords];

namespace {

// Driver calls that name the calling thread's current CUDA context: its handle
// and its ID, unique for the life of the process.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

bool current_context_id(unsigned long long* id)
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    if (get_current == nullptr || get_id == nullptr) return false;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

std::mutex g_err_mu;
std::map<unsigned long long, unsigned int*> g_err_addr;   // device address of the words, per context ID

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int g_dev_ok[kMaxDevices];   // 0 unknown, 1 supported, -1 not supported

// The kernels are built for sm_100a only: require compute capability 10.0.
fp4q_status_t check_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return FP4Q_ERROR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return FP4Q_ERROR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_dev_ok[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return FP4Q_ERROR_CUDA;
        }
        g_dev_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    return g_dev_ok[dev] == 1 ? FP4Q_SUCCESS : FP4Q_ERROR_UNSUPPORTED_DEVICE;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int block_len(int fmt) { return fmt == FP4Q_MXFP4 ? 32 : 16; }

bool valid_format(int fmt)
{
    return fmt == FP4Q_NVFP4 || fmt == FP4Q_NVFP4_RAZER || fmt == FP4Q_MXFP4 || fmt == FP4Q_NVFP4_RAZER_W;
}

// Shape checks shared by every entry point.
fp4q_status_t check_shape(int64_t rows, int64_t cols, int fmt, int rotate)
{
    if (!valid_format(fmt) || (rotate != 0 && rotate != 1)) return FP4Q_ERROR_INVALID_VALUE;
    if (rows < 0 || cols < 0) return FP4Q_ERROR_INVALID_VALUE;
    if (cols % block_len(fmt) != 0 || (rotate && cols % 32 != 0)) return FP4Q_ERROR_SHAPE;
    if (cols > 0 && rows > ((int64_t)1 << 62) / cols) return FP4Q_ERROR_SHAPE;
    return FP4Q_SUCCESS;
}

fp4q_status_t check_matrix(const void* p, int64_t cols, int64_t ld)
{
    if (p == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    if (ld < cols) return FP4Q_ERROR_SHAPE;
    if (ld % 8 != 0 || !aligned(p, 16)) return FP4Q_ERROR_MISALIGNED;
    if (ld > ((int64_t)1 << 62)) return FP4Q_ERROR_SHAPE;
    return FP4Q_SUCCESS;
}

fp4q_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? FP4Q_SUCCESS : FP4Q_ERROR_CUDA; }

// Known flags only; the MX exponent flag only with MXFP4.
bool valid_flags(uint32_t flags, int fmt)
{
    if (flags & ~(FP4Q_FLAG_TENSOR_SCALE_GIVEN | FP4Q_FLAG_MX_CEIL_SCALE)) return false;
    return !(flags & FP4Q_FLAG_MX_CEIL_SCALE) || fmt == FP4Q_MXFP4;
}

}  // namespace

// The address belongs to one context: look it up with cudaGetSymbolAddress in
// the calling thread's current context the first time, and cache it under the
// context's ID (after cudaDeviceReset, or under another context, a new lookup).
unsigned int* fp4q::device_error_words()
{
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    if (have_id) {
        std::lock_guard<std::mutex> lk(g_err_mu);
        auto it = g_err_addr.find(id);
        if (it != g_err_addr.end()) return it->second;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fp4q_error_words) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return nullptr;
    }
    if (have_id || current_context_id(&id)) {
        std::lock_guard<std::mutex> lk(g_err_mu);
        g_err_addr[id] = static_cast<unsigned int*>(p);
    }
    return static_cast<unsigned int*>(p);
}

extern "C" {

int fp4q_abi_version(void) { return FP4Q_ABI_VERSION; }

const char* fp4q_status_string(fp4q_status_t s)
{
    switch (s) {
        case FP4Q_SUCCESS: return "success";
        case FP4Q_ERROR_INVALID_VALUE: return "invalid value (null pointer, bad enum or flag, negative size)";
        case FP4Q_ERROR_SHAPE: return "bad shape (cols not a multiple of the block or rotation group, ld < cols, or size overflow)";
        case FP4Q_ERROR_MISALIGNED: return "misaligned pointer or leading dimension";
        case FP4Q_ERROR_WORKSPACE: return "workspace missing, misaligned or too small";
        case FP4Q_ERROR_UNSUPPORTED_DEVICE: return "current device is not sm_100 (compute capability 10.0)";
        case FP4Q_ERROR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

size_t fp4q_workspace_size(int64_t rows, int64_t cols, fp4q_format_t fmt, int rotate)
{
    (void)rows; (void)cols; (void)fmt; (void)rotate;
    return kWorkspaceBytes;
}

fp4q_status_t fp4q_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                            fp4q_format_t fmt, int rotate, uint32_t flags,
                            uint8_t* codes, uint8_t* scales, float* tensor_scale, double* mse,
                            void* workspace, size_t workspace_bytes, fp4q_stream_t stream)
{
    fp4q_status_t s = check_shape(rows, cols, fmt, rotate);
    if (s != FP4Q_SUCCESS) return s;
    if (!valid_flags(flags, fmt)) return FP4Q_ERROR_INVALID_VALUE;
    const bool nv = fmt != FP4Q_MXFP4;
    const bool given = (flags & FP4Q_FLAG_TENSOR_SCALE_GIVEN) != 0;
    if (nv && tensor_scale == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    if (nv && !aligned(tensor_scale, 4)) return FP4Q_ERROR_MISALIGNED;
    if (mse != nullptr && !aligned(mse, 8)) return FP4Q_ERROR_MISALIGNED;
    const int64_t n = rows * cols;
    const bool need_ws = n > 0 && ((nv && !given) || mse != nullptr);
    if (n > 0) {
        if ((s = check_matrix(x, cols, ldx)) != FP4Q_SUCCESS) return s;
        if (codes == nullptr || scales == nullptr) return FP4Q_ERROR_INVALID_VALUE;
        if (!aligned(codes, 16) || !aligned(scales, 16)) return FP4Q_ERROR_MISALIGNED;
    }
    if (need_ws && (workspace == nullptr || !aligned(workspace, 16) || workspace_bytes < kWorkspaceBytes))
        return FP4Q_ERROR_WORKSPACE;
    if ((s = check_device()) != FP4Q_SUCCESS) return s;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (n == 0) {
        if (nv && !given && cudaMemsetAsync(tensor_scale, 0, sizeof(float), st) != cudaSuccess) return FP4Q_ERROR_CUDA;
        if (mse && cudaMemsetAsync(mse, 0, sizeof(double), st) != cudaSuccess) return FP4Q_ERROR_CUDA;
        return FP4Q_SUCCESS;
    }

    char* ws = static_cast<char*>(workspace);
    double* sse_part = ws ? reinterpret_cast<double*>(ws + kWsSseOffset) : nullptr;
    float* amax_part = ws ? reinterpret_cast<float*>(ws + kWsAmaxOffset) : nullptr;
    const Geometry g = make_geometry(rows, cols, ldx);
    const uint16_t* xp = static_cast<const uint16_t*>(x);

    int n_amax = 0;
    if (nv && !given) {
        if ((s = from_cuda(launch_amax(xp, g, rotate, amax_part, &n_amax, st))) != FP4Q_SUCCESS) return s;
    }
    int n_sse = 0;
    s = from_cuda(launch_quantize(xp, g, fmt, rotate, mse != nullptr, given ? 1 : 0,
                                  (flags & FP4Q_FLAG_MX_CEIL_SCALE) ? 1 : 0, codes, scales,
                                  tensor_scale, amax_part, n_amax, sse_part, &n_sse, st));
    if (s != FP4Q_SUCCESS) return s;
    if (mse) s = from_cuda(launch_sse_finalize(sse_part, n_sse, (double)n, mse, st));
    return s;
}

fp4q_status_t fp4q_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                              int64_t rows, int64_t cols, fp4q_format_t fmt, int rotate,
                              void* y, int64_t ldy, fp4q_stream_t stream)
{
    fp4q_status_t s = check_shape(rows, cols, fmt, rotate);
    if (s != FP4Q_SUCCESS) return s;
    const bool nv = fmt != FP4Q_MXFP4;
    if (nv && tensor_scale == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    if (nv && !aligned(tensor_scale, 4)) return FP4Q_ERROR_MISALIGNED;
    const int64_t n = rows * cols;
    if (n > 0) {
        if ((s = check_matrix(y, cols, ldy)) != FP4Q_SUCCESS) return s;
        if (codes == nullptr || scales == nullptr) return FP4Q_ERROR_INVALID_VALUE;
        if (!aligned(codes, 16) || !aligned(scales, 16)) return FP4Q_ERROR_MISALIGNED;
    }
    if ((s = check_device()) != FP4Q_SUCCESS) return s;
    if (n == 0) return FP4Q_SUCCESS;
    const Geometry g = make_geometry(rows, cols, ldy);
    return from_cuda(launch_dequantize(codes, scales, tensor_scale, g, fmt, rotate, static_cast<uint16_t*>(y),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status_t fp4q_error(const void* x, int64_t ldx,
                         const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                         int64_t rows, int64_t cols, fp4q_format_t fmt, int rotate,
                         double* mse, void* workspace, size_t workspace_bytes, fp4q_stream_t stream)
{
    fp4q_status_t s = check_shape(rows, cols, fmt, rotate);
    if (s != FP4Q_SUCCESS) return s;
    const bool nv = fmt != FP4Q_MXFP4;
    if (mse == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    if (!aligned(mse, 8)) return FP4Q_ERROR_MISALIGNED;
    if (nv && tensor_scale == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    if (nv && !aligned(tensor_scale, 4)) return FP4Q_ERROR_MISALIGNED;
    const int64_t n = rows * cols;
    if (n > 0) {
        if ((s = check_matrix(x, cols, ldx)) != FP4Q_SUCCESS) return s;
        if (codes == nullptr || scales == nullptr) return FP4Q_ERROR_INVALID_VALUE;
        if (!aligned(codes, 16) || !aligned(scales, 16)) return FP4Q_ERROR_MISALIGNED;
        if (workspace == nullptr || !aligned(workspace, 16) || workspace_bytes < kWorkspaceBytes)
            return FP4Q_ERROR_WORKSPACE;
    }
    if ((s = check_device()) != FP4Q_SUCCESS) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (n == 0) return from_cuda(cudaMemsetAsync(mse, 0, sizeof(double), st));
    char* ws = static_cast<char*>(workspace);
    double* sse_part = reinterpret_cast<double*>(ws + kWsSseOffset);
    const Geometry g = make_geometry(rows, cols, ldx);
    int n_sse = 0;
    s = from_cuda(launch_error(static_cast<const uint16_t*>(x), codes, scales, tensor_scale, g, fmt, rotate,
                               sse_part, &n_sse, st));
    if (s != FP4Q_SUCCESS) return s;
    return from_cuda(launch_sse_finalize(sse_part, n_sse, (double)n, mse, st));
}

fp4q_status_t fp4q_tensor_scale(const void* x, int64_t rows, int64_t cols, int64_t ldx, fp4q_format_t fmt,
                                int rotate, float* tensor_scale, void* workspace, size_t workspace_bytes,
                                fp4q_stream_t stream)
{
    fp4q_status_t s = check_shape(rows, cols, fmt, rotate);
    if (s != FP4Q_SUCCESS) return s;
    if (fmt == FP4Q_MXFP4 || tensor_scale == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    if (!aligned(tensor_scale, 4)) return FP4Q_ERROR_MISALIGNED;
    const int64_t n = rows * cols;
    if (n > 0) {
        if ((s = check_matrix(x, cols, ldx)) != FP4Q_SUCCESS) return s;
        if (workspace == nullptr || !aligned(workspace, 16) || workspace_bytes < kWorkspaceBytes)
            return FP4Q_ERROR_WORKSPACE;
    }
    if ((s = check_device()) != FP4Q_SUCCESS) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (n == 0) return from_cuda(cudaMemsetAsync(tensor_scale, 0, sizeof(float), st));
    float* amax_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kWsAmaxOffset);
    const Geometry g = make_geometry(rows, cols, ldx);
    int n_amax = 0;
    s = from_cuda(launch_amax(static_cast<const uint16_t*>(x), g, rotate, amax_part, &n_amax, st));
    if (s != FP4Q_SUCCESS) return s;
    return from_cuda(launch_tensor_scale(amax_part, n_amax, fmt, tensor_scale, st));
}

fp4q_status_t fp4q_device_errors(uint32_t* bits, int clear)
{
    if (bits == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    fp4q_status_t s = check_device();
    if (s != FP4Q_SUCCESS) return s;
    unsigned int w[kErrorWords] = {0, 0, 0, 0};
    if (cudaMemcpyFromSymbol(w, g_fp4q_error_words, sizeof w) != cudaSuccess) {
        cudaGetLastError();
        return FP4Q_ERROR_CUDA;
    }
    if (clear) {
        const unsigned int zero[kErrorWords] = {0, 0, 0, 0};
        if (cudaMemcpyToSymbol(g_fp4q_error_words, zero, sizeof zero) != cudaSuccess) {
            cudaGetLastError();
            return FP4Q_ERROR_CUDA;
        }
    }
    *bits = w[0];
    return FP4Q_SUCCESS;
}

fp4q_status_t fp4q_device_error_site(uint32_t* site, uint64_t* offset)
{
    if (site == nullptr || offset == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    fp4q_status_t s = check_device();
    if (s != FP4Q_SUCCESS) return s;
    unsigned int w[kErrorWords] = {0, 0, 0, 0};
    if (cudaMemcpyFromSymbol(w, g_fp4q_error_words, sizeof w) != cudaSuccess) {
        cudaGetLastError();
        return FP4Q_ERROR_CUDA;
    }
    *site = w[1];
    *offset = (uint64_t)w[2] | ((uint64_t)w[3] << 32);
    return FP4Q_SUCCESS;
}

int fp4q_debug_build(void) { return FP4Q_DEBUG ? 1 : 0; }

fp4q_status_t fp4q_selftest_timeout(fp4q_stream_t stream)
{
    fp4q_status_t s = check_device();
    if (s != FP4Q_SUCCESS) return s;
    return from_cuda(launch_timeout_selftest(reinterpret_cast<cudaStream_t>(stream)));
}

int64_t fp4q_outlier_capacity(int64_t cols, double max_frac)
{
    if (cols < 0 || !(max_frac >= 0.0 && max_frac <= 1.0)) return 0;
    return outlier_capacity(cols, max_frac);
}

fp4q_status_t fp4q_separate_outliers(const void* x, int64_t rows, int64_t cols, int64_t ldx, double k,
                                     double max_frac, void* bulk, int64_t ldb, uint16_t* out_cols,
                                     uint16_t* out_vals, int32_t* out_count, fp4q_stream_t stream)
{
    if (rows < 0 || cols < 0 || !(k > 0.0 && k < 1e300) || !(max_frac >= 0.0 && max_frac <= 1.0))
        return FP4Q_ERROR_INVALID_VALUE;
    if (cols % 8 != 0 || cols > 65536 || rows >= ((int64_t)1 << 31)) return FP4Q_ERROR_SHAPE;
    if (rows == 0) return FP4Q_SUCCESS;
    fp4q_status_t s;
    if (cols == 0) {   // no elements: every row has no outliers
        if (out_count == nullptr) return FP4Q_ERROR_INVALID_VALUE;
        if (!aligned(out_count, 4)) return FP4Q_ERROR_MISALIGNED;
        if ((s = check_device()) != FP4Q_SUCCESS) return s;
        return from_cuda(cudaMemsetAsync(out_count, 0, sizeof(int32_t) * (size_t)rows,
                                         reinterpret_cast<cudaStream_t>(stream)));
    }
    if ((s = check_matrix(x, cols, ldx)) != FP4Q_SUCCESS) return s;
    if ((s = check_matrix(bulk, cols, ldb)) != FP4Q_SUCCESS) return s;
    const int64_t cap = outlier_capacity(cols, max_frac);
    if (out_count == nullptr || (cap > 0 && (out_cols == nullptr || out_vals == nullptr)))
        return FP4Q_ERROR_INVALID_VALUE;
    if (!aligned(out_count, 4) || !aligned(out_cols, 2) || !aligned(out_vals, 2)) return FP4Q_ERROR_MISALIGNED;
    if ((s = check_device()) != FP4Q_SUCCESS) return s;
    return from_cuda(launch_separate_outliers(static_cast<const uint16_t*>(x), rows, cols, ldx, k, cap,
                                              static_cast<uint16_t*>(bulk), ldb, out_cols, out_vals, out_count,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status_t fp4q_scatter_outliers(const uint16_t* out_cols, const uint16_t* out_vals, const int32_t* out_count,
                                    int64_t rows, int64_t cols, int64_t cap, void* y, int64_t ldy,
                                    fp4q_stream_t stream)
{
    if (rows < 0 || cols < 0 || cap < 0 || cap > cols) return FP4Q_ERROR_INVALID_VALUE;
    if (rows == 0 || cap == 0) return FP4Q_SUCCESS;
    if (out_cols == nullptr || out_vals == nullptr || out_count == nullptr || y == nullptr)
        return FP4Q_ERROR_INVALID_VALUE;
    if (ldy < cols) return FP4Q_ERROR_SHAPE;
    if (!aligned(y, 2) || !aligned(out_count, 4) || !aligned(out_cols, 2) || !aligned(out_vals, 2))
        return FP4Q_ERROR_MISALIGNED;
    fp4q_status_t s = check_device();
    if (s != FP4Q_SUCCESS) return s;
    return from_cuda(launch_scatter_outliers(out_cols, out_vals, out_count, rows, cols, cap,
                                             static_cast<uint16_t*>(y), ldy, reinterpret_cast<cudaStream_t>(stream)));
}

int fp4q_mma_planes(fp4q_format_t fmt)
{
    if (fmt == FP4Q_NVFP4) return 1;
    if (fmt == FP4Q_NVFP4_RAZER || fmt == FP4Q_NVFP4_RAZER_W) return 2;
    return 0;
}

size_t fp4q_mma_sf_bytes(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0 || rows > ((int64_t)1 << 40) || cols > ((int64_t)1 << 40)) return 0;
    return (size_t)mma_sf_bytes(rows, cols);
}

fp4q_status_t fp4q_mma_pack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                            fp4q_format_t fmt, uint8_t* planes, uint8_t* sf, fp4q_stream_t stream)
{
    if (fp4q_mma_planes(fmt) == 0 || rows < 0 || cols < 0) return FP4Q_ERROR_INVALID_VALUE;
    if (cols % 16 != 0 || rows > ((int64_t)1 << 40) || cols > ((int64_t)1 << 40)) return FP4Q_ERROR_SHAPE;
    if (rows * cols == 0) return FP4Q_SUCCESS;
    if (codes == nullptr || scales == nullptr || planes == nullptr || sf == nullptr) return FP4Q_ERROR_INVALID_VALUE;
    if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(planes, 16) || !aligned(sf, 16))
        return FP4Q_ERROR_MISALIGNED;
    fp4q_status_t s = check_device();
    if (s != FP4Q_SUCCESS) return s;
    return from_cuda(launch_mma_pack(codes, scales, rows, cols, fmt, planes, sf,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status_t fp4q_gemm(const uint8_t* a_planes, const uint8_t* a_sf, int a_np, const float* a_scale,
                        const uint8_t* w_planes, const uint8_t* w_sf, int w_np, const float* w_scale,
                        int64_t M, int64_t N, int64_t K, void* y, int64_t ldy, fp4q_stream_t stream)
{
    if ((a_np != 1 && a_np != 2) || (w_np != 1 && w_np != 2)) return FP4Q_ERROR_INVALID_VALUE;
    if (M < 0 || N < 0 || K < 0) return FP4Q_ERROR_INVALID_VALUE;
    if (K == 0 || K % 256 != 0 || N % 8 != 0 || ldy < N || M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) ||
        K >= ((int64_t)1 << 31) || ldy >= ((int64_t)1 << 31))
        return FP4Q_ERROR_SHAPE;
    if (ldy % 8 != 0) return FP4Q_ERROR_MISALIGNED;
    if (M == 0 || N == 0) return FP4Q_SUCCESS;
    if (a_planes == nullptr || a_sf == nullptr || a_scale == nullptr || w_planes == nullptr || w_sf == nullptr ||
        w_scale == nullptr || y == nullptr)
        return FP4Q_ERROR_INVALID_VALUE;
    if (!aligned(a_planes, 16) || !aligned(a_sf, 16) || !aligned(w_planes, 16) || !aligned(w_sf, 16) ||
        !aligned(y, 16) || !aligned(a_scale, 4) || !aligned(w_scale, 4))
        return FP4Q_ERROR_MISALIGNED;
    fp4q_status_t s = check_device();
    if (s != FP4Q_SUCCESS) return s;
    return from_cuda(launch_gemm_w4a4(a_planes, a_sf, a_np, a_scale, w_planes, w_sf, w_np, w_scale, M, N, K,
                                      static_cast<uint16_t*>(y), ldy, reinterpret_cast<cudaStream_t>(stream)));
}

size_t fp4q_batch_workspace_size(int count, const fp4q_tensor_desc_t* tensors, fp4q_format_t fmt, int rotate)
{
    (void)count; (void)tensors; (void)fmt; (void)rotate;
    return batch_workspace_bytes();
}

fp4q_status_t fp4q_quantize_batch(int count, const fp4q_tensor_desc_t* tensors, fp4q_format_t fmt, int rotate,
                                  uint32_t flags, void* workspace, size_t workspace_bytes, fp4q_stream_t stream)
{
    if (count < 0 || (count > 0 && tensors == nullptr)) return FP4Q_ERROR_INVALID_VALUE;
    if (!valid_flags(flags, fmt)) return FP4Q_ERROR_INVALID_VALUE;
    const bool nv = fmt != FP4Q_MXFP4;
    const bool given = (flags & FP4Q_FLAG_TENSOR_SCALE_GIVEN) != 0;
    fp4q_status_t s;
    for (int k = 0; k < count; ++k) {
        const fp4q_tensor_desc_t& t = tensors[k];
        if ((s = check_shape(t.rows, t.cols, fmt, rotate)) != FP4Q_SUCCESS) return s;
        if (nv && t.tensor_scale == nullptr) return FP4Q_ERROR_INVALID_VALUE;
        if (nv && !aligned(t.tensor_scale, 4)) return FP4Q_ERROR_MISALIGNED;
        if (t.mse != nullptr && !aligned(t.mse, 8)) return FP4Q_ERROR_MISALIGNED;
        if (t.rows * t.cols > 0) {
            if ((s = check_matrix(t.x, t.cols, t.ldx)) != FP4Q_SUCCESS) return s;
            if (t.codes == nullptr || t.scales == nullptr) return FP4Q_ERROR_INVALID_VALUE;
            if (!aligned(t.codes, 16) || !aligned(t.scales, 16)) return FP4Q_ERROR_MISALIGNED;
        }
    }
    if (count == 0) return FP4Q_SUCCESS;
    if (workspace == nullptr || !aligned(workspace, 16) ||
        workspace_bytes < fp4q_batch_workspace_size(count, tensors, fmt, rotate))
        return FP4Q_ERROR_WORKSPACE;
    if ((s = check_device()) != FP4Q_SUCCESS) return s;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    std::vector<BatchTensor> work;
    work.reserve((size_t)count);
    for (int k = 0; k < count; ++k) {
        const fp4q_tensor_desc_t& t = tensors[k];
        if (t.rows * t.cols == 0) {   // empty: the scalar outputs are 0, as with fp4q_quantize
            if (nv && !given && cudaMemsetAsync(t.tensor_scale, 0, sizeof(float), st) != cudaSuccess) return FP4Q_ERROR_CUDA;
            if (t.mse && cudaMemsetAsync(t.mse, 0, sizeof(double), st) != cudaSuccess) return FP4Q_ERROR_CUDA;
            continue;
        }
        work.push_back(BatchTensor{t.x, t.rows, t.cols, t.ldx, t.codes, t.scales, t.tensor_scale, t.mse});
    }
    if (!work.empty() &&
        launch_quantize_batch(work.data(), (int)work.size(), fmt, rotate, given ? 1 : 0,
                              (flags & FP4Q_FLAG_MX_CEIL_SCALE) ? 1 : 0, workspace, st) != cudaSuccess) {
        cudaGetLastError();
        return FP4Q_ERROR_CUDA;
    }
    return FP4Q_SUCCESS;
}

}  // extern "C"
