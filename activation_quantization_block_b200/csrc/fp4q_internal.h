// Internal interface between the C ABI layer (fp4q_api.cu) and the kernels
// (fp4q_kernels.cu).  Not installed; not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fp4q {

constexpr int kThreads = 256;        // threads per CTA for every streaming kernel
constexpr int kTileCtasPerSm = 3;        // resident CTAs per SM the tile kernels are compiled for
constexpr int kMaxPartials = 4096;   // upper bound on CTAs of one pass (per-CTA partial slots)

// Workspace layout: fp64 partial sums, then fp32 partial maxima.
constexpr size_t kWsSseOffset = 0;
constexpr size_t kWsAmaxOffset = kMaxPartials * sizeof(double);
constexpr size_t kWorkspaceBytes = kWsAmaxOffset + kMaxPartials * sizeof(float);

// Geometry of a bf16 matrix seen as consecutive 16-element "halves" (one
// NVFP4 block each); a unit is two consecutive halves = 32 elements.
struct Geometry {
    int64_t rows, cols, ld;   // ld: row stride of the bf16 matrix in elements
    int64_t halves;           // rows * cols / 16
    int64_t halves_per_row;   // cols / 16
    int64_t units;            // ceil(halves / 2)
};

inline Geometry make_geometry(int64_t rows, int64_t cols, int64_t ld)
{
    Geometry g;
    g.rows = rows; g.cols = cols; g.ld = ld;
    g.halves = rows * cols / 16;
    g.halves_per_row = cols / 16;
    g.units = (g.halves + 1) / 2;
    return g;
}

// Launchers: return cudaSuccess or the launch error.  `grid_out` (nullable)
// receives the number of CTAs launched (= partial slots written).
cudaError_t launch_amax(const uint16_t* x, const Geometry& g, int rotate, float* partials,
                        int* grid_out, cudaStream_t st);

cudaError_t launch_quantize(const uint16_t* x, const Geometry& g, int fmt, int rotate, int want_sse,
                            int scale_given, int mx_ceil, uint8_t* codes, uint8_t* scales, float* tensor_scale,
                            const float* amax_partials, int n_amax, double* sse_partials,
                            int* grid_out, cudaStream_t st);

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                              const Geometry& g, int fmt, int rotate, uint16_t* y, cudaStream_t st);

cudaError_t launch_error(const uint16_t* x, const uint8_t* codes, const uint8_t* scales,
                         const float* tensor_scale, const Geometry& g, int fmt, int rotate,
                         double* sse_partials, int* grid_out, cudaStream_t st);

cudaError_t launch_sse_finalize(const double* partials, int n, double count, double* mse,
                                cudaStream_t st);

// The library's device error words in the calling thread's current CUDA
// context, one array that every kernel records into: [0] error bits
// (FP4Q_DEVICE_ERROR_*), [1] the site of the first out-of-bounds access a
// FP4Q_DEBUG build found, [2] and [3] its byte offset (low and high halves).
// Null when the address cannot be had (the launchers then fail the call).
constexpr int kErrorWords = 4;
unsigned int* device_error_words();

// Tensor-core operand form and the W4A4 product (fp4q_gemm.cu).
int64_t mma_sf_bytes(int64_t rows, int64_t cols);
cudaError_t launch_mma_pack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, int fmt,
                            uint8_t* planes, uint8_t* sf, cudaStream_t st);
cudaError_t launch_gemm_w4a4(const uint8_t* a_planes, const uint8_t* a_sf, int a_np, const float* a_scale,
                             const uint8_t* w_planes, const uint8_t* w_sf, int w_np, const float* w_scale, int64_t M,
                             int64_t N, int64_t K, uint16_t* y, int64_t ldy, cudaStream_t st);

// Failure-path self-test (fp4q_selftest.cu).
cudaError_t launch_timeout_selftest(cudaStream_t st);

// Sparse outlier separation (fp4q_outliers.cu).
int64_t outlier_capacity(int64_t cols, double max_frac);
cudaError_t launch_separate_outliers(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx, double k, int64_t cap,
                                     uint16_t* bulk, int64_t ldb, uint16_t* out_cols, uint16_t* out_vals,
                                     int32_t* out_count, cudaStream_t st);
cudaError_t launch_scatter_outliers(const uint16_t* out_cols, const uint16_t* out_vals, const int32_t* out_count,
                                    int64_t rows, int64_t cols, int64_t cap, uint16_t* y, int64_t ldy, cudaStream_t st);

// Tile count of a bf16 matrix's view (see make_view): 16 KB tiles.
int64_t view_tiles(const Geometry& g);

// One tensor of a batch (device pointers; mse may be null).
struct BatchTensor {
    const void* x;
    int64_t rows, cols, ldx;
    uint8_t* codes;
    uint8_t* scales;
    float* tensor_scale;
    double* mse;
};

// Batch workspace: three rotating slots of per-CTA absmax and error partials.
size_t batch_workspace_bytes();

// Quantize n non-empty tensors as a chain of persistent kernels, one per tensor
// (absmax pass of tensor j interleaved with the quantize pass of tensor j-1).
// single_layout (n == 1): the partials use the single-call workspace layout
// (kWorkspaceBytes) instead of the batch's rotating slots.
cudaError_t launch_quantize_batch(const BatchTensor* ts, int n, int fmt, int rotate, int scale_given, int mx_ceil,
                                  void* workspace, cudaStream_t st, bool single_layout = false);

}  // namespace fp4q
