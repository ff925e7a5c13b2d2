// Host-side launch helpers shared by the kernel translation units: SM count
// and occupancy caches, TMA tensor-map encoding of a bf16 matrix's tile view,
// and kernel launch with optional programmatic dependent launch.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "fp4q_common.cuh"

namespace fp4q {


inline std::mutex& launch_mutex()
{
    static std::mutex mu;
    return mu;
}

inline int sm_count()
{
    constexpr int kMaxDevices = 64;
    static int counts[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lk(launch_mutex());
    int* g_sm_count = counts;
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

// Resident CTAs per SM for a kernel with `smem` bytes of dynamic shared memory,
// cached per (kernel, device); sets the shared-memory attribute on first use.
template <typename K>
int ctas_per_sm(K kernel, int smem, int threads = kThreads)
{
    static std::map<std::pair<const void*, int>, int> g_occupancy;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
    std::lock_guard<std::mutex> lk(launch_mutex());
    auto it = g_occupancy.find(key);
    if (it != g_occupancy.end()) return it->second;
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess || n <= 0) n = 1;
    g_occupancy[key] = n;
    return n;
}

template <typename K>
int grid_for(K kernel, int smem, int64_t tiles, int threads = kThreads)
{
    int64_t cap = (int64_t)sm_count() * ctas_per_sm(kernel, smem, threads);
    if (cap > kMaxPartials) cap = kMaxPartials;
    const int64_t g = tiles < cap ? tiles : cap;
    return g < 1 ? 1 : (int)g;
}

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// The tile view of a bf16 matrix and its TMA map (box 64 x rows, 128-byte swizzle).
inline bool make_view(const void* base, const Geometry& g, CUtensorMap* map, Tiles* tl, int rows = kTileRows)
{
    const int64_t n = g.rows * g.cols;
    const bool flat = (g.ld == g.cols || g.rows == 1) && n % 64 == 0 && n / 64 < ((int64_t)1 << 31);
    cuuint64_t dims[2];
    cuuint64_t strides[1];
    if (flat) {
        dims[0] = 64;
        dims[1] = (cuuint64_t)(n / 64);
        strides[0] = 128;
        tl->count = (n / 64 + rows - 1) / rows;
        tl->col_tiles = 0;
    } else {
        if (g.rows >= ((int64_t)1 << 31) || g.cols >= ((int64_t)1 << 31)) return false;
        dims[0] = (cuuint64_t)g.cols;
        dims[1] = (cuuint64_t)g.rows;
        strides[0] = (cuuint64_t)(g.ld * 2);
        tl->col_tiles = (g.cols + kTileCols - 1) / kTileCols;
        tl->count = tl->col_tiles * ((g.rows + rows - 1) / rows);
    }
    tl->rows = g.rows;
    tl->cols = g.cols;
    tl->units = n / 32;
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    cuuint32_t box[2] = {kTileCols, (cuuint32_t)rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tile count of the view make_view() builds for g.
inline int64_t view_tile_count(const Geometry& g)
{
    const int64_t n = g.rows * g.cols;
    const bool flat = (g.ld == g.cols || g.rows == 1) && n % 64 == 0 && n / 64 < ((int64_t)1 << 31);
    if (flat) return (n / 64 + kTileRows - 1) / kTileRows;
    return ((g.cols + kTileCols - 1) / kTileCols) * ((g.rows + kTileRows - 1) / kTileRows);
}

inline bool is_flat(const Tiles& tl) { return tl.col_tiles == 0; }

// Launch with `smem` bytes of dynamic shared memory; with pdl the kernel may
// start while the previous kernel on the stream drains (it waits with
// griddepcontrol.wait before reading that kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_threads(void (*kernel)(KArgs...), int grid, int threads, int smem, bool pdl, cudaStream_t st,
                           Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), int grid, int smem, bool pdl, cudaStream_t st, Args... args)
{
    return launch_threads(kernel, grid, kThreads, smem, pdl, st, args...);
}


}  // namespace fp4q
