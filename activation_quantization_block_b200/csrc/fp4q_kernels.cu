// fp4q kernels for sm_100a: tensor absmax, fused quantize, dequantize, error,
// and the fixed-order fp64 finaliser for the squared-error sums.
//
// Work decomposition.  Every kernel streams 16 KB tiles of 128 rows x 64 bf16
// through a TMA pipeline (fp4q_tma.cuh).  A contiguous matrix whose size is a
// multiple of 64 is viewed as [N/64][64] ("flat"), so a tile is 16 KB of
// consecutive elements; otherwise the view is [rows][cols] with the row
// stride, and a tile is 128 rows x 64 columns.  Thread t of a CTA owns the
// unit (tile row t/2, half t%2): 32 consecutive elements of one matrix row,
// i.e. two NVFP4 blocks or one MXFP4 block / rotation group, 16 bytes of
// codes and 2 (NVFP4) or 1 (MXFP4) scale bytes.  The 32-point rotation runs
// in the thread's registers.  Grids are persistent (resident CTAs per SM x
// SMs) and walk the tiles round-robin.
//
// Kernels of one call are chained with programmatic dependent launch: the
// quantize pass starts fetching its first tiles while the absmax pass drains
// and waits (griddepcontrol.wait) only before it reads the absmax partials;
// the absmax pass walks the tiles forwards and the quantize pass backwards, so
// the quantize pass begins on the tiles the absmax pass left in L2.
//
// Method references (title, section):
//  "RaZeR: Pushing the Limits of NVFP4 Quantization with Redundant Zero
//   Remapping": sect. 1 (E2M1 set, E4M3 block scale from the block absmax,
//   unused scale sign bit), sect. 2.2 (-0 code remapped to a special value
//   chosen per block by minimum squared error; one bit -> the pair +-5;
//   weights: a 6-bit E3M3 block scale and two bits -> four special values).
//  "TORQ: Two-Level Orthogonal Rotation for MXFP4 Quantization": sect. 1
//   (32-element blocks, shared exponent, e2m1 codebook), sect. 2 (orthogonal
//   intra-block rotation before quantization).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "fp4q_launch.cuh"

namespace fp4q {

// ---------------------------------------------------------------------------
// Kernels
// ---------------------------------------------------------------------------

struct AmaxArgs {
    Tiles tl;
    float* partials;
    unsigned* err;          // the library's device error words
};

// Q0: per-CTA maxima of |x| (of |H x| when rotating).
template <bool ROT, bool FLAT>
__global__ void __launch_bounds__(kThreads) amax_kernel(const __grid_constant__ CUtensorMap xmap, AmaxArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ float shf[32];
    const Pipe p = pipe_setup(smem_raw);
    const Schedule sc = make_schedule(a.tl.count, false);
    const int t = threadIdx.x;
    if (t == 0)
        for (int64_t j = 0; j < sc.mine && j < kStages; ++j) pipe_issue<FLAT>(p, &xmap, a.tl, sc, j);
    pdl_trigger();
    float m = 0.0f;
    for (int64_t j = 0; j < sc.mine; ++j) {
        if (!pipe_acquire(p, j)) {
            pipe_fail(p, j, j + kStages < sc.mine ? j + kStages : sc.mine, a.err);
            break;
        }
        m = fmaxf(m, amax_tile<ROT>(p.tiles + (uint32_t)(j % kStages) * kTileBytes));
        pipe_release(p, j);
        if (t == 0 && j + kStages < sc.mine) {
            if (!pipe_stage_free(p, j)) {
                pipe_fail(p, j + 1, j + kStages, a.err);
                break;
            }
            pipe_issue<FLAT>(p, &xmap, a.tl, sc, j + kStages);
        }
    }
    m = block_max(m, shf);
    if (t == 0 && in_bounds(4 * (int64_t)blockIdx.x, 4, 4 * (int64_t)kMaxPartials, kSiteAmaxPartialStore, a.err))
        a.partials[blockIdx.x] = m;
}

struct QuantArgs {
    Tiles tl;
    uint8_t* codes;
    uint8_t* scales;
    float* tensor_scale;
    const float* amax_partials;
    int n_amax;
    int scale_given;
    int reverse;
    int mx_ceil;
    double* sse_partials;
    unsigned* err;          // the library's device error words
};

// CTA shape of the quantize pass per format.  NVFP4 and the RaZeR weight
// mode measured faster with ten warps, tiles of 160 rows (20 KB) and two CTAs
// per SM (up to 96 registers a thread); RaZeR and MXFP4 keep eight warps,
// 128-row tiles and three CTAs per SM.  Thread t owns unit (row t / 2, half
// t % 2), so threads = 2 x rows.
template <int FMT>
struct QuantShape {
    static constexpr bool kWide = FMT == kNV || FMT == kRW;
    static constexpr int kRows = kWide ? 160 : kTileRows;
    static constexpr int kThreads = 2 * kRows;
    static constexpr int kWarps = kThreads / 32;
    static constexpr int kCtasPerSm = kWide ? 2 : kTileCtasPerSm;
    static constexpr int kTileBytes = kRows * 128;
    static constexpr int kSmemBytes = pipe_smem_bytes(kTileBytes);
};
static_assert(QuantShape<kRZ>::kThreads == kThreads && QuantShape<kMX>::kThreads == kThreads,
              "RaZeR and MXFP4 keep the streaming kernels' shape");

inline int quant_rows(int fmt) { return (fmt == kNV || fmt == kRW) ? QuantShape<kNV>::kRows : kTileRows; }

// Q1-Q6: rotate, block scale, encode, RaZeR select, pack, store, SSE partials.
template <int FMT, bool ROT, bool SSE, bool FLAT>
__global__ void __launch_bounds__(QuantShape<FMT>::kThreads, QuantShape<FMT>::kCtasPerSm)
    quantize_kernel(const __grid_constant__ CUtensorMap xmap, QuantArgs a)
{
    using Shape = QuantShape<FMT>;
    constexpr int kThreads = Shape::kThreads;
    constexpr int kRows = Shape::kRows;
    constexpr int kTileBytes = Shape::kTileBytes;
    extern __shared__ uint8_t smem_raw[];
    __shared__ float shf[32];
    __shared__ double shd[32];
    const Pipe p = pipe_setup<kTileBytes, Shape::kWarps>(smem_raw);
    const Schedule sc = make_schedule(a.tl.count, a.reverse != 0);
    const int t = threadIdx.x;
    // x was complete before the preceding kernel of this call started, so the
    // first tiles may be fetched before waiting for that kernel.
    if (t == 0)
        for (int64_t j = 0; j < sc.mine && j < kStages; ++j) pipe_issue<FLAT, kRows>(p, &xmap, a.tl, sc, j);
    pdl_wait();

    // Tensor scale (NVFP4 formats): s_t = RN(A / (6 * 448)), or RN(A / (6 * 30))
    // in the weight mode, from the absmax partials.
    float s_t = 0.0f;
    if (FMT != kMX) {
        if (a.scale_given) {
            s_t = *a.tensor_scale;
        } else {
            float m = 0.0f;
            for (int i = t; i < a.n_amax; i += kThreads)
                if (in_bounds(4 * (int64_t)i, 4, 4 * (int64_t)kMaxPartials, kSiteAmaxPartialLoad, a.err))
                    m = fmaxf(m, a.amax_partials[i]);
            m = block_max(m, shf);
            s_t = tensor_scale_of<FMT>(m);
            if (blockIdx.x == 0 && t == 0) *a.tensor_scale = s_t;
        }
    }
    pdl_trigger();
    __shared__ NvTable nvt;
    const NvScale nsc = nv_scale_setup<FMT>(s_t, &nvt);

    double acc = 0.0;
    for (int64_t j = 0; j < sc.mine; ++j) {
        if (!pipe_acquire(p, j)) {
            pipe_fail(p, j, j + kStages < sc.mine ? j + kStages : sc.mine, a.err);
            break;
        }
        const uint32_t tile = p.tiles + (uint32_t)(j % kStages) * kTileBytes;
        acc += quantize_tile<FMT, ROT, SSE, FLAT, kRows>(tile, a.tl, sc.tile(j), a.codes, a.scales, nsc,
                                                         a.mx_ceil != 0, a.err);
        pipe_release(p, j);
        if (t == 0 && j + kStages < sc.mine) {
            if (!pipe_stage_free(p, j)) {
                pipe_fail(p, j + 1, j + kStages, a.err);
                break;
            }
            pipe_issue<FLAT, kRows>(p, &xmap, a.tl, sc, j + kStages);
        }
    }
    if (SSE) {
        acc = block_sum(acc, shd);
        if (t == 0 && in_bounds(8 * (int64_t)blockIdx.x, 8, 8 * (int64_t)kMaxPartials, kSiteSsePartialStore, a.err))
            a.sse_partials[blockIdx.x] = acc;
    }
}

struct ErrArgs {
    Tiles tl;
    const uint8_t* codes;
    const uint8_t* scales;
    const float* tensor_scale;
    double* sse_partials;
    unsigned* err;          // the library's device error words
};

// Q8: squared error of a given encoding against x.
template <int FMT, bool ROT, bool FLAT>
__global__ void __launch_bounds__(kThreads, kTileCtasPerSm) error_kernel(const __grid_constant__ CUtensorMap xmap, ErrArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ double shd[32];
    const Pipe p = pipe_setup(smem_raw);
    const Schedule sc = make_schedule(a.tl.count, false);
    const int t = threadIdx.x;
    if (t == 0)
        for (int64_t j = 0; j < sc.mine && j < kStages; ++j) pipe_issue<FLAT>(p, &xmap, a.tl, sc, j);
    pdl_trigger();
    const float s_t = (FMT != kMX) ? *a.tensor_scale : 0.0f;
    const bool a16 = FLAT || (a.tl.cols % 32) == 0;
    const uint32_t r = (uint32_t)t >> 1, h = (uint32_t)t & 1u;
    double acc = 0.0;
    for (int64_t j = 0; j < sc.mine; ++j) {
        const Unit u = unit_of<FLAT>(a.tl, sc.tile(j), t);
        uint32_t cw[4] = {0, 0, 0, 0}, sb[2] = {0, 0};
        if (u.valid) {
            int64_t co, so;
            unit_offsets<FLAT, FMT>(a.tl, u, co, so);
            load_packed<FMT>(a.codes, a.scales, co, so, u.full, a16, cw, sb, a.tl.rows * a.tl.cols / 2,
                             a.tl.rows * a.tl.cols / (FMT == kMX ? 32 : 16), a.err);
        }
        if (!pipe_acquire(p, j)) {
            pipe_fail(p, j, j + kStages < sc.mine ? j + kStages : sc.mine, a.err);
            break;
        }
        if (u.valid) {
            const uint32_t tile = p.tiles + (uint32_t)(j % kStages) * kTileBytes;
            uint32_t w[16];
            load_unit_words(tile, r, h, w);
            float xh[32], x[32];
            decode_unit<FMT>(cw, sb, s_t, xh);
            if (ROT) wht32_inplace(xh);
            if (!u.full) {
#pragma unroll
                for (int i = 16; i < 32; ++i) xh[i] = 0.0f;
            }
            unpack16(w, x);
            unpack16(w + 8, x + 16);
            acc += sse_of<32>(x, xh);
        }
        pipe_release(p, j);
        if (t == 0 && j + kStages < sc.mine) {
            if (!pipe_stage_free(p, j)) {
                pipe_fail(p, j + 1, j + kStages, a.err);
                break;
            }
            pipe_issue<FLAT>(p, &xmap, a.tl, sc, j + kStages);
        }
    }
    acc = block_sum(acc, shd);
    if (t == 0 && in_bounds(8 * (int64_t)blockIdx.x, 8, 8 * (int64_t)kMaxPartials, kSiteSsePartialStore, a.err))
        a.sse_partials[blockIdx.x] = acc;
}

struct DeqArgs {
    Tiles tl;
    const uint8_t* codes;
    const uint8_t* scales;
    const float* tensor_scale;
    unsigned* err;          // the library's device error words
};

// Q7: reconstruct bf16 tiles in shared memory (the swizzled layout of the
// loads) and write them with TMA stores; two output buffers alternate, and
// the next unit's codes are fetched while the current one is written.
template <int FMT, bool ROT, bool FLAT>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(const __grid_constant__ CUtensorMap ymap, DeqArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const Schedule sc = make_schedule(a.tl.count, false);
    const int t = threadIdx.x;
    pdl_trigger();
    const float s_t = (FMT != kMX) ? *a.tensor_scale : 0.0f;
    const bool a16 = FLAT || (a.tl.cols % 32) == 0;
    const uint32_t r = (uint32_t)t >> 1, h = (uint32_t)t & 1u;

    uint32_t cw[4] = {0, 0, 0, 0}, sb[2] = {0, 0};
    Unit u{};
    if (sc.mine > 0) {
        u = unit_of<FLAT>(a.tl, sc.tile(0), t);
        if (u.valid) {
            int64_t co, so;
            unit_offsets<FLAT, FMT>(a.tl, u, co, so);
            load_packed<FMT>(a.codes, a.scales, co, so, u.full, a16, cw, sb, a.tl.rows * a.tl.cols / 2,
                             a.tl.rows * a.tl.cols / (FMT == kMX ? 32 : 16), a.err);
        }
    }
    for (int64_t j = 0; j < sc.mine; ++j) {
        const int64_t k = sc.tile(j);
        const Unit cur = u;
        const uint32_t ccw[4] = {cw[0], cw[1], cw[2], cw[3]}, csb[2] = {sb[0], sb[1]};
        if (j + 1 < sc.mine) {
            u = unit_of<FLAT>(a.tl, sc.tile(j + 1), t);
            if (u.valid) {
                int64_t co, so;
                unit_offsets<FLAT, FMT>(a.tl, u, co, so);
                load_packed<FMT>(a.codes, a.scales, co, so, u.full, a16, cw, sb, a.tl.rows * a.tl.cols / 2,
                             a.tl.rows * a.tl.cols / (FMT == kMX ? 32 : 16), a.err);
            }
        }
        uint32_t o[16] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
        if (cur.valid) {
            float xh[32];
            decode_unit<FMT>(ccw, csb, s_t, xh);
            if (ROT) wht32_inplace(xh);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = pack_bf16x2_rn(xh[2 * i], xh[2 * i + 1]);
        }
        const uint32_t buf = base + (uint32_t)(j & 1) * kTileBytes;
        // the TMA store issued from this buffer two tiles ago must have read it
        if (t == 0) bulk_wait_reads_but_last();
        __syncthreads();
#pragma unroll
        for (int c = 0; c < 4; ++c)
            sts128(tile_chunk(buf, r, 4 * h + c), make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]));
        fence_async_smem();
        __syncthreads();
        if (t == 0) {
            int x, y;
            tile_origin<FLAT>(a.tl, k, x, y);
            tma_store_tile(&ymap, x, y, buf);
            bulk_commit();
        }
    }
    if (t == 0) bulk_wait_all();
}

// Sum n fp64 partials in a fixed order and write sum / count.
__global__ void __launch_bounds__(kThreads) sse_finalize_kernel(const double* partials, int n, double count,
                                                                double* mse, unsigned* err)
{
    __shared__ double sh[kThreads];
    pdl_wait();
    double s = 0.0;
    for (int i = threadIdx.x; i < n; i += kThreads)
        if (in_bounds(8 * (int64_t)i, 8, 8 * (int64_t)kMaxPartials, kSiteSsePartialLoad, err)) s += partials[i];
    sh[threadIdx.x] = s;
    __syncthreads();
    for (int o = kThreads / 2; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *mse = count > 0.0 ? sh[0] / count : 0.0;
}

// ---------------------------------------------------------------------------
// Host side: tensor maps, grids, launches
// ---------------------------------------------------------------------------

cudaError_t launch_amax(const uint16_t* x, const Geometry& g, int rotate, float* partials, int* grid_out,
                        cudaStream_t st)
{
    CUtensorMap map;
    AmaxArgs a;
    if (!make_view(x, g, &map, &a.tl)) return cudaErrorInvalidValue;
    a.partials = partials;
    if ((a.err = device_error_words()) == nullptr) return cudaErrorInvalidSymbol;
    auto go = [&](auto kernel) {
        const int grid = grid_for(kernel, kPipeSmemBytes, a.tl.count);
        if (grid_out) *grid_out = grid;
        return launch(kernel, grid, kPipeSmemBytes, false, st, map, a);
    };
    const bool flat = is_flat(a.tl);
    if (rotate) return flat ? go(amax_kernel<true, true>) : go(amax_kernel<true, false>);
    return flat ? go(amax_kernel<false, true>) : go(amax_kernel<false, false>);
}

template <int FMT, bool ROT>
static cudaError_t quantize_dispatch(const CUtensorMap& map, const QuantArgs& a, bool sse, bool pdl, int* grid_out,
                                     cudaStream_t st)
{
    using Shape = QuantShape<FMT>;
    auto go = [&](auto kernel) {
        const int grid = grid_for(kernel, Shape::kSmemBytes, a.tl.count, Shape::kThreads);
        if (grid_out) *grid_out = grid;
        return launch_threads(kernel, grid, Shape::kThreads, Shape::kSmemBytes, pdl, st, map, a);
    };
    const bool flat = is_flat(a.tl);
    if (sse) return flat ? go(quantize_kernel<FMT, ROT, true, true>) : go(quantize_kernel<FMT, ROT, true, false>);
    return flat ? go(quantize_kernel<FMT, ROT, false, true>) : go(quantize_kernel<FMT, ROT, false, false>);
}

cudaError_t launch_quantize(const uint16_t* x, const Geometry& g, int fmt, int rotate, int want_sse,
                            int scale_given, int mx_ceil, uint8_t* codes, uint8_t* scales, float* tensor_scale,
                            const float* amax_partials, int n_amax, double* sse_partials, int* grid_out,
                            cudaStream_t st)
{
    CUtensorMap map;
    QuantArgs a;
    if (!make_view(x, g, &map, &a.tl, quant_rows(fmt))) return cudaErrorInvalidValue;
    if ((a.err = device_error_words()) == nullptr) return cudaErrorInvalidSymbol;
    a.codes = codes;
    a.scales = scales;
    a.tensor_scale = tensor_scale;
    a.amax_partials = amax_partials;
    a.n_amax = n_amax;
    a.scale_given = scale_given;
    a.mx_ceil = mx_ceil;
    // after an absmax pass: start where that pass ended (its last tiles are in L2)
    const bool after_amax = fmt != kMX && !scale_given;
    a.reverse = after_amax ? 1 : 0;
    a.sse_partials = sse_partials;
    const bool sse = want_sse != 0;
    switch (fmt * 2 + (rotate ? 1 : 0)) {
        case 0: return quantize_dispatch<kNV, false>(map, a, sse, after_amax, grid_out, st);
        case 1: return quantize_dispatch<kNV, true>(map, a, sse, after_amax, grid_out, st);
        case 2: return quantize_dispatch<kRZ, false>(map, a, sse, after_amax, grid_out, st);
        case 3: return quantize_dispatch<kRZ, true>(map, a, sse, after_amax, grid_out, st);
        case 4: return quantize_dispatch<kMX, false>(map, a, sse, after_amax, grid_out, st);
        case 5: return quantize_dispatch<kMX, true>(map, a, sse, after_amax, grid_out, st);
        case 6: return quantize_dispatch<kRW, false>(map, a, sse, after_amax, grid_out, st);
        case 7: return quantize_dispatch<kRW, true>(map, a, sse, after_amax, grid_out, st);
        default: return cudaErrorInvalidValue;
    }
}

constexpr int kDeqSmemBytes = 2 * kTileBytes + 1024;

template <int FMT, bool ROT>
static cudaError_t dequantize_dispatch(const CUtensorMap& map, const DeqArgs& a, cudaStream_t st)
{
    auto go = [&](auto kernel) {
        const int grid = grid_for(kernel, kDeqSmemBytes, a.tl.count);
        return launch(kernel, grid, kDeqSmemBytes, false, st, map, a);
    };
    return is_flat(a.tl) ? go(dequantize_kernel<FMT, ROT, true>) : go(dequantize_kernel<FMT, ROT, false>);
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                              const Geometry& g, int fmt, int rotate, uint16_t* y, cudaStream_t st)
{
    CUtensorMap map;
    DeqArgs a;
    if (!make_view(y, g, &map, &a.tl)) return cudaErrorInvalidValue;
    if ((a.err = device_error_words()) == nullptr) return cudaErrorInvalidSymbol;
    a.codes = codes;
    a.scales = scales;
    a.tensor_scale = tensor_scale;
    switch (fmt * 2 + (rotate ? 1 : 0)) {
        case 0: return dequantize_dispatch<kNV, false>(map, a, st);
        case 1: return dequantize_dispatch<kNV, true>(map, a, st);
        case 2: return dequantize_dispatch<kRZ, false>(map, a, st);
        case 3: return dequantize_dispatch<kRZ, true>(map, a, st);
        case 4: return dequantize_dispatch<kMX, false>(map, a, st);
        case 5: return dequantize_dispatch<kMX, true>(map, a, st);
        case 6: return dequantize_dispatch<kRW, false>(map, a, st);
        case 7: return dequantize_dispatch<kRW, true>(map, a, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int FMT, bool ROT>
static cudaError_t error_dispatch(const CUtensorMap& map, const ErrArgs& a, int* grid_out, cudaStream_t st)
{
    auto go = [&](auto kernel) {
        const int grid = grid_for(kernel, kPipeSmemBytes, a.tl.count);
        if (grid_out) *grid_out = grid;
        return launch(kernel, grid, kPipeSmemBytes, false, st, map, a);
    };
    return is_flat(a.tl) ? go(error_kernel<FMT, ROT, true>) : go(error_kernel<FMT, ROT, false>);
}

cudaError_t launch_error(const uint16_t* x, const uint8_t* codes, const uint8_t* scales,
                         const float* tensor_scale, const Geometry& g, int fmt, int rotate,
                         double* sse_partials, int* grid_out, cudaStream_t st)
{
    CUtensorMap map;
    ErrArgs a;
    if (!make_view(x, g, &map, &a.tl)) return cudaErrorInvalidValue;
    if ((a.err = device_error_words()) == nullptr) return cudaErrorInvalidSymbol;
    a.codes = codes;
    a.scales = scales;
    a.tensor_scale = tensor_scale;
    a.sse_partials = sse_partials;
    switch (fmt * 2 + (rotate ? 1 : 0)) {
        case 0: return error_dispatch<kNV, false>(map, a, grid_out, st);
        case 1: return error_dispatch<kNV, true>(map, a, grid_out, st);
        case 2: return error_dispatch<kRZ, false>(map, a, grid_out, st);
        case 3: return error_dispatch<kRZ, true>(map, a, grid_out, st);
        case 4: return error_dispatch<kMX, false>(map, a, grid_out, st);
        case 5: return error_dispatch<kMX, true>(map, a, grid_out, st);
        case 6: return error_dispatch<kRW, false>(map, a, grid_out, st);
        case 7: return error_dispatch<kRW, true>(map, a, grid_out, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_sse_finalize(const double* partials, int n, double count, double* mse, cudaStream_t st)
{
    unsigned* err = device_error_words();
    if (err == nullptr) return cudaErrorInvalidSymbol;
    return launch(sse_finalize_kernel, 1, 0, true, st, partials, n, count, mse, err);
}

int64_t view_tiles(const Geometry& g) { return view_tile_count(g); }

}  // namespace fp4q
