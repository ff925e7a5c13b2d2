// Batch quantization: a chain of persistent kernels with programmatic
// dependent launch, one kernel per tensor.
//
// With the tensor scale computed (NVFP4 formats), kernel j of a batch of n
// tensors streams, interleaved in proportion to their tile counts:
//   - the quantize tiles of tensor j-1 (its tensor scale comes from the
//     absmax partials kernel j-1 wrote), and
//   - the absmax tiles of tensor j (partials for kernel j+1),
// and its CTA 0 turns the error partials of tensor j-2 into its MSE.  So the
// memory-bound absmax pass of one tensor runs inside the same SMs as the
// ALU-bound quantize pass of the previous one, every dependency crosses a
// kernel boundary (griddepcontrol.wait), and no CTA ever waits on another.
// Kernel 0 holds only absmax tiles, kernel n only quantize tiles, and kernel
// n+1 only finalises.  With the scale given, or for MXFP4, kernel j quantizes
// tensor j and finalises tensor j-1.
//
// Every kernel fetches its first tiles before waiting for its predecessor:
// all inputs were complete when the first kernel of the batch started, and a
// kernel lets its successor launch only after it has passed that wait, so a
// kernel never starts before its predecessor's predecessor has finished.
// Partial buffers rotate over three slots: kernel j reads slot j-1 and writes
// slot j, so a kernel overlapping its predecessor's tail never writes a slot
// that is still being read.  Tiles are assigned to CTAs by a fixed schedule,
// so every partial sum is formed in a fixed order.
//
// Method references (title, section): as fp4q_common.cuh.
#include <new>
#include <vector>

#include "fp4q_launch.cuh"

namespace fp4q {

constexpr int kRing = 3;   // rotating partial-buffer slots

// CTA shape of the chain: ten warps and tiles of 160 rows (20 KB), two CTAs
// per SM with up to 96 registers a thread, measured faster in every format
// than eight warps and 128 rows at three CTAs per SM (80 registers, where the
// RaZeR encoders spill) and than twelve warps and 192 rows at two per SM.
// Thread t owns unit (row t / 2, half t % 2), so threads = 2 x rows.  The
// shape is a parameter of the format so that one format can move alone.
template <int FMT>
struct ChainShape {
    static constexpr int kRows = 160;
    static constexpr int kThreads = 2 * kRows;
    static constexpr int kWarps = kThreads / 32;
    static constexpr int kCtasPerSm = 2;
    static constexpr int kStages = 4;
    static constexpr int kTileBytes = kRows * 128;
    static constexpr int kSmemBytes = pipe_smem_bytes(kTileBytes, kStages);
};

inline int chain_rows(int fmt) { return fmt == kRW ? ChainShape<kRW>::kRows : ChainShape<kRZ>::kRows; }
static_assert(ChainShape<kNV>::kRows == ChainShape<kRZ>::kRows && ChainShape<kMX>::kRows == ChainShape<kRZ>::kRows,
              "chain_rows gives the weight mode its own shape and one shape to the other formats");
static_assert(ChainShape<kRZ>::kRows % 8 == 0 && ChainShape<kRW>::kRows % 8 == 0,
              "a tile is whole 1024-byte swizzle atoms of 8 rows");
static_assert(ChainShape<kRZ>::kThreads <= 512 && ChainShape<kRW>::kThreads <= 512, "finaliser tree covers 512");
static_assert(ChainShape<kRZ>::kRows <= 256, "TMA box rows");

struct ChainArgs {
    // quantize part
    Tiles qtl;
    uint8_t* codes;
    uint8_t* scales;
    float* tensor_scale;
    const float* amax_in;   // absmax partials of the quantized tensor (computed scale)
    double* sse_out;        // this kernel's per-CTA error partials of the quantized tensor
    int32_t n_amax_in;
    int32_t has_q, q_flat, computed;
    // absmax part
    Tiles atl;
    float* amax_out;        // this kernel's per-CTA absmax partials
    int32_t has_a, a_flat;
    // finaliser part
    const double* sse_in;
    double* fin_mse;
    double fin_count;
    int32_t n_sse_in;
    int32_t has_fin;
    int32_t mx_ceil;
    unsigned* err;          // the library's device error words
};

template <int FMT, bool ROT, bool SSE>
__global__ void __launch_bounds__(ChainShape<FMT>::kThreads, ChainShape<FMT>::kCtasPerSm)
    chain_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap amap, ChainArgs a)
{
    using Shape = ChainShape<FMT>;
    constexpr int kThreads = Shape::kThreads;
    constexpr int kTileBytes = Shape::kTileBytes;
    constexpr int kRows = Shape::kRows;
    constexpr int kStages = Shape::kStages;
    extern __shared__ uint8_t smem_raw[];
    __shared__ float shf[32];
    __shared__ double shd[kThreads];
    __shared__ NvTable nvt;
    const Pipe p = pipe_setup<kTileBytes, Shape::kWarps, kStages>(smem_raw);
    const int t = threadIdx.x;

    // Items of this kernel: nq quantize tiles (walked backwards) and na absmax
    // tiles.  CTA b owns quantize tiles b, b + G, ... and absmax tiles
    // G-1-b, 2G-1-b, ... (so a CTA with one quantize tile more than another
    // tends to have one absmax tile less), and walks its two lists
    // interleaved in proportion to their lengths.  Each CTA thus gets an even
    // share of both kinds, whatever the parity of G.
    const int64_t nq = a.has_q ? a.qtl.count : 0;
    const int64_t na = a.has_a ? a.atl.count : 0;
    const int64_t G = gridDim.x, b = blockIdx.x, ab = G - 1 - b;
    const int64_t my_q = b < nq ? (nq - 1 - b) / G + 1 : 0;
    const int64_t my_a = ab < na ? (na - 1 - ab) / G + 1 : 0;
    const int64_t mine = my_q + my_a;
    // The items in order: before item jj come k = floor(jj my_q / mine)
    // quantize items, stepped without a division (rem = jj my_q - k mine, in
    // [0, mine); my_q <= mine, so one step adds at most one).  Thread 0 walks
    // the list kStages items ahead for the refills, and every thread walks its
    // own copy as it consumes the items, all in registers (item slots in shared
    // memory, or a shared-memory cursor, measured slower at 96 registers).
    int cur_k = 0, cur_rem = 0;   // fits: a tensor in device memory has fewer than 2^24 tiles
    auto next_item = [&](int64_t jj, bool& is_q, int64_t& tile) {
        const int64_t k0 = cur_k;
        cur_rem += (int)my_q;
        if (cur_rem >= (int)mine) {
            cur_rem -= (int)mine;
            ++cur_k;
        }
        is_q = cur_k > k0;
        tile = is_q ? nq - 1 - (b + k0 * G) : ab + (jj - k0) * G;
    };
    auto issue = [&](int64_t jj) {   // thread 0, for jj = 0, 1, 2, ... in order
        bool is_q;
        int64_t tile;
        next_item(jj, is_q, tile);
        const int s = (int)(jj % kStages);
        int x, y;
        if (is_q) {
            if (a.q_flat) tile_origin<true, kRows>(a.qtl, tile, x, y);
            else tile_origin<false, kRows>(a.qtl, tile, x, y);
        } else {
            if (a.a_flat) tile_origin<true, kRows>(a.atl, tile, x, y);
            else tile_origin<false, kRows>(a.atl, tile, x, y);
        }
        mbar_arm(p.full + 8 * s, kTileBytes);
        tma_load_tile(p.tiles + s * kTileBytes, is_q ? &qmap : &amap, x, y, p.full + 8 * s);
    };
    if (t == 0)
        for (int64_t jj = 0; jj < mine && jj < kStages; ++jj) issue(jj);
    pdl_wait();

    // Tensor scale of the quantized tensor, from its absmax partials.
    float s_t = 0.0f;
    if (a.has_q && FMT != kMX) {
        if (a.computed) {
            float mx = 0.0f;
            for (int i = t; i < a.n_amax_in; i += kThreads)
                if (in_bounds(4 * (int64_t)i, 4, 4 * (int64_t)kMaxPartials, kSiteAmaxPartialLoad, a.err))
                    mx = fmaxf(mx, a.amax_in[i]);
            mx = block_max(mx, shf);
            s_t = tensor_scale_of<FMT>(mx);
            if (b == 0 && t == 0) *a.tensor_scale = s_t;
        } else {
            s_t = *a.tensor_scale;
        }
    }
    // Finaliser: fixed-order sum of the previous kernel's error partials.
    if (a.has_fin && b == 0) {
        double s = 0.0;
        for (int i = t; i < a.n_sse_in; i += kThreads)
            if (in_bounds(8 * (int64_t)i, 8, 8 * (int64_t)kMaxPartials, kSiteSsePartialLoad, a.err)) s += a.sse_in[i];
        shd[t] = s;
        __syncthreads();
        for (int o = 256; o > 0; o >>= 1) {   // fixed-order tree over kThreads <= 512 partial sums
            if (t < o && t + o < kThreads) shd[t] += shd[t + o];
            __syncthreads();
        }
        if (t == 0) *a.fin_mse = a.fin_count > 0.0 ? shd[0] / a.fin_count : 0.0;
    }
    pdl_trigger();
    NvScale nsc{};
    if (a.has_q && FMT != kMX) nsc = nv_scale_setup<FMT>(s_t, &nvt);
    // Every thread finishes the prologue before the tile loop.
    __syncthreads();

    double acc = 0.0;
    float m = 0.0f;
    int ck = 0, crem = 0;   // this thread's copy of the item walk
    for (int64_t jj = 0; jj < mine; ++jj) {
        if (!pipe_acquire<kStages>(p, jj)) {
            pipe_fail<kStages>(p, jj, jj + kStages < mine ? jj + kStages : mine, a.err);
            break;
        }
        const int s = (int)(jj % kStages);
        const int ck0 = ck;
        crem += (int)my_q;
        if (crem >= (int)mine) {
            crem -= (int)mine;
            ++ck;
        }
        const bool is_q = ck > ck0;
        const int64_t tile = nq - 1 - (b + (int64_t)ck0 * G);   // used for quantize items only
        const uint32_t tp = p.tiles + (uint32_t)s * kTileBytes;
        if (is_q) {
            if (a.q_flat)
                acc += quantize_tile<FMT, ROT, SSE, true, kRows>(tp, a.qtl, tile, a.codes, a.scales, nsc,
                                                                 a.mx_ceil != 0, a.err);
            else
                acc += quantize_tile<FMT, ROT, SSE, false, kRows>(tp, a.qtl, tile, a.codes, a.scales, nsc,
                                                                  a.mx_ceil != 0, a.err);
        } else {
            m = fmaxf(m, amax_tile<ROT>(tp));
        }
        pipe_release<kStages>(p, jj);
        if (t == 0 && jj + kStages < mine) {
            if (!pipe_stage_free<kStages>(p, jj)) {
                pipe_fail<kStages>(p, jj + 1, jj + kStages, a.err);
                break;
            }
            issue(jj + kStages);
        }
    }
    if (a.has_a) {
        m = block_max(m, shf);
        if (t == 0 && in_bounds(4 * b, 4, 4 * (int64_t)kMaxPartials, kSiteAmaxPartialStore, a.err)) a.amax_out[b] = m;
    }
    if (a.has_q && SSE) {
        acc = block_sum(acc, shd);
        if (t == 0 && in_bounds(8 * b, 8, 8 * (int64_t)kMaxPartials, kSiteSsePartialStore, a.err)) a.sse_out[b] = acc;
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

namespace {

template <int FMT, bool ROT, bool SSE>
cudaError_t chain_go(const CUtensorMap& qmap, const CUtensorMap& amap, const ChainArgs& a, int64_t tiles, bool pdl,
                     int* grid_out, cudaStream_t st)
{
    using Shape = ChainShape<FMT>;
    auto kernel = chain_kernel<FMT, ROT, SSE>;
    const int grid = grid_for(kernel, Shape::kSmemBytes, tiles, Shape::kThreads);
    *grid_out = grid;
    return launch_threads(kernel, grid, Shape::kThreads, Shape::kSmemBytes, pdl, st, qmap, amap, a);
}

cudaError_t chain_dispatch(int fmt, bool rotate, bool sse, const CUtensorMap& qmap, const CUtensorMap& amap,
                           const ChainArgs& a, int64_t tiles, bool pdl, int* grid_out, cudaStream_t st)
{
    switch (fmt * 4 + (rotate ? 2 : 0) + (sse ? 1 : 0)) {
        case 0: return chain_go<kNV, false, false>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 1: return chain_go<kNV, false, true>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 2: return chain_go<kNV, true, false>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 3: return chain_go<kNV, true, true>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 4: return chain_go<kRZ, false, false>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 5: return chain_go<kRZ, false, true>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 6: return chain_go<kRZ, true, false>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 7: return chain_go<kRZ, true, true>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 8: return chain_go<kMX, false, false>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 9: return chain_go<kMX, false, true>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 10: return chain_go<kMX, true, false>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 11: return chain_go<kMX, true, true>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 12: return chain_go<kRW, false, false>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 13: return chain_go<kRW, false, true>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 14: return chain_go<kRW, true, false>(qmap, amap, a, tiles, pdl, grid_out, st);
        case 15: return chain_go<kRW, true, true>(qmap, amap, a, tiles, pdl, grid_out, st);
        default: return cudaErrorInvalidValue;
    }
}

struct View {
    CUtensorMap map;
    Tiles tl;
};

}  // namespace

size_t batch_workspace_bytes() { return (size_t)kRing * kMaxPartials * (sizeof(float) + sizeof(double)); }

cudaError_t launch_quantize_batch(const BatchTensor* ts, int n, int fmt, int rotate, int scale_given, int mx_ceil,
                                  void* workspace, cudaStream_t st, bool single_layout)
{
    if (n <= 0) return cudaSuccess;
    const bool computed = fmt != kMX && !scale_given;
    bool sse = false;
    for (int k = 0; k < n; ++k) sse = sse || ts[k].mse != nullptr;
    char* ws = static_cast<char*>(workspace);
    // One tensor needs one slot of each kind (launch 0 writes the absmax
    // partials that launch 1 reads; the launch that quantizes writes the error
    // partials the next one reads), so it fits the single-call workspace.
    single_layout = single_layout && n == 1;
    auto amax_slot = [&](int64_t j) {
        if (single_layout) return reinterpret_cast<float*>(ws + kWsAmaxOffset);
        return reinterpret_cast<float*>(ws + (j % kRing) * kMaxPartials * 4);
    };
    auto sse_slot = [&](int64_t j) {
        if (single_layout) return reinterpret_cast<double*>(ws + kWsSseOffset);
        return reinterpret_cast<double*>(ws + (size_t)kRing * kMaxPartials * 4 + (j % kRing) * kMaxPartials * 8);
    };
    std::vector<View> views((size_t)n);
    for (int k = 0; k < n; ++k) {
        const Geometry g = make_geometry(ts[k].rows, ts[k].cols, ts[k].ldx);
        if (!make_view(ts[k].x, g, &views[(size_t)k].map, &views[(size_t)k].tl, chain_rows(fmt)))
            return cudaErrorInvalidValue;
    }
    unsigned* err = device_error_words();
    if (err == nullptr) return cudaErrorInvalidSymbol;
    const int lag = computed ? 1 : 0;            // kernel j quantizes tensor j - lag
    std::vector<int> grids((size_t)n + 2, 0);    // CTAs (= partials written) of kernel j
    for (int64_t j = 0; j < n + lag + 1; ++j) {
        ChainArgs a = {};
        a.mx_ceil = mx_ceil;
        a.err = err;
        const int64_t kq = j - lag;              // tensor quantized by kernel j
        const int64_t ka = computed ? j : -1;    // tensor whose absmax pass kernel j runs
        const int64_t kf = j - lag - 1;          // tensor whose MSE kernel j finalises
        a.has_q = kq >= 0 && kq < n;
        a.has_a = ka >= 0 && ka < n;
        a.has_fin = kf >= 0 && kf < n && ts[kf].mse != nullptr;
        if (!a.has_q && !a.has_a && !a.has_fin) continue;
        const CUtensorMap* qmap = &views[0].map;
        const CUtensorMap* amap = &views[0].map;
        int64_t tiles = 0;
        if (a.has_q) {
            const View& v = views[(size_t)kq];
            qmap = &v.map;
            a.qtl = v.tl;
            a.q_flat = is_flat(v.tl) ? 1 : 0;
            a.codes = ts[kq].codes;
            a.scales = ts[kq].scales;
            a.tensor_scale = ts[kq].tensor_scale;
            a.computed = computed ? 1 : 0;
            if (computed) {
                a.amax_in = amax_slot(kq);
                a.n_amax_in = grids[(size_t)kq];
            }
            a.sse_out = sse_slot(j);
            tiles += v.tl.count;
        }
        if (a.has_a) {
            const View& v = views[(size_t)ka];
            amap = &v.map;
            a.atl = v.tl;
            a.a_flat = is_flat(v.tl) ? 1 : 0;
            a.amax_out = amax_slot(j);
            tiles += v.tl.count;
        }
        if (a.has_fin) {
            a.sse_in = sse_slot(j - 1);
            a.n_sse_in = grids[(size_t)(j - 1)];
            a.fin_count = (double)(ts[kf].rows * ts[kf].cols);
            a.fin_mse = ts[kf].mse;
        }
        int grid = 0;
        const cudaError_t e = chain_dispatch(fmt, rotate != 0, sse, *qmap, *amap, a, tiles, j > 0, &grid, st);
        if (e != cudaSuccess) return e;
        grids[(size_t)j] = grid;
    }
    return cudaSuccess;
}

}  // namespace fp4q
