// Tensor-core operand form of an NVFP4-family matrix, and the W4A4 product on
// the sm_100a block-scaled tensor cores (tcgen05.mma kind::mxf4nvf4).
//
// "RaZeR: Pushing the Limits of NVFP4 Quantization with Redundant Zero
// Remapping", technical summary sect. 2.3: on existing tensor cores the GEMM
// handles the remapped code with two passes.  Here the operand form splits a
// RaZeR matrix into two code planes whose decoded sum is the reconstruction:
// plane 0 reads every special value s as its base b (the largest E2M1
// magnitude below |s|, signed: +-4 for +-5, +-2 for +-2.5), plane 1 holds
// s - b at those elements and +0 elsewhere.  The tensor core reads code
// 0b1000 as -0, so without the split it would drop the special values.  The
// product of an A with pa planes and a W with pw planes is the sum of the
// pa * pw plane products; the kernel runs them as one accumulation over
// pa * pw * K, the "passes".
//
// Scale bytes go to the layout the tensor core reads through tcgen05.cp
// (32 x 128-bit, replicated to the four lane quadrants): 512-byte atoms of
// 128 rows x 4 blocks, byte (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4.
//
// GEMM kernel: persistent, two CTAs per SM walking 128 x 128 output tiles, 6
// warps each.  Thread 0 streams k-tiles of 256 elements (A 16 KB, W 16 KB,
// scale atoms 4 KB) through a 3-stage ring with TMA (128-byte swizzle, each CTA
// loading its own tiles), running ahead across tile boundaries; thread 32
// copies the scale atoms of a landed stage into tensor memory and issues the
// four 128 x 128 x 64 MMAs, then commits the stage back to the producer; warps
// 2-5 read a finished fp32 accumulator from tensor memory (each warp its lane
// quadrant), scale it by s_a * s_w, store bf16 and hand the accumulator back.
// Two CTAs per SM (111 KB of shared memory and 256 tensor-memory columns each)
// keep two MMA streams per SM; one CTA of 128 x 256 tiles ran 8-11 % slower.
// Every wait is bounded; a CTA that gives up records kErrPipelineTimeout,
// waits (bounded) for its copies and MMAs, frees its tensor memory and
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fp4q_launch.cuh"

namespace fp4q {

// ---------------------------------------------------------------------------
// Operand form
// ---------------------------------------------------------------------------

struct PackArgs {
    const uint8_t* codes;
    const uint8_t* scales;
    uint8_t* planes;
    uint8_t* sf;
    int64_t rows, cols;
    int64_t rows_pad, nb, nb_pad;   // rows padded to 128, blocks per row, blocks padded to 4
    unsigned* err;                  // the library's device error words
};

// Bit 0 of every nibble of w that equals 0b1000.
__device__ __forceinline__ uint32_t nibbles_eq8(uint32_t w)
{
    const uint32_t t = w ^ 0x88888888u;                          // zero nibbles where w == 8
    const uint32_t z = ~(((t & 0x77777777u) + 0x77777777u) | t) & 0x88888888u;
    return z >> 3;
}

// One thread per (row, block) of the padded scale grid: the block's 8 code
// bytes to its plane(s), its scale byte to the atom; padding gets 0.
template <int FMT>
__global__ void __launch_bounds__(256) mma_pack_kernel(PackArgs a)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.rows_pad * a.nb_pad) return;
    const int64_t r = i / a.nb_pad, kb = i - r * a.nb_pad;
    const int64_t atoms = a.nb_pad / 4;
    const int64_t off = ((r / 128) * atoms + kb / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4;
    const int64_t sf_bytes = (a.rows_pad / 128) * (a.nb_pad / 4) * 512, n = a.rows * a.cols;
    constexpr int P = kRazer<FMT> ? 2 : 1;
    if (!in_bounds(off, 1, sf_bytes, kSiteSfStore, a.err)) return;
    if (r >= a.rows || kb >= a.nb) {
        a.sf[off] = 0;
        return;
    }
    if (!in_bounds(r * a.nb + kb, 1, n / 16, kSiteScalesLoad, a.err) ||
        !in_bounds(r * (a.cols / 2) + 8 * kb, 8, n / 2, kSiteCodesLoad, a.err) ||
        !in_bounds(r * P * (a.cols / 2) + 8 * kb, P == 1 ? 8 : a.cols / 2 + 8, P * n / 2, kSitePlanesStore, a.err))
        return;
    const uint32_t sb = a.scales[r * a.nb + kb];
    const uint2 c = *reinterpret_cast<const uint2*>(a.codes + r * (a.cols / 2) + 8 * kb);
    uint32_t mag;
    if (FMT == kRW) mag = e4m3_rn_satfinite(e3m3_to_f32(sb & 0x3Fu));   // exact: E3M3 values are E4M3 values
    else if (FMT == kRZ) mag = sb & 0x7Fu;
    else mag = sb;
    a.sf[off] = (uint8_t)mag;
    if (!kRazer<FMT>) {
        *reinterpret_cast<uint2*>(a.planes + r * (a.cols / 2) + 8 * kb) = c;
        return;
    }
    // base / residual codes of this block's special value
    uint32_t base, res;
    if (FMT == kRZ) {
        const uint32_t sg = (sb & 0x80u) ? 8u : 0u;
        base = 0x6u | sg;                                          // +-4
        res = 0x2u | sg;                                           // +-1
    } else {
        const uint32_t sg = (sb & 0x40u) ? 8u : 0u;
        const bool p2 = (sb & 0x80u) != 0u;
        base = (p2 ? 0x4u : 0x6u) | sg;                            // +-2 or +-4
        res = (p2 ? 0x1u : 0x2u) | sg;                             // +-0.5 or +-1
    }
    const uint32_t m0 = nibbles_eq8(c.x) * 15u, m1 = nibbles_eq8(c.y) * 15u;
    uint8_t* row = a.planes + r * a.cols;                          // two planes of cols/2 bytes
    *reinterpret_cast<uint2*>(row + 8 * kb) =
        make_uint2((c.x & ~m0) | ((base * 0x11111111u) & m0), (c.y & ~m1) | ((base * 0x11111111u) & m1));
    *reinterpret_cast<uint2*>(row + a.cols / 2 + 8 * kb) =
        make_uint2((res * 0x11111111u) & m0, (res * 0x11111111u) & m1);
}

int64_t mma_sf_bytes(int64_t rows, int64_t cols) { return ((rows + 127) / 128) * ((cols / 16 + 3) / 4) * 512; }

cudaError_t launch_mma_pack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, int fmt,
                            uint8_t* planes, uint8_t* sf, cudaStream_t st)
{
    PackArgs a;
    a.codes = codes;
    a.scales = scales;
    a.planes = planes;
    a.sf = sf;
    a.rows = rows;
    a.cols = cols;
    a.rows_pad = (rows + 127) / 128 * 128;
    a.nb = cols / 16;
    a.nb_pad = (a.nb + 3) / 4 * 4;
    if ((a.err = device_error_words()) == nullptr) return cudaErrorInvalidSymbol;
    const int64_t n = a.rows_pad * a.nb_pad;
    if (n == 0) return cudaSuccess;
    const int64_t blocks = (n + 255) / 256;
    if (blocks >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    switch (fmt) {
        case kNV: mma_pack_kernel<kNV><<<(unsigned)blocks, 256, 0, st>>>(a); break;
        case kRZ: mma_pack_kernel<kRZ><<<(unsigned)blocks, 256, 0, st>>>(a); break;
        case kRW: mma_pack_kernel<kRW><<<(unsigned)blocks, 256, 0, st>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// tcgen05 helpers
// ---------------------------------------------------------------------------

namespace tc {

constexpr int kBM = 128, kBN = 128, kBK = 256;       // tile: rows of A, rows of W, elements of K
constexpr int kStagesG = 3;
constexpr int kCtasPerSm = 2;
constexpr int kABytes = kBM * kBK / 2;               // 16 KB
constexpr int kBBytes = kBN * kBK / 2;               // 16 KB
constexpr int kSfaBytes = (kBM / 128) * (kBK / 64) * 512;   // 2 KB
constexpr int kSfbBytes = (kBN / 128) * (kBK / 64) * 512;   // 2 KB
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr int kEpilogueWarps = 4;
constexpr int kGemmThreads = 64 + 32 * kEpilogueWarps;   // loader warp, MMA warp, epilogue warps
constexpr int kTmemCols = 256;
// Tensor-memory columns: accumulator 0..127, then per stage s the scale
// factors of that stage's k-tile (A 16 columns, W 16: four MMAs of 4 columns
// each), so that copying the next stage's scales never waits for the MMAs
// reading this stage's.
constexpr uint32_t kTmemSf0 = kBN;
constexpr uint32_t kTmemSfStage = 32;
constexpr uint32_t kTmemSfbOff = 16;
static_assert(kTmemSf0 + kStagesG * kTmemSfStage <= (uint32_t)kTmemCols, "scale factors exceed the allocation");
constexpr int kGemmSmem = kStagesG * kStageBytes + 1024 + 256;

// Instruction descriptor of kind::mxf4nvf4 with 16-element UE4M3 scales:
// A and B E2M1 (format 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: start >> 4,
// leading offset 1 (unused with the swizzle), stride 1024 B between 8-row
// groups, descriptor version 1, layout type 2.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// Descriptor of a 32-row x 16-byte scale atom (rows 16 B apart, no swizzle,
// 8-row groups 128 B apart) for tcgen05.cp.
__device__ __forceinline__ uint64_t desc_atom(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 32) | (1ull << 46);
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void copy_atom_to_tmem(uint32_t taddr, uint64_t desc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ void mma_block16(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa, uint32_t sfb, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(kIdesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
}

// Arrive on `bar` once every MMA and copy this thread issued before has completed.
__device__ __forceinline__ void commit_to(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's lane quadrant.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace tc

struct GemmArgs {
    const uint8_t* a_sf;
    const uint8_t* w_sf;
    const float* a_scale;
    const float* w_scale;
    uint16_t* y;
    int64_t M, N, K, ldy;
    int32_t a_planes, w_planes;
    unsigned* err;          // the library's device error words
};

// Y[m][n] = s_a s_w sum over plane pairs and k of A_p[m][k] W_q[n][k].
// Persistent: CTA b of G takes output tiles b, b + G, ...  Warp 0 (one thread)
// loads, warp 1 (one thread) issues the MMAs and owns the tensor memory,
// warps 2-5 drain the accumulator (warp w reads lane quadrant w % 4).  The
// loads run ahead across tile boundaries; the MMAs of a tile wait until the
// previous tile's accumulator has been read ("acc_empty").
__global__ void __launch_bounds__(tc::kGemmThreads, tc::kCtasPerSm)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap wmap, GemmArgs g)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[2 * kStagesG + 3];   // full[s], empty[s], acc_full, acc_empty, drain
    __shared__ uint32_t tmem_base_sh;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int64_t n_tiles_n = (g.N + kBN - 1) / kBN;
    const int64_t n_tiles = ((g.M + kBM - 1) / kBM) * n_tiles_n;
    const int64_t my_tiles = (int64_t)blockIdx.x < n_tiles ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t bar0 = smem_u32(bars);
    auto full = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bar0 + 8u * (uint32_t)(kStagesG + s); };
    const uint32_t acc_full = bar0 + 8u * (uint32_t)(2 * kStagesG);
    const uint32_t acc_empty = acc_full + 8u;
    const uint32_t drain = acc_full + 16u;
    auto stage_a = [&](int s) { return base + (uint32_t)(s * kStageBytes); };
    auto stage_b = [&](int s) { return stage_a(s) + kABytes; };
    auto stage_sfa = [&](int s) { return stage_b(s) + kBBytes; };
    auto stage_sfb = [&](int s) { return stage_sfa(s) + kSfaBytes; };

    if (t == 0) {
        for (int s = 0; s < kStagesG; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpilogueWarps);
        mbar_init(drain, 1);
        mbar_init_fence();
    }
    if (warp == 1) {
        const uint32_t dst = smem_u32(&tmem_base_sh);
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base_sh;

    const int64_t kt_per_seg = g.K / kBK;
    const int64_t iters = kt_per_seg * g.a_planes * g.w_planes;   // k-tiles per output tile
    const int64_t atoms_k = g.K / 64;                       // scale atoms per 128-row block
    const int64_t half_k = g.K / 2;                         // bytes of one plane row
    auto tile_mn = [&](int64_t j, int64_t& mt, int64_t& nt) {
        const int64_t tile = (int64_t)blockIdx.x + j * gridDim.x;
        mt = tile / n_tiles_n;
        nt = tile - mt * n_tiles_n;
    };

    if (t == 0) {
        // ---- producer: k-tiles of every output tile, one ring across tiles ----
        int64_t gi = 0;   // k-tiles issued so far
        bool ok = true;
        for (int64_t j = 0; j < my_tiles && ok; ++j) {
            int64_t mt, nt;
            tile_mn(j, mt, nt);
            const uint32_t tx = (uint32_t)(kABytes + kBBytes + kSfaBytes + kSfbBytes);
            for (int64_t i = 0; i < iters; ++i, ++gi) {
                const int s = (int)(gi % kStagesG);
                if (gi >= kStagesG && !mbar_wait(empty(s), (uint32_t)(((gi / kStagesG) - 1) & 1))) {
                    ok = false;
                    break;
                }
                const int64_t seg = i / kt_per_seg, kt = i - seg * kt_per_seg;
                const int64_t pa = seg % g.a_planes, pw = seg / g.a_planes;
                mbar_arm(full(s), tx);
                tc::tma_load_2d(stage_a(s), &amap, (int)(pa * half_k + kt * (kBK / 2)), (int)(mt * kBM), full(s));
                tc::tma_load_2d(stage_b(s), &wmap, (int)(pw * half_k + kt * (kBK / 2)), (int)(nt * kBN), full(s));
                tc::bulk_load(stage_sfa(s), g.a_sf + (mt * atoms_k + 4 * kt) * 512, kSfaBytes, full(s));
                tc::bulk_load(stage_sfb(s), g.w_sf + (nt * atoms_k + 4 * kt) * 512, kSfbBytes, full(s));
            }
        }
        if (!ok) {
            atomicOr(g.err, kErrPipelineTimeout);
            for (int64_t q = gi - kStagesG < 0 ? 0 : gi - kStagesG; q < gi; ++q)   // copies still in flight
                mbar_wait(full((int)(q % kStagesG)), (uint32_t)((q / kStagesG) & 1));
        }
    } else if (t == 32) {
        // ---- MMA issuer ----
        int64_t gi = 0;
        bool ok = true;
        for (int64_t j = 0; j < my_tiles && ok; ++j) {
            if (j > 0 && !mbar_wait(acc_empty, (uint32_t)((j - 1) & 1))) {   // previous accumulator drained
                ok = false;
                break;
            }
            tc::fence_after_sync();
            for (int64_t i = 0; i < iters; ++i, ++gi) {
                const int s = (int)(gi % kStagesG);
                if (!mbar_wait(full(s), (uint32_t)((gi / kStagesG) & 1))) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                // scale atoms -> tensor memory: 4 columns per MMA for A and for W
                const uint32_t sfa = tmem + kTmemSf0 + kTmemSfStage * (uint32_t)s, sfb = sfa + kTmemSfbOff;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    tc::copy_atom_to_tmem(sfa + 4u * q, tc::desc_atom(stage_sfa(s) + 512u * q));
                    tc::copy_atom_to_tmem(sfb + 4u * q, tc::desc_atom(stage_sfb(s) + 512u * q));
                }
                const uint64_t da = tc::desc_sw128(stage_a(s)), db = tc::desc_sw128(stage_b(s));
#pragma unroll
                for (int q = 0; q < 4; ++q)   // K = 64 per MMA: 32 bytes along the swizzled row
                    tc::mma_block16(tmem, da + 2u * q, db + 2u * q, sfa + 4u * q, sfb + 4u * q,
                                    (i > 0 || q > 0) ? 1u : 0u);
                tc::commit_to(empty(s));
            }
            if (ok) tc::commit_to(acc_full);   // arrives when the tile's MMAs have completed
        }
        if (!ok) {
            atomicOr(g.err, kErrPipelineTimeout);
            tc::commit_to(drain);              // wait (bounded) for the MMAs issued so far
            mbar_wait(drain, 0u);
        }
    } else if (warp >= 2) {
        // ---- epilogue: warp w reads accumulator rows 32 (w % 4) .. + 31 ----
        const int quad = warp & 3;
        const float alpha = __fmul_rn(*g.a_scale, *g.w_scale);
        const uint32_t trow = tmem + ((uint32_t)(32 * quad) << 16);
        for (int64_t j = 0; j < my_tiles; ++j) {
            if (!mbar_wait(acc_full, (uint32_t)(j & 1))) {
                if (lane == 0) atomicOr(g.err, kErrPipelineTimeout);
                break;
            }
            tc::fence_after_sync();
            int64_t mt, nt;
            tile_mn(j, mt, nt);
            const int64_t m = mt * kBM + 32 * quad + lane, n0 = nt * kBN;
#pragma unroll 1
            for (int c = 0; c < kBN; c += 32) {
                if (n0 + c >= g.N) break;   // uniform across the warp
                float v[32];
                tc::tmem_ld32(trow + (uint32_t)c, v);
                if (m < g.M && in_bounds(2 * (m * g.ldy + n0 + c), 2 * (g.N - n0 - c < 32 ? g.N - n0 - c : 32),
                                         2 * ((g.M - 1) * g.ldy + g.N), kSiteGemmStore, g.err)) {
                    uint16_t* yrow = g.y + m * g.ldy + n0 + c;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (n0 + c + 8 * q >= g.N) break;
                        uint4 o;
                        o.x = pack_bf16x2_rn(__fmul_rn(alpha, v[8 * q + 0]), __fmul_rn(alpha, v[8 * q + 1]));
                        o.y = pack_bf16x2_rn(__fmul_rn(alpha, v[8 * q + 2]), __fmul_rn(alpha, v[8 * q + 3]));
                        o.z = pack_bf16x2_rn(__fmul_rn(alpha, v[8 * q + 4]), __fmul_rn(alpha, v[8 * q + 5]));
                        o.w = pack_bf16x2_rn(__fmul_rn(alpha, v[8 * q + 6]), __fmul_rn(alpha, v[8 * q + 7]));
                        *reinterpret_cast<uint4*>(yrow + 8 * q) = o;
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acc_empty) : "memory");
        }
    }
    __syncwarp();
    // Every MMA has completed here: the epilogue waited for each tile's commit,
    // or the MMA thread drained its own after a failure.
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// 2-D uint8 tensor map over a [rows][inner] byte matrix, box {128 bytes, box_rows}, 128-byte swizzle.
static bool make_byte_map(CUtensorMap* map, const void* base, int64_t inner, int64_t rows, int box_rows)
{
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)inner};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemm_w4a4(const uint8_t* a_planes, const uint8_t* a_sf, int a_np, const float* a_scale,
                             const uint8_t* w_planes, const uint8_t* w_sf, int w_np, const float* w_scale, int64_t M,
                             int64_t N, int64_t K, uint16_t* y, int64_t ldy, cudaStream_t st)
{
    using namespace tc;
    if (M == 0 || N == 0) return cudaSuccess;
    CUtensorMap amap, wmap;
    if (!make_byte_map(&amap, a_planes, a_np * K / 2, M, kBM)) return cudaErrorInvalidValue;
    if (!make_byte_map(&wmap, w_planes, w_np * K / 2, N, kBN)) return cudaErrorInvalidValue;
    GemmArgs g;
    g.a_sf = a_sf;
    g.w_sf = w_sf;
    g.a_scale = a_scale;
    g.w_scale = w_scale;
    g.y = y;
    g.M = M;
    g.N = N;
    g.K = K;
    g.ldy = ldy;
    g.a_planes = a_np;
    g.w_planes = w_np;
    if ((g.err = device_error_words()) == nullptr) return cudaErrorInvalidSymbol;
    const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
    if (tiles >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const int64_t cap = (int64_t)kCtasPerSm * sm_count();           // persistent: two CTAs per SM
    const int64_t grid = tiles < cap ? tiles : cap;
    const cudaError_t e = cudaFuncSetAttribute(gemm_w4a4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               kGemmSmem);
    if (e != cudaSuccess) return e;
    gemm_w4a4_kernel<<<(unsigned)grid, kGemmThreads, kGemmSmem, st>>>(amap, wmap, g);
    return cudaGetLastError();
}

}  // namespace fp4q
