// fp4q kernels for sm_100a: tensor absmax, fused quantize, dequantize, error,
// and the fixed-order fp64 finaliser for the squared-error sums.
//
// Work decomposition.  A bf16 matrix is a sequence of 16-element halves (one
// NVFP4 block each); one thread owns a unit of two consecutive halves, i.e.
// 32 elements = 64 bytes of input, 16 bytes of codes and 2 (NVFP4) or 1
// (MXFP4) scale bytes.  With rotation or MXFP4 the two halves are one aligned
// 32-group of a row, so the whole Walsh-Hadamard butterfly runs in the
// thread's registers.  Consecutive lanes own consecutive units, so each warp
// streams 2 KB of input and writes 512 contiguous bytes of codes per step.
// Kernels are grid-strided over units with a grid sized to the resident
// capacity of the device.
//
// Method references (title, section):
//  "RaZeR: Pushing the Limits of NVFP4 Quantization with Redundant Zero
//   Remapping": sect. 1 (E2M1 set, E4M3 block scale from the block absmax,
//   unused scale sign bit), sect. 2.2 (-0 code remapped to a special value
//   chosen per block by minimum squared error; one bit -> the pair +-5).
//  "TORQ: Two-Level Orthogonal Rotation for MXFP4 Quantization": sect. 1
//   (32-element blocks, shared exponent, e2m1 codebook), sect. 2 (orthogonal
//   intra-block rotation before quantization; S-step maps the block maximum
//   to the top of the code range).
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "fp4q_device.cuh"
#include "fp4q_internal.h"

namespace fp4q {

enum { kNV = 0, kRZ = 1, kMX = 2 };

// ---------------------------------------------------------------------------
// Geometry helpers
// ---------------------------------------------------------------------------

// Element offset of half h.  CONTIG: rows are packed (ld == cols).
template <bool CONTIG>
__device__ __forceinline__ int64_t half_offset(const Geometry& g, int64_t h)
{
    if (CONTIG) return h * 16;
    int64_t row = h / g.halves_per_row;
    int64_t c = h - row * g.halves_per_row;
    return row * g.ld + c * 16;
}

// Load the 32 bf16 of unit u as 16 words.  PAIRED: both halves are known to
// lie in one row (cols a multiple of 32), so the second half follows the first.
template <bool CONTIG, bool PAIRED>
__device__ __forceinline__ void load_unit(const uint16_t* __restrict__ x, const Geometry& g, int64_t u,
                                          bool full, uint32_t* w)
{
    const int64_t h0 = 2 * u;
    const uint16_t* p0 = x + half_offset<CONTIG>(g, h0);
    uint4 a = ldg_nc_v4(p0), b = ldg_nc_v4(p0 + 8);
    uint4 c = make_uint4(0, 0, 0, 0), d = make_uint4(0, 0, 0, 0);
    if (full) {
        const uint16_t* p1 = (CONTIG || PAIRED) ? p0 + 16 : x + half_offset<CONTIG>(g, h0 + 1);
        c = ldg_nc_v4(p1);
        d = ldg_nc_v4(p1 + 8);
    }
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    w[8] = c.x; w[9] = c.y; w[10] = c.z; w[11] = c.w;
    w[12] = d.x; w[13] = d.y; w[14] = d.z; w[15] = d.w;
}

__device__ __forceinline__ void unpack32(const uint32_t* w, float* y)
{
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        y[2 * k] = bf16_lo(w[k]);
        y[2 * k + 1] = bf16_hi(w[k]);
    }
}

// ---------------------------------------------------------------------------
// Block reductions (fixed order within a CTA)
// ---------------------------------------------------------------------------

__device__ __forceinline__ float block_max(float v, float* sh)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) sh[warp] = v;
    __syncthreads();
    v = (threadIdx.x < (blockDim.x >> 5)) ? sh[threadIdx.x] : 0.0f;
    if (warp == 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if (lane == 0) sh[0] = v;
    }
    __syncthreads();
    return sh[0];
}

__device__ __forceinline__ double block_sum(double v, double* sh)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) sh[warp] = v;
    __syncthreads();
    v = (threadIdx.x < (blockDim.x >> 5)) ? sh[threadIdx.x] : 0.0;
    if (warp == 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    }
    return v;  // valid in thread 0
}

// ---------------------------------------------------------------------------
// Per-block encoders
// ---------------------------------------------------------------------------

// One 16-element NVFP4 block.  y: the (rotated) values; s_t / six_st: tensor
// scale and RN(6 s_t).  Writes two code words and the scale byte; with SSE,
// xh receives the fp32 reconstruction RN(q * den).
template <bool RAZER, bool SSE>
__device__ __forceinline__ void encode_nv16(const float* y, float s_t, float six_st, uint32_t* cw,
                                            uint32_t& sb_out, float* xh)
{
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(y[i]));
    const float t = six_st > 0.0f ? __fdiv_rn(a, six_st) : 0.0f;
    uint32_t sb = e4m3_rn_satfinite(t);
    const float den = __fmul_rn(e4m3_to_f32(sb), s_t);
    const float r = den != 0.0f ? __frcp_rn(den) : 0.0f;   // zero scale -> every code 0
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(y[i], r);
    uint32_t w0 = canonical_zero(e2m1x8(v));
    uint32_t w1 = canonical_zero(e2m1x8(v + 8));

    float q[16];
    if (SSE) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 p = e2m1x2_to_f32((w0 >> (8 * k)) & 0xFFu);
            q[2 * k] = p.x; q[2 * k + 1] = p.y;
            float2 s = e2m1x2_to_f32((w1 >> (8 * k)) & 0xFFu);
            q[8 + 2 * k] = s.x; q[8 + 2 * k + 1] = s.y;
        }
    }

    if (RAZER) {
        // Gain of remapping element i to sign(v_i) * 5: for |v_i| in (4.5, 5.5)
        // the regular value is 4 (|v| <= 5) or 6, and
        //   (|v| - q)^2 - (|v| - 5)^2 = 1 - 2 | |v| - 5 |,
        // positive exactly on that open interval and clamped to 0 elsewhere.
        // Every term is a multiple of 2^-20 in [0, 1], so the fp32 sums below
        // are exact in any order.  S = gain(+5) - gain(-5), T = gain(+5) + gain(-5).
        float S = 0.0f, T = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float c = __saturatef(__fmaf_rn(-2.0f, fabsf(fabsf(v[i]) - 5.0f), 1.0f));
            S += copysignf(c, v[i]);
            T += c;
        }
        if (T > 0.0f) {
            const bool neg = S < 0.0f;   // -5 only when strictly better
            uint32_t m0 = 0, m1 = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float c = __saturatef(__fmaf_rn(-2.0f, fabsf(fabsf(v[i]) - 5.0f), 1.0f));
                const bool win = c > 0.0f && (signbit(v[i]) != 0) == neg;
                if (win) {
                    if (i < 8) m0 |= 0xFu << (4 * i);
                    else m1 |= 0xFu << (4 * (i - 8));
                    if (SSE) q[i] = neg ? -5.0f : 5.0f;
                }
            }
            w0 = (w0 & ~m0) | (m0 & 0x88888888u);
            w1 = (w1 & ~m1) | (m1 & 0x88888888u);
            if (neg) sb |= 0x80u;
        }
    }
    if (SSE) {
#pragma unroll
        for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(q[i], den);
    }
    cw[0] = w0;
    cw[1] = w1;
    sb_out = sb;
}

// One 32-element MXFP4 block.
template <bool SSE>
__device__ __forceinline__ void encode_mx32(const float* y, uint32_t* cw, uint32_t& sb_out, float* xh)
{
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(y[i]));
    int e = -127;
    float r = 0.0f;
    uint32_t sb = 0;
    if (a > 0.0f) {
        e = floor_log2_f32(a) - 2;          // 2 = exponent of the largest E2M1 value
        e = e < -127 ? -127 : (e > 127 ? 127 : e);
        sb = (uint32_t)(e + 127);
        r = exp2i(-e);
    }
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(y[i], r);
#pragma unroll
    for (int k = 0; k < 4; ++k) cw[k] = canonical_zero(e2m1x8(v + 8 * k));
    if (SSE) {
        const float s = exp2i(e);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float2 p = e2m1x2_to_f32((cw[k] >> (8 * j)) & 0xFFu);
                xh[8 * k + 2 * j] = __fmul_rn(p.x, s);
                xh[8 * k + 2 * j + 1] = __fmul_rn(p.y, s);
            }
        }
    }
    sb_out = sb;
}

// ---------------------------------------------------------------------------
// Decoders (shared by dequantize and error)
// ---------------------------------------------------------------------------

template <bool RAZER>
__device__ __forceinline__ void decode_nv16(uint32_t w0, uint32_t w1, uint32_t sb, float s_t, float* xh)
{
    const float den = __fmul_rn(e4m3_to_f32(RAZER ? (sb & 0x7Fu) : sb), s_t);
    const float special = (sb & 0x80u) ? -5.0f : 5.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t b0 = (w0 >> (8 * k)) & 0xFFu, b1 = (w1 >> (8 * k)) & 0xFFu;
        float2 p = e2m1x2_to_f32(b0);
        float2 s = e2m1x2_to_f32(b1);
        if (RAZER) {
            if ((b0 & 0xFu) == 8u) p.x = special;
            if ((b0 >> 4) == 8u) p.y = special;
            if ((b1 & 0xFu) == 8u) s.x = special;
            if ((b1 >> 4) == 8u) s.y = special;
        }
        xh[2 * k] = __fmul_rn(p.x, den);
        xh[2 * k + 1] = __fmul_rn(p.y, den);
        xh[8 + 2 * k] = __fmul_rn(s.x, den);
        xh[8 + 2 * k + 1] = __fmul_rn(s.y, den);
    }
}

__device__ __forceinline__ void decode_mx32(const uint32_t* cw, uint32_t sb, float* xh)
{
    const float s = exp2i((int)sb - 127);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float2 p = e2m1x2_to_f32((cw[k] >> (8 * j)) & 0xFFu);
            xh[8 * k + 2 * j] = __fmul_rn(p.x, s);
            xh[8 * k + 2 * j + 1] = __fmul_rn(p.y, s);
        }
    }
}

// Read the codes and scale bytes of unit u (dense layouts).
template <int FMT>
__device__ __forceinline__ void load_packed(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                            int64_t u, bool full, uint32_t* cw, uint32_t* sb)
{
    if (full) {
        uint4 c = ldg_nc_v4(codes + 16 * u);
        cw[0] = c.x; cw[1] = c.y; cw[2] = c.z; cw[3] = c.w;
    } else {
        uint2 c = *reinterpret_cast<const uint2*>(codes + 16 * u);
        cw[0] = c.x; cw[1] = c.y; cw[2] = 0; cw[3] = 0;
    }
    if (FMT == kMX) {
        sb[0] = __ldg(scales + u);
        sb[1] = 0;
    } else if (full) {
        const uint32_t two = __ldg(reinterpret_cast<const unsigned short*>(scales) + u);
        sb[0] = two & 0xFFu;
        sb[1] = two >> 8;
    } else {
        sb[0] = __ldg(scales + 2 * u);
        sb[1] = 0;
    }
}

template <int FMT>
__device__ __forceinline__ void decode_unit(const uint32_t* cw, const uint32_t* sb, float s_t, float* xh)
{
    if (FMT == kMX) {
        decode_mx32(cw, sb[0], xh);
    } else {
        decode_nv16<FMT == kRZ>(cw[0], cw[1], sb[0], s_t, xh);
        decode_nv16<FMT == kRZ>(cw[2], cw[3], sb[1], s_t, xh + 16);
    }
}

// Sum of squared errors of one unit.  The fast path squares and sums in fp32;
// a unit whose fp32 sum overflowed or may have lost terms to underflow (|x| near
// the top of the bf16 range, or bf16 subnormals) is recomputed in fp64.
__device__ __forceinline__ double unit_sse(const uint32_t* w, const float* xh)
{
    float e = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float d0 = bf16_lo(w[k]) - xh[2 * k];
        const float d1 = bf16_hi(w[k]) - xh[2 * k + 1];
        e = __fmaf_rn(d0, d0, e);
        e = __fmaf_rn(d1, d1, e);
    }
    if (e < 0x1p-100f || !(e <= 3.0e38f)) {
        double ed = 0.0;
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
            const double d0 = (double)bf16_lo(w[k]) - (double)xh[2 * k];
            const double d1 = (double)bf16_hi(w[k]) - (double)xh[2 * k + 1];
            ed = fma(d0, d0, ed);
            ed = fma(d1, d1, ed);
        }
        return ed;
    }
    return (double)e;
}

// ---------------------------------------------------------------------------
// Kernels
// ---------------------------------------------------------------------------

struct AmaxArgs {
    const uint16_t* x;
    Geometry g;
    float* partials;
};

template <bool ROT, bool CONTIG, bool PAIRED>
__global__ void __launch_bounds__(kThreads) amax_kernel(AmaxArgs a)
{
    __shared__ float sh[32];
    float m = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < a.g.units; u += stride) {
        const bool full = 2 * u + 1 < a.g.halves;
        uint32_t w[16];
        load_unit<CONTIG, PAIRED>(a.x, a.g, u, full, w);
        float y[32];
        unpack32(w, y);
        if (ROT) wht32_inplace(y);
#pragma unroll
        for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(y[i]));
    }
    m = block_max(m, sh);
    if (threadIdx.x == 0) a.partials[blockIdx.x] = m;
}

struct QuantArgs {
    const uint16_t* x;
    Geometry g;
    uint8_t* codes;
    uint8_t* scales;
    float* tensor_scale;
    const float* amax_partials;
    int n_amax;
    int scale_given;
    double* sse_partials;
};

template <int FMT, bool ROT, bool SSE, bool CONTIG>
__global__ void __launch_bounds__(kThreads) quantize_kernel(QuantArgs a)
{
    constexpr bool PAIRED = (FMT == kMX) || ROT;
    __shared__ float shf[32];
    __shared__ double shd[32];

    // Tensor scale (NVFP4 formats): s_t = RN(A / (6 * 448)), A reduced from
    // the absmax pass's per-CTA maxima in every CTA.
    float s_t = 0.0f;
    if (FMT != kMX) {
        if (a.scale_given) {
            s_t = *a.tensor_scale;
        } else {
            float m = 0.0f;
            for (int i = threadIdx.x; i < a.n_amax; i += kThreads) m = fmaxf(m, a.amax_partials[i]);
            m = block_max(m, shf);
            s_t = __fdiv_rn(m, 2688.0f);
            if (blockIdx.x == 0 && threadIdx.x == 0) *a.tensor_scale = s_t;
        }
    }
    const float six_st = __fmul_rn(6.0f, s_t);

    double acc = 0.0;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < a.g.units; u += stride) {
        const bool full = 2 * u + 1 < a.g.halves;
        uint32_t w[16];
        load_unit<CONTIG, PAIRED>(a.x, a.g, u, full, w);
        float y[32];
        unpack32(w, y);
        if (ROT) wht32_inplace(y);

        uint32_t cw[4], sb0, sb1 = 0;
        float xh[32];
        if (FMT == kMX) {
            encode_mx32<SSE>(y, cw, sb0, xh);
        } else {
            encode_nv16<FMT == kRZ, SSE>(y, s_t, six_st, cw, sb0, xh);
            encode_nv16<FMT == kRZ, SSE>(y + 16, s_t, six_st, cw + 2, sb1, xh + 16);
        }
        if (SSE) {
            if (ROT) wht32_inplace(xh);
            acc += unit_sse(w, xh);
        }
        uint8_t* cp = a.codes + 16 * u;
        if (full) {
            stg_v4(cp, make_uint4(cw[0], cw[1], cw[2], cw[3]));
            if (FMT == kMX) a.scales[u] = (uint8_t)sb0;
            else reinterpret_cast<unsigned short*>(a.scales)[u] = (unsigned short)(sb0 | (sb1 << 8));
        } else {
            stg_v2(cp, cw[0], cw[1]);
            a.scales[2 * u] = (uint8_t)sb0;
        }
    }
    if (SSE) {
        acc = block_sum(acc, shd);
        if (threadIdx.x == 0) a.sse_partials[blockIdx.x] = acc;
    }
}

struct DeqArgs {
    const uint8_t* codes;
    const uint8_t* scales;
    const float* tensor_scale;
    Geometry g;
    uint16_t* y;
};

template <int FMT, bool ROT, bool CONTIG>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(DeqArgs a)
{
    constexpr bool PAIRED = (FMT == kMX) || ROT;
    const float s_t = (FMT != kMX) ? *a.tensor_scale : 0.0f;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < a.g.units; u += stride) {
        const bool full = 2 * u + 1 < a.g.halves;
        uint32_t cw[4], sb[2];
        load_packed<FMT>(a.codes, a.scales, u, full, cw, sb);
        float xh[32];
        decode_unit<FMT>(cw, sb, s_t, xh);
        if (ROT) wht32_inplace(xh);
        uint32_t o[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = pack_bf16x2_rn(xh[2 * k], xh[2 * k + 1]);
        uint16_t* p0 = a.y + half_offset<CONTIG>(a.g, 2 * u);
        stg_v4(p0, make_uint4(o[0], o[1], o[2], o[3]));
        stg_v4(p0 + 8, make_uint4(o[4], o[5], o[6], o[7]));
        if (full) {
            uint16_t* p1 = (CONTIG || PAIRED) ? p0 + 16 : a.y + half_offset<CONTIG>(a.g, 2 * u + 1);
            stg_v4(p1, make_uint4(o[8], o[9], o[10], o[11]));
            stg_v4(p1 + 8, make_uint4(o[12], o[13], o[14], o[15]));
        }
    }
}

struct ErrArgs {
    const uint16_t* x;
    const uint8_t* codes;
    const uint8_t* scales;
    const float* tensor_scale;
    Geometry g;
    double* sse_partials;
};

template <int FMT, bool ROT, bool CONTIG>
__global__ void __launch_bounds__(kThreads) error_kernel(ErrArgs a)
{
    constexpr bool PAIRED = (FMT == kMX) || ROT;
    __shared__ double shd[32];
    const float s_t = (FMT != kMX) ? *a.tensor_scale : 0.0f;
    double acc = 0.0;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < a.g.units; u += stride) {
        const bool full = 2 * u + 1 < a.g.halves;
        uint32_t w[16];
        load_unit<CONTIG, PAIRED>(a.x, a.g, u, full, w);
        uint32_t cw[4], sb[2];
        load_packed<FMT>(a.codes, a.scales, u, full, cw, sb);
        float xh[32];
        decode_unit<FMT>(cw, sb, s_t, xh);
        if (ROT) wht32_inplace(xh);
        if (!full) {
#pragma unroll
            for (int i = 16; i < 32; ++i) xh[i] = 0.0f;
        }
        acc += unit_sse(w, xh);
    }
    acc = block_sum(acc, shd);
    if (threadIdx.x == 0) a.sse_partials[blockIdx.x] = acc;
}

// Sum n fp64 partials in a fixed order and write sum / count.
__global__ void __launch_bounds__(kThreads) sse_finalize_kernel(const double* partials, int n, double count,
                                                                double* mse)
{
    __shared__ double sh[kThreads];
    double s = 0.0;
    for (int i = threadIdx.x; i < n; i += kThreads) s += partials[i];
    sh[threadIdx.x] = s;
    __syncthreads();
    for (int o = kThreads / 2; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *mse = count > 0.0 ? sh[0] / count : 0.0;
}

// ---------------------------------------------------------------------------
// Launch helpers
// ---------------------------------------------------------------------------

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_sm_count[kMaxDevices];

int sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

// Resident CTAs per SM for a kernel, cached per (kernel, device).
std::map<std::pair<const void*, int>, int> g_occupancy;

template <typename K>
int ctas_per_sm(K kernel)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_occupancy.find(key);
    if (it != g_occupancy.end()) return it->second;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, 0) != cudaSuccess || n <= 0) n = 1;
    g_occupancy[key] = n;
    return n;
}

template <typename K>
int grid_for(K kernel, int64_t units)
{
    const int64_t need = (units + kThreads - 1) / kThreads;
    int64_t cap = (int64_t)sm_count() * ctas_per_sm(kernel);
    if (cap > kMaxPartials) cap = kMaxPartials;
    int64_t g = need < cap ? need : cap;
    return g < 1 ? 1 : (int)g;
}

}  // namespace

cudaError_t launch_amax(const uint16_t* x, const Geometry& g, int rotate, float* partials, int* grid_out,
                        cudaStream_t st)
{
    AmaxArgs a{x, g, partials};
    const bool contig = g.ld == g.cols;
    const bool paired = (g.cols % 32) == 0;
    auto go = [&](auto kernel) {
        const int grid = grid_for(kernel, g.units);
        if (grid_out) *grid_out = grid;
        kernel<<<grid, kThreads, 0, st>>>(a);
        return cudaGetLastError();
    };
    if (rotate) return contig ? go(amax_kernel<true, true, true>) : go(amax_kernel<true, false, true>);
    if (contig) return go(amax_kernel<false, true, false>);
    return paired ? go(amax_kernel<false, false, true>) : go(amax_kernel<false, false, false>);
}

template <int FMT, bool ROT>
static cudaError_t quantize_dispatch(const QuantArgs& a, bool sse, bool contig, int* grid_out, cudaStream_t st)
{
    auto go = [&](auto kernel) {
        const int grid = grid_for(kernel, a.g.units);
        if (grid_out) *grid_out = grid;
        kernel<<<grid, kThreads, 0, st>>>(a);
        return cudaGetLastError();
    };
    if (sse) return contig ? go(quantize_kernel<FMT, ROT, true, true>) : go(quantize_kernel<FMT, ROT, true, false>);
    return contig ? go(quantize_kernel<FMT, ROT, false, true>) : go(quantize_kernel<FMT, ROT, false, false>);
}

cudaError_t launch_quantize(const uint16_t* x, const Geometry& g, int fmt, int rotate, int want_sse,
                            int scale_given, uint8_t* codes, uint8_t* scales, float* tensor_scale,
                            const float* amax_partials, int n_amax, double* sse_partials, int* grid_out,
                            cudaStream_t st)
{
    QuantArgs a{x, g, codes, scales, tensor_scale, amax_partials, n_amax, scale_given, sse_partials};
    const bool contig = g.ld == g.cols;
    const bool sse = want_sse != 0;
    switch (fmt * 2 + (rotate ? 1 : 0)) {
        case 0: return quantize_dispatch<kNV, false>(a, sse, contig, grid_out, st);
        case 1: return quantize_dispatch<kNV, true>(a, sse, contig, grid_out, st);
        case 2: return quantize_dispatch<kRZ, false>(a, sse, contig, grid_out, st);
        case 3: return quantize_dispatch<kRZ, true>(a, sse, contig, grid_out, st);
        case 4: return quantize_dispatch<kMX, false>(a, sse, contig, grid_out, st);
        case 5: return quantize_dispatch<kMX, true>(a, sse, contig, grid_out, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int FMT, bool ROT>
static cudaError_t dequantize_dispatch(const DeqArgs& a, bool contig, cudaStream_t st)
{
    auto go = [&](auto kernel) {
        kernel<<<grid_for(kernel, a.g.units), kThreads, 0, st>>>(a);
        return cudaGetLastError();
    };
    return contig ? go(dequantize_kernel<FMT, ROT, true>) : go(dequantize_kernel<FMT, ROT, false>);
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                              const Geometry& g, int fmt, int rotate, uint16_t* y, cudaStream_t st)
{
    DeqArgs a{codes, scales, tensor_scale, g, y};
    const bool contig = g.ld == g.cols;
    switch (fmt * 2 + (rotate ? 1 : 0)) {
        case 0: return dequantize_dispatch<kNV, false>(a, contig, st);
        case 1: return dequantize_dispatch<kNV, true>(a, contig, st);
        case 2: return dequantize_dispatch<kRZ, false>(a, contig, st);
        case 3: return dequantize_dispatch<kRZ, true>(a, contig, st);
        case 4: return dequantize_dispatch<kMX, false>(a, contig, st);
        case 5: return dequantize_dispatch<kMX, true>(a, contig, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int FMT, bool ROT>
static cudaError_t error_dispatch(const ErrArgs& a, bool contig, int* grid_out, cudaStream_t st)
{
    auto go = [&](auto kernel) {
        const int grid = grid_for(kernel, a.g.units);
        if (grid_out) *grid_out = grid;
        kernel<<<grid, kThreads, 0, st>>>(a);
        return cudaGetLastError();
    };
    return contig ? go(error_kernel<FMT, ROT, true>) : go(error_kernel<FMT, ROT, false>);
}

cudaError_t launch_error(const uint16_t* x, const uint8_t* codes, const uint8_t* scales,
                         const float* tensor_scale, const Geometry& g, int fmt, int rotate,
                         double* sse_partials, int* grid_out, cudaStream_t st)
{
    ErrArgs a{x, codes, scales, tensor_scale, g, sse_partials};
    const bool contig = g.ld == g.cols;
    switch (fmt * 2 + (rotate ? 1 : 0)) {
        case 0: return error_dispatch<kNV, false>(a, contig, grid_out, st);
        case 1: return error_dispatch<kNV, true>(a, contig, grid_out, st);
        case 2: return error_dispatch<kRZ, false>(a, contig, grid_out, st);
        case 3: return error_dispatch<kRZ, true>(a, contig, grid_out, st);
        case 4: return error_dispatch<kMX, false>(a, contig, grid_out, st);
        case 5: return error_dispatch<kMX, true>(a, contig, grid_out, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_sse_finalize(const double* partials, int n, double count, double* mse, cudaStream_t st)
{
    sse_finalize_kernel<<<1, kThreads, 0, st>>>(partials, n, count, mse);
    return cudaGetLastError();
}

}  // namespace fp4q
