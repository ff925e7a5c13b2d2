// Device code shared by the single-tensor kernels (fp4q_kernels.cu) and the
// batch scheduler (fp4q_batch.cu): tile and unit geometry, block encoders and
// decoders, error sums, CTA reductions and the TMA tile pipeline.
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
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "fp4q_device.cuh"
#include "fp4q_internal.h"
#include "fp4q_tma.cuh"

namespace fp4q {

// Formats, numbered as the C ABI's: NVFP4, RaZeR (activation mode: +-5),
// MXFP4, RaZeR weight mode (E3M3 scale, +-5 and +-2.5).
enum { kNV = 0, kRZ = 1, kMX = 2, kRW = 3 };

template <int FMT> constexpr bool kRazer = FMT == kRZ || FMT == kRW;

// The second special-value pair of the weight mode.
constexpr float kRazerWPair = 2.5f;

// s_t = RN(A / (6 * largest block-scale value)): 6 * 448 for the E4M3 scale,
// 6 * 30 for the weight mode's E3M3 scale.
template <int FMT>
__device__ __forceinline__ float tensor_scale_of(float amax)
{
    return __fdiv_rn(amax, FMT == kRW ? 180.0f : 2688.0f);
}


// ---------------------------------------------------------------------------
// Tiles and units
// ---------------------------------------------------------------------------

struct Tiles {
    int64_t count;       // number of tiles
    int64_t col_tiles;   // 2-D view: tiles across the columns (ceil(cols / 64))
    int64_t rows, cols;  // matrix shape
    int64_t units;       // flat view: N / 32
};

template <bool FLAT, int ROWS = kTileRows>
__device__ __forceinline__ void tile_origin(const Tiles& tl, int64_t k, int& x, int& y)
{
    if (FLAT) {
        x = 0;
        y = (int)(k * ROWS);
    } else {
        const int64_t rt = k / tl.col_tiles;
        x = (int)((k - rt * tl.col_tiles) * kTileCols);
        y = (int)(rt * ROWS);
    }
}

// The unit thread t owns in tile k: its row and column, whether it exists,
// whether both 16-element halves exist, and its unit index in the flat view.
struct Unit {
    int64_t row, col, flat;
    bool valid, full;
};

template <bool FLAT, int ROWS = kTileRows>
__device__ __forceinline__ Unit unit_of(const Tiles& tl, int64_t k, int t)
{
    Unit u;
    if (FLAT) {
        u.flat = k * (2 * ROWS) + t;
        u.valid = u.flat < tl.units;
        u.full = true;
        u.row = u.col = 0;
    } else {
        const int64_t rt = k / tl.col_tiles;
        const int64_t ct = k - rt * tl.col_tiles;
        u.row = rt * ROWS + (t >> 1);
        u.col = ct * kTileCols + 32 * (t & 1);
        u.valid = u.row < tl.rows && u.col < tl.cols;
        u.full = u.col + 32 <= tl.cols;
        u.flat = 0;
    }
    return u;
}

// Offsets of a unit's codes and scale bytes in the dense layouts.
template <bool FLAT, int FMT>
__device__ __forceinline__ void unit_offsets(const Tiles& tl, const Unit& u, int64_t& code_off, int64_t& scale_off)
{
    constexpr int B = FMT == kMX ? 32 : 16;
    if (FLAT) {
        code_off = 16 * u.flat;
        scale_off = (32 / B) * u.flat;
    } else {
        code_off = u.row * (tl.cols / 2) + u.col / 2;
        scale_off = u.row * (tl.cols / B) + u.col / B;
    }
}

// Store 16 (full) or 8 bytes of codes; a16 tells whether the address is 16-byte aligned.
__device__ __forceinline__ void store_codes(uint8_t* p, const uint32_t* cw, bool full, bool a16)
{
    if (full && a16) {
        stg_v4(p, make_uint4(cw[0], cw[1], cw[2], cw[3]));
    } else {
        stg_v2(p, cw[0], cw[1]);
        if (full) stg_v2(p + 8, cw[2], cw[3]);
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
// Squared error
// ---------------------------------------------------------------------------

// Sum of squares of 16 differences, exact in fp64 range: the values are
// scaled by 2^-k, 2^k the power of two at or below their largest magnitude
// (in two exact steps, so 2^-k never overflows), squared and summed in fp32,
// and the sum is scaled back by 2^2k in fp64.  Used when a fast fp32 sum
// overflowed or may have lost terms to underflow (|x| near the top of the bf16
// range, or bf16 subnormals).
__device__ __forceinline__ double sse16_rescaled(const float* d)
{
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(d[i]));
    if (m == 0.0f || !(m <= 3.4e38f)) return m == 0.0f ? 0.0 : (double)INFINITY;
    const int k = floor_log2_f32(m);              // in [-149, 127]
    const int k1 = -k / 2, k2 = -k - k1;           // each in [-64, 75]
    const float s1 = __uint_as_float((uint32_t)(k1 + 127) << 23);
    const float s2 = __uint_as_float((uint32_t)(k2 + 127) << 23);
    float es = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float t = __fmul_rn(__fmul_rn(d[i], s1), s2);
        es = __fmaf_rn(t, t, es);
    }
    return (double)es * __longlong_as_double((long long)(2 * k + 1023) << 52);
}

// Sum of squared errors of 16 values (x - xh), the differences in fp32.
__device__ __forceinline__ double sse16(const float* x, const float* xh)
{
    float2 acc = make_float2(0.0f, 0.0f);
    float d[16];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const float2 e = sub2_rn(make_float2(x[i], x[i + 1]), make_float2(xh[i], xh[i + 1]));
        d[i] = e.x;
        d[i + 1] = e.y;
        acc = fma2_rn(e, e, acc);
    }
    const float es = acc.x + acc.y;
    if (es >= 0x1p-100f && es <= 3.0e38f) return (double)es;
    return sse16_rescaled(d);
}

template <int N>
__device__ __forceinline__ double sse_of(const float* x, const float* xh)
{
    double e = sse16(x, xh);
    if (N == 32) e += sse16(x + 16, xh + 16);
    return e;
}

// ---------------------------------------------------------------------------
// Encoders
// ---------------------------------------------------------------------------

__device__ __forceinline__ void unpack16(const uint32_t* w, float* y)
{
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float2 p = bf16x2_to_f32(w[k]);
        y[2 * k] = p.x;
        y[2 * k + 1] = p.y;
    }
}

// Decode 16 codes (two words) to their E2M1 values.
__device__ __forceinline__ void decode16(uint32_t w0, uint32_t w1, float* q)
{
    e2m1x8_to_f32(w0, q);
    e2m1x8_to_f32(w1, q + 8);
}

// Per-tensor constants of the NVFP4 block-scale step, shared by a CTA: for
// each of the 127 non-negative finite E4M3 bytes b (the 64 E3M3 codes in the
// weight mode), den[b] = RN(dec(b) * s_t),
// rcp[b] = RN(1 / den[b]) (0 when den[b] = 0: a zero scale zeroes every code)
// and den[b]^2 (exact in binary64).  The quotient t = RN(a / RN(6 s_t)) uses
// inv6 = RN(1 / RN(6 s_t)) and one correction step (Markstein's theorem: with
// y = RN(1/b) and a faithful q = RN(a y), the residual r = a - q b is exact and
// RN(q + r y) = RN(a / b)); `exact_div` selects IEEE division when RN(6 s_t)
// is outside [2^-64, 2^64], where the theorem's no-underflow conditions are
// not guaranteed.
struct NvTable {
    float2 dr[128];       // {den, rcp}
    double den2[128];     // den^2
};

struct NvScale {
    float s_t, six_st, inv6;
    bool exact_div;
    uint32_t tab;         // shared address of the CTA's NvTable
};

template <int FMT>
__device__ __forceinline__ NvScale nv_scale_setup(float s_t, NvTable* tab)
{
    NvScale c;
    c.s_t = s_t;
    c.six_st = __fmul_rn(6.0f, s_t);
    c.exact_div = !(c.six_st >= 0x1p-64f && c.six_st <= 0x1p64f);
    c.inv6 = c.exact_div ? 0.0f : __frcp_rn(c.six_st);
    for (int b = threadIdx.x; b < 128; b += blockDim.x) {
        float d = 0.0f;
        if (FMT == kRW) d = b < 64 ? __fmul_rn(e3m3_to_f32((uint32_t)b), s_t) : 0.0f;
        else d = b < 127 ? __fmul_rn(e4m3_to_f32((uint32_t)b), s_t) : 0.0f;
        tab->dr[b] = make_float2(d, d != 0.0f ? __frcp_rn(d) : 0.0f);
        tab->den2[b] = (double)d * (double)d;
    }
    __syncthreads();
    c.tab = smem_u32(tab);
    return c;
}

// {den, rcp} of the unsigned scale code sb.
__device__ __forceinline__ float2 nv_den_rcp(const NvScale& c, uint32_t sb)
{
    float2 v;
    asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(c.tab + 8u * sb));
    return v;
}

// den^2 of the unsigned scale code sb.
__device__ __forceinline__ double nv_den2(const NvScale& c, uint32_t sb)
{
    double v;
    asm("ld.shared.f64 %0, [%1];" : "=d"(v) : "r"(c.tab + (uint32_t)offsetof(NvTable, den2) + 8u * sb));
    return v;
}

// t = RN(a / RN(6 s_t)) for a >= 0.
__device__ __forceinline__ float nv_block_ratio(const NvScale& c, float a)
{
    if (c.exact_div) return c.six_st > 0.0f ? __fdiv_rn(a, c.six_st) : 0.0f;
    const float q = __fmul_rn(a, c.inv6);
    const float r = __fmaf_rn(-q, c.six_st, a);
    return __fmaf_rn(r, c.inv6, q);
}

// Unsigned block-scale code of a block with absmax a: E4M3, or E3M3 in the
// weight mode, of t = RN(a / RN(6 s_t)), nearest even, saturating.
template <int FMT>
__device__ __forceinline__ uint32_t nv_scale_code(const NvScale& c, float a)
{
    const float t = nv_block_ratio(c, a);
    return FMT == kRW ? e3m3_rn_sat(t) : e4m3_rn_satfinite(t);
}

// Decoded block scale of scale byte sb (its selector bits ignored).
template <int FMT>
__device__ __forceinline__ float nv_scale_value(uint32_t sb)
{
    if (FMT == kRW) return e3m3_to_f32(sb & 0x3Fu);
    return e4m3_to_f32(FMT == kRZ ? (sb & 0x7Fu) : sb);
}

// The special value code 0b1000 stands for in a block with scale byte sb:
// activation mode +5, or -5 with bit 7 set; weight mode, by bits 6..7,
// +5, -5, +2.5, -2.5.
template <int FMT>
__device__ __forceinline__ float razer_special(uint32_t sb)
{
    if (FMT == kRW) {
        const float m = (sb & 0x80u) ? kRazerWPair : 5.0f;
        return (sb & 0x40u) ? -m : m;
    }
    return (sb & 0x80u) ? -5.0f : 5.0f;
}

// RaZeR remap of one block given cs[i] = sign(v_i) * gain_i, the signed gains
// of remapping element i to sign(v_i) * 5 (multiples of 2^-20 in [-1, 1]),
// and their exact sum S = gain(+5) - gain(-5): -5 only when its gain is
// strictly larger.  Winners are the candidates of the chosen sign.  With
// x = cs * (+-2^40), every candidate has |x| >= 2^20 and encodes (saturating)
// as +6 = 0b0111 when it wins and as -6 = 0b1111 otherwise, and every other
// element as +-0; so bit 0 and not bit 3 of a nibble flags a winner, whose
// code becomes 0b1000.
__device__ __forceinline__ void razer_apply(const float* cs, float S, uint32_t& w0, uint32_t& w1, uint32_t& sb)
{
    const float sk = S < 0.0f ? -0x1p40f : 0x1p40f;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const float2 p = mul2_rn(make_float2(cs[i], cs[i + 1]), make_float2(sk, sk));
        x[i] = p.x;
        x[i + 1] = p.y;
    }
    const uint32_t k0 = e2m1x8(x), k1 = e2m1x8(x + 8);
    const uint32_t f0 = k0 & ~(k0 >> 3) & 0x11111111u;
    const uint32_t f1 = k1 & ~(k1 >> 3) & 0x11111111u;
    w0 = (w0 & ~(f0 * 15u)) | (f0 << 3);
    w1 = (w1 & ~(f1 * 15u)) | (f1 << 3);
    if (S < 0.0f) sb |= 0x80u;
}

// RaZeR selection from the scaled values alone (any magnitude).  For |v| in
// (4.5, 5.5) the regular value is 4 (|v| <= 5) or 6 and
//   (|v| - q)^2 - (|v| - 5)^2 = 1 - 2 | |v| - 5 |,
// positive exactly on that open interval; elsewhere the gain is clamped to 0.
// |v| - 5 is exact there, so each gain is a multiple of 2^-20 and every sum of
// them is exact in any order.
__device__ __forceinline__ void razer_tent(const float* v, uint32_t& w0, uint32_t& w1, uint32_t& sb)
{
    float cs[16];
    float2 sp[8];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        cs[i] = copysignf(__saturatef(__fmaf_rn(-2.0f, fabsf(fabsf(v[i]) - 5.0f), 1.0f)), v[i]);
#pragma unroll
    for (int i = 0; i < 8; ++i) sp[i] = make_float2(cs[2 * i], cs[2 * i + 1]);
#pragma unroll
    for (int k = 4; k > 0; k >>= 1)
#pragma unroll
        for (int i = 0; i < k; ++i) sp[i] = add2_rn(sp[i], sp[i + k]);
    razer_apply(cs, sp[0].x + sp[0].y, w0, w1, sb);
}

// Gain of remapping |v| to 2.5: its regular value is 2 (|v| <= 2.5) or 3,
// and (|v| - q)^2 - (|v| - 2.5)^2 = 1/4 - | |v| - 2.5 |, positive exactly on
// (2.25, 2.75) and clamped to 0 elsewhere; |v| - 2.5 is exact there, so the
// gain is a multiple of 2^-22.
__device__ __forceinline__ float razer_gain_w2(float v)
{
    return __saturatef(0.25f - fabsf(fabsf(v) - kRazerWPair));
}

// Rewrite the winners flagged in k (nibbles 0xF) to 0b1000.
__device__ __forceinline__ uint32_t apply_winners(uint32_t w, uint32_t k)
{
    const uint32_t f = k & (k >> 3) & 0x11111111u;
    return (w & ~(f * 15u)) | (f << 3);
}


// Weight-mode selection in running form.  w0, w1 hold the block's regular
// codes.  For each run of eight elements: the gains of 5 (from e = q - v when
// GE, else from v) and of 2.5, their sums and signed sums, and one candidate
// marker per element for both pairs (no element is a candidate of both): the
// E2M1 code of sign(v) * gain * 2^40, +6 (0x7) for a candidate of a positive
// member, -6 (0xF) of a negative one, +-0 otherwise.  Gains of 5 are multiples
// of 2^-20 up to 1 and gains of 2.5 multiples of 2^-22 up to 1/4, so every sum
// is exact in any order and the comparisons are exact.  For either pair the
// better member's gain is (U + |S|) / 2; the pair 2.5 is taken only when its
// gain is strictly larger, and in a pair the negative member only when its
// gain is strictly larger (ties go to the lower selector; a block with no gain
// keeps selector 0).  The winners are the chosen value's candidates: markers
// of the chosen sign (bit 3 flipped when the positive member wins) whose
// element belongs to the chosen pair.  Returns the chosen gain.
template <bool GE>
__device__ __forceinline__ float razer_w_select(const float* v, const float* e, uint32_t& w0, uint32_t& w1,
                                                uint32_t& sb)
{
    float2 u5 = make_float2(0.0f, 0.0f), s5 = u5, u2 = u5, s2 = u5;
    uint32_t k[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const int j = 8 * hh + i;
            float g0, g1;
            if (GE) {
                g0 = __saturatef(__fmaf_rn(2.0f, fabsf(e[j]), -1.0f));
                g1 = __saturatef(__fmaf_rn(2.0f, fabsf(e[j + 1]), -1.0f));
            } else {
                g0 = __saturatef(__fmaf_rn(-2.0f, fabsf(fabsf(v[j]) - 5.0f), 1.0f));
                g1 = __saturatef(__fmaf_rn(-2.0f, fabsf(fabsf(v[j + 1]) - 5.0f), 1.0f));
            }
            const float h0 = razer_gain_w2(v[j]), h1 = razer_gain_w2(v[j + 1]);
            const float2 c5 = make_float2(copysignf(g0, v[j]), copysignf(g1, v[j + 1]));
            const float2 c2 = make_float2(copysignf(h0, v[j]), copysignf(h1, v[j + 1]));
            u5 = add2_rn(u5, make_float2(g0, g1));
            s5 = add2_rn(s5, c5);
            u2 = add2_rn(u2, make_float2(h0, h1));
            s2 = add2_rn(s2, c2);
            // one marker for both pairs: no element is a candidate of both, so
            // at most one of c5, c2 is nonzero and their sum is exact
            const float2 m = mul2_rn(add2_rn(c5, c2), make_float2(0x1p40f, 0x1p40f));
            x[i] = m.x;
            x[i + 1] = m.y;
        }
        k[hh] = e2m1x8(x);
    }
    const float S5 = s5.x + s5.y, S2 = s2.x + s2.y;
    const float t5 = (u5.x + u5.y) + fabsf(S5), t2 = (u2.x + u2.y) + fabsf(S2);
    const bool p2 = t2 > t5;
    const bool neg = (p2 ? S2 : S5) < 0.0f;
    const uint32_t flip = neg ? 0u : 0x88888888u;
    // The pair a candidate belongs to is bit 1 of its regular code's
    // magnitude: 4 and 6 (codes 6, 7) for 5, 2 and 3 (codes 4, 5) for 2.5.
    const uint32_t pm = p2 ? 0x11111111u : 0u;
    // Bit 0 of a marker survives only where its element belongs to the chosen pair.
    w0 = apply_winners(w0, (k[0] ^ flip) & ((((w0 >> 1) ^ pm) & 0x11111111u) | 0xEEEEEEEEu));
    w1 = apply_winners(w1, (k[1] ^ flip) & ((((w1 >> 1) ^ pm) & 0x11111111u) | 0xEEEEEEEEu));
    sb |= (p2 ? 0x80u : 0u) | (neg ? 0x40u : 0u);
    return 0.5f * fmaxf(t5, t2);
}

// Selection from the scaled values for either RaZeR mode.
template <int FMT>
__device__ __forceinline__ void razer_from_v(const float* v, uint32_t& w0, uint32_t& w1, uint32_t& sb)
{
    if (FMT == kRW) razer_w_select<false>(v, nullptr, w0, w1, sb);
    else razer_tent(v, w0, w1, sb);
}

// ---------------------------------------------------------------------------
// Unrotated NVFP4 / RaZeR blocks straight from the bf16 tile
// ---------------------------------------------------------------------------

struct BlockOut {
    uint32_t w0, w1, sb;
    double sse;
};

// One block recomputed in full from its bf16 words in shared memory (chunks
// at a0 and a1), given its unsigned scale byte and {den, rcp}: codes, scale
// byte and the squared error in the original domain, each difference
// y - RN(q den) taken in fp32 (zero when the element is reproduced) and
// squared and summed in fp64.  Elements are scaled by r = RN(1 / den), or
// divided by den where r overflowed to infinity.  Taken for the rare blocks the
// fast path below does not cover.
template <int FMT>
__device__ __noinline__ BlockOut nv_block_exact(uint32_t a0, uint32_t a1, uint32_t sb, float den, float r)
{
    constexpr bool RAZER = kRazer<FMT>;
    uint32_t w[8];
    const uint4 c0 = lds128(a0), c1 = lds128(a1);
    w[0] = c0.x; w[1] = c0.y; w[2] = c0.z; w[3] = c0.w;
    w[4] = c1.x; w[5] = c1.y; w[6] = c1.z; w[7] = c1.w;
    float y[16], v[16];
    unpack16(w, y);
    if (isinf(r)) {   // RN(1 / den) overflowed (den below about 2^-128): scale by division
#pragma unroll 1
        for (int i = 0; i < 16; ++i) v[i] = __fdiv_rn(y[i], den);
    } else {
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float2 p = mul2_rn(make_float2(y[i], y[i + 1]), make_float2(r, r));
            v[i] = p.x;
            v[i + 1] = p.y;
        }
    }
    BlockOut o;
    o.w0 = canonical_zero(e2m1x8(v));
    o.w1 = canonical_zero(e2m1x8(v + 8));
    o.sb = sb;
    if (RAZER) razer_from_v<FMT>(v, o.w0, o.w1, o.sb);
    float q[16];
    decode16(o.w0, o.w1, q);
    const float special = razer_special<FMT>(o.sb);
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t nib = ((i < 8 ? o.w0 : o.w1) >> (4 * (i & 7))) & 0xFu;
        const float qi = (RAZER && nib == 8u) ? special : q[i];
        const double d = (double)(y[i] - __fmul_rn(qi, den));
        s = fma(d, d, s);
    }
    o.sse = s;
    return o;
}

// One unrotated 16-element NVFP4 / RaZeR block from its eight bf16x2 words w
// (chunks a0, a1 of the tile): two code words, the scale byte and, when SSE,
// the block's squared error.
//
// The squared error is formed in the scaled domain.  With v = RN(y r) the
// scaled values and q the regular grid values, e = q - v is exact (see
// e2m1x8_diff) and the block's error is den^2 (sum e^2 - G), where G is the
// total gain of the RaZeR winners (0 for NVFP4).  For a candidate (|v| in
// (4.5, 5.5), q = +-4 or +-6) the gain 1 - 2||v| - 5| equals 2|e| - 1, and
// sat(2|e| - 1) is 0 for every other element as long as |v| <= 6.5, so gains,
// decision and G come from e with no further per-element work (the weight
// mode's gains of 2.5 come from v, see razer_gain_w2).  den v differs
// from y by at most 2^-23 |y| (two roundings), the only departure from the
// exact error besides fp32 rounding of the sum.
//
// Blocks outside the fast path's assumptions are recomputed by
// nv_block_exact: max |v| > 6.5 (a saturated scale byte, or a subnormal one
// far below the block absmax), a fast sum below 2^-30 (the block is reproduced
// exactly or almost, and the exact sum keeps a zero error zero), or one that
// is not finite (an infinite reciprocal: den below about 2^-128, where the
// exact path divides).  A subnormal den with a finite reciprocal (den in
// [2^-128, 2^-126), only in tensors whose absmax is below about 2^-105) stays
// on the fast path: RN(q den) may round there by half a subnormal quantum,
// which moves the block's error by about 2^-20 of itself.
template <int FMT, bool SSE>
__device__ __forceinline__ void nv_block(const uint32_t* w, uint32_t a0, uint32_t a1, const NvScale& sc,
                                         uint32_t& c0, uint32_t& c1, uint32_t& sb_out, double& sse)
{
    constexpr bool RAZER = kRazer<FMT>;
    const uint32_t mm = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(w[0], w[1]), bf16x2_absmax(w[2], w[3])),
                                      bf16x2_absmax(bf16x2_absmax(w[4], w[5]), bf16x2_absmax(w[6], w[7])));
    const float a = bf16x2_hmax_abs(mm);
    uint32_t sb = nv_scale_code<FMT>(sc, a);
    const float2 dr = nv_den_rcp(sc, sb);
    float v[16];
    {
        float y[16];
        unpack16(w, y);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float2 p = mul2_rn(make_float2(y[i], y[i + 1]), make_float2(dr.y, dr.y));
            v[i] = p.x;
            v[i + 1] = p.y;
        }
    }
    if (!SSE) {
        if (isinf(dr.y)) {   // RN(1 / den) overflowed: the exact path divides
            const BlockOut o = nv_block_exact<FMT>(a0, a1, sb, dr.x, dr.y);
            c0 = o.w0;
            c1 = o.w1;
            sb_out = o.sb;
            return;
        }
        uint32_t w0 = canonical_zero(e2m1x8(v)), w1 = canonical_zero(e2m1x8(v + 8));
        if (RAZER) razer_from_v<FMT>(v, w0, w1, sb);
        c0 = w0;
        c1 = w1;
        sb_out = sb;
        return;
    }
    float e[16];
    uint32_t w0 = e2m1x8_diff(v, e), w1 = e2m1x8_diff(v + 8, e + 8);
    float2 sq[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        sq[i] = mul2_rn(make_float2(e[2 * i], e[2 * i + 1]), make_float2(e[2 * i], e[2 * i + 1]));
        sq[i] = fma2_rn(make_float2(e[2 * i + 8], e[2 * i + 9]), make_float2(e[2 * i + 8], e[2 * i + 9]), sq[i]);
    }
    sq[0] = add2_rn(add2_rn(sq[0], sq[1]), add2_rn(sq[2], sq[3]));
    float sv = sq[0].x + sq[0].y;
    w0 = canonical_zero(w0);
    w1 = canonical_zero(w1);
    const uint32_t sb0 = sb;
    if (FMT == kRW) {
        sv -= razer_w_select<true>(v, e, w0, w1, sb);
    } else if (RAZER) {
        float cs[16];
        float2 gp[8], sp[8];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float g0 = __saturatef(__fmaf_rn(2.0f, fabsf(e[i]), -1.0f));
            const float g1 = __saturatef(__fmaf_rn(2.0f, fabsf(e[i + 1]), -1.0f));
            cs[i] = copysignf(g0, v[i]);
            cs[i + 1] = copysignf(g1, v[i + 1]);
            gp[i / 2] = make_float2(g0, g1);
            sp[i / 2] = make_float2(cs[i], cs[i + 1]);
        }
        // pairwise sums (exact in any order)
#pragma unroll
        for (int k = 4; k > 0; k >>= 1)
#pragma unroll
            for (int i = 0; i < k; ++i) {
                gp[i] = add2_rn(gp[i], gp[i + k]);
                sp[i] = add2_rn(sp[i], sp[i + k]);
            }
        const float S = sp[0].x + sp[0].y;
        sv -= 0.5f * ((gp[0].x + gp[0].y) + fabsf(S));   // G = max(gain(+5), gain(-5))
        razer_apply(cs, S, w0, w1, sb);
    }
    const bool fast = sv >= 0x1p-30f && sv <= 0x1p64f && (!RAZER || __fmul_rn(a, dr.y) <= 6.5f);
    if (fast) {
        c0 = w0;
        c1 = w1;
        sb_out = sb;
        sse = (double)sv * nv_den2(sc, sb0);
    } else {
        const BlockOut o = nv_block_exact<FMT>(a0, a1, sb0, dr.x, dr.y);
        c0 = o.w0;
        c1 = o.w1;
        sb_out = o.sb;
        sse = o.sse;
    }
}

// ---------------------------------------------------------------------------
// NVFP4 / RaZeR blocks, eight elements at a time
// ---------------------------------------------------------------------------
//
// A block's elements are encoded in two runs of eight, each adding to running
// sums, so that no per-element array outlives its run:
//  - the codes (cvt.rn.satfinite.e2m1x2: nearest even, saturating);
//  - with SSE, e = q - v for the regular grid value q of each scaled value v
//    (exact, see e2m1x8_diff) and the sum of e^2;
//  - RaZeR: for each element its gain of moving to sign(v) * 5 -- for |v| in
//    (4.5, 5.5) the regular value is 4 or 6 and (|v| - q)^2 - (|v| - 5)^2 =
//    1 - 2 ||v| - 5| = 2 |e| - 1, clamped at 0 elsewhere -- summed as U (all
//    gains) and S (gains signed by v).  Every gain is a multiple of 2^-20 in
//    [0, 1], so both sums are exact in fp32 whatever the order; gain(+5) =
//    (U + S) / 2 and gain(-5) = (U - S) / 2.  A candidate marker per element,
//    the E2M1 code of sign(v) * gain * 2^40, is +6 (0x7) for a candidate of
//    +5, -6 (0xF) for one of -5 and +-0 otherwise;
//  - the weight mode adds the pair 2.5 the same way (gain 1/4 - ||v| - 2.5|,
//    multiples of 2^-22 up to 1/4).  Candidates of 2.5 and of 5 never
//    overlap, so one marker word serves both pairs; bit 1 of an element's
//    regular code magnitude tells which pair it is a candidate of.
// The 2|e| - 1 form of the gain of 5 holds while |v| <= 6.5; blocks beyond
// that take the exact path (nv_block_exact_f32), which forms gains from v.

struct NvRun {
    uint32_t cw[2];          // code words, eight nibbles each
    uint32_t k[2];           // candidate markers of 5 and (weight mode) of 2.5
    float2 sq;               // sum of e^2, two lanes
    float2 u5, s5, u2, s2;   // sums of the gains and of the signed gains, two lanes
};

// One run of eight scaled values v into run h (0 or 1) of the block.  GE: the
// gains of 5 come from e (the fast path); otherwise from v.
template <int FMT, bool SSE, bool GE>
__device__ __forceinline__ void nv_run8(const float* v, int h, NvRun& st)
{
    constexpr bool RAZER = kRazer<FMT>;
    float g[8];
    if (SSE) {
        float e[8];
        st.cw[h] = e2m1x8_diff(v, e);
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            st.sq = fma2_rn(make_float2(e[i], e[i + 1]), make_float2(e[i], e[i + 1]), st.sq);
        if (RAZER && GE) {
#pragma unroll
            for (int i = 0; i < 8; ++i) g[i] = __saturatef(__fmaf_rn(2.0f, fabsf(e[i]), -1.0f));
        }
    } else {
        st.cw[h] = e2m1x8(v);
    }
    if (RAZER && !(SSE && GE)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = __saturatef(__fmaf_rn(-2.0f, fabsf(fabsf(v[i]) - 5.0f), 1.0f));
    }
    if (RAZER) {
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float2 gg = make_float2(g[i], g[i + 1]);
            float2 cs = make_float2(copysignf(g[i], v[i]), copysignf(g[i + 1], v[i + 1]));
            st.u5 = add2_rn(st.u5, gg);
            st.s5 = add2_rn(st.s5, cs);
            if (FMT == kRW) {
                const float g0 = razer_gain_w2(v[i]), g1 = razer_gain_w2(v[i + 1]);
                const float2 c2 = make_float2(copysignf(g0, v[i]), copysignf(g1, v[i + 1]));
                st.u2 = add2_rn(st.u2, make_float2(g0, g1));
                st.s2 = add2_rn(st.s2, c2);
                cs = add2_rn(cs, c2);   // one marker for both pairs: no element is a candidate of both
            }
            const float2 m = mul2_rn(cs, make_float2(0x1p40f, 0x1p40f));
            x[i] = m.x;
            x[i + 1] = m.y;
        }
        st.k[h] = e2m1x8(x);
    }
}

// The block's RaZeR choice from its running sums: -5 only when its gain is
// strictly larger than that of +5 (equal gains, or none, keep +5 with bit 7
// clear); in the weight mode the pair 2.5 only when its better member gains
// strictly more than the better of +-5, and in a pair the negative member
// only when it gains strictly more (ties go to the lower selector; bits 6..7:
// 0 +5, 1 -5, 2 +2.5, 3 -2.5).  Canonicalises -0 codes to +0, writes the
// winners' codes as 0b1000 and the selector into sb, and returns the chosen
// total gain (0 for NVFP4).
template <int FMT>
__device__ __forceinline__ float nv_finish(NvRun& st, uint32_t& sb)
{
    st.cw[0] = canonical_zero(st.cw[0]);
    st.cw[1] = canonical_zero(st.cw[1]);
    if (!kRazer<FMT>) return 0.0f;
    const float U5 = st.u5.x + st.u5.y, S5 = st.s5.x + st.s5.y;
    float G;
    bool neg;
    uint32_t k0 = st.k[0], k1 = st.k[1];
    if (FMT == kRW) {
        const float U2 = st.u2.x + st.u2.y, S2 = st.s2.x + st.s2.y;
        const float t5 = U5 + fabsf(S5), t2 = U2 + fabsf(S2);
        const bool p2 = t2 > t5;
        neg = (p2 ? S2 : S5) < 0.0f;
        // Keep the markers of the chosen pair: bit 1 of the regular code's
        // magnitude is set for 4 and 6 (candidates of 5), clear for 2 and 3.
        const uint32_t pm = p2 ? 0x11111111u : 0u;
        k0 &= (((st.cw[0] >> 1) ^ pm) & 0x11111111u) | 0xEEEEEEEEu;
        k1 &= (((st.cw[1] >> 1) ^ pm) & 0x11111111u) | 0xEEEEEEEEu;
        sb |= (p2 ? 0x80u : 0u) | (neg ? 0x40u : 0u);
        G = 0.5f * fmaxf(t5, t2);
    } else {
        neg = S5 < 0.0f;
        if (neg) sb |= 0x80u;
        G = 0.5f * (U5 + fabsf(S5));
    }
    // markers of the chosen sign become 0xF: those of +5 (0x7) by flipping bit 3
    const uint32_t flip = neg ? 0u : 0x88888888u;
    st.cw[0] = apply_winners(st.cw[0], k0 ^ flip);
    st.cw[1] = apply_winners(st.cw[1], k1 ^ flip);
    return G;
}

// Exact squared error of eight values y against the reconstruction RN(q den)
// of code word cw (RaZeR code 0b1000: the special value of scale byte sb),
// each difference and its square summed in fp64, as the oracle does.
template <int FMT>
__device__ __forceinline__ double nv_sse8_exact(const float* y, uint32_t cw, uint32_t sb, float den)
{
    float q[8];
    e2m1x8_to_f32(cw, q);
    const float special = razer_special<FMT>(sb);
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float qi = (kRazer<FMT> && ((cw >> (4 * i)) & 0xFu) == 8u) ? special : q[i];
        const double d = (double)y[i] - (double)__fmul_rn(qi, den);
        s = fma(d, d, s);
    }
    return s;
}

// Scaled values of eight y: RN(y r), or RN(y / den) where r overflowed (DIV).
template <bool DIV>
__device__ __forceinline__ void nv_scale8(const float* y, float den, float r, float* v)
{
    if (DIV && isinf(r)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fdiv_rn(y[i], den);
    } else {
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float2 p = mul2_rn(make_float2(y[i], y[i + 1]), make_float2(r, r));
            v[i] = p.x;
            v[i + 1] = p.y;
        }
    }
}

// One block of sixteen fp32 values y (rotated ones on the rotated path) with
// absmax a, encoded from scratch in the exact way: gains from v, the error in
// fp64 from the reconstruction, and division wherever RN(1 / den) overflowed
// (DIV).  For the rare blocks the fast path does not cover (nv_block_redo).
template <int FMT, bool SSE, bool DIV>
__device__ __forceinline__ void nv_block_exact_f32(const float* y, uint32_t sb, float den, float r, uint32_t& c0,
                                               uint32_t& c1, uint32_t& sb_out, double& sse)
{
    NvRun st = {};
    float v[8];
    nv_scale8<DIV>(y, den, r, v);
    nv_run8<FMT, false, false>(v, 0, st);
    nv_scale8<DIV>(y + 8, den, r, v);
    nv_run8<FMT, false, false>(v, 1, st);
    nv_finish<FMT>(st, sb);
    c0 = st.cw[0];
    c1 = st.cw[1];
    sb_out = sb;
    if (SSE) sse = nv_sse8_exact<FMT>(y, c0, sb, den) + nv_sse8_exact<FMT>(y + 8, c1, sb, den);
}

// The error of a block from its running sums, den^2 (sum e^2 - G), valid when
// it is not too small (a block reproduced exactly or almost keeps the exact
// sum, so that an exact reconstruction has error 0) and finite, and when
// max |v| <= 6.5 for RaZeR (the 2|e| - 1 form of the gains).  den v differs
// from y by at most 2^-23 |y| (two roundings), the only departure from the
// exact error besides the fp32 rounding of the sums.
template <int FMT>
__device__ __forceinline__ bool nv_fast_error(const NvRun& st, float G, float a, float r, float& sv)
{
    sv = (st.sq.x + st.sq.y) - G;
    return sv >= 0x1p-30f && sv <= 0x1p64f && (!kRazer<FMT> || __fmul_rn(a, r) <= 6.5f);
}

// One block of sixteen fp32 values y with absmax a (the rotated path): codes,
// scale byte and, when SSE, the error in y's domain from the running sums.
// Returns false (outputs unset) when the fast path does not hold -- an
// overflowed reciprocal, or a fast error that does not hold -- and the caller
// redoes the block (nv_block_redo).
template <int FMT, bool SSE>
__device__ __forceinline__ bool nv_block_f32(const float* y, float a, const NvScale& sc, uint32_t& c0,
                                             uint32_t& c1, uint32_t& sb_out, double& sse)
{
    uint32_t sb = nv_scale_code<FMT>(sc, a);
    const float2 dr = nv_den_rcp(sc, sb);
    if (isinf(dr.y)) return false;
    const uint32_t sb0 = sb;
    NvRun st = {};
    float v[8];
    nv_scale8<false>(y, dr.x, dr.y, v);
    nv_run8<FMT, SSE, true>(v, 0, st);
    nv_scale8<false>(y + 8, dr.x, dr.y, v);
    nv_run8<FMT, SSE, true>(v, 1, st);
    const float G = nv_finish<FMT>(st, sb);
    float sv = 0.0f;
    if (SSE && !nv_fast_error<FMT>(st, G, a, dr.y, sv)) return false;
    c0 = st.cw[0];
    c1 = st.cw[1];
    sb_out = sb;
    if (SSE) sse = (double)sv * nv_den2(sc, sb0);
    return true;
}

// One 32-element MXFP4 block of fp32 values y with absmax a.  The exponent is
// floor(log2 a) - 2 (values in [6, 8) 2^e saturate to 6) or, with ceil, the
// smallest e with a <= 6 * 2^e: one more when a's significand exceeds 1.5
// ("TORQ: Two-Level Orthogonal Rotation for MXFP4 Quantization", sect. 2,
// S-step: the block maximum onto the largest code), at most 125 so that
// 6 * 2^e stays finite in fp32.  v = y 2^-e is exact, so e = q - v is exact
// and the error (q - v)^2 2^2e is formed in the scaled domain; the fp32 sum
// of e^2 is the only rounding.
template <bool SSE>
__device__ __forceinline__ void mx_block(const float* y, float a, bool ceil, uint32_t* cw, uint32_t& sb_out,
                                         double& sse)
{
    int e = -127;
    float r = 0.0f;
    uint32_t sb = 0;
    if (a > 0.0f) {
        e = floor_log2_f32(a) - 2;          // 2 = exponent of the largest E2M1 value
        if (ceil) e = min(e + significand_above_1p5(a), 125);
        e = e < -127 ? -127 : (e > 127 ? 127 : e);
        sb = (uint32_t)(e + 127);
        r = exp2i(-e);
    }
    float2 sq = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float2 p = mul2_rn(make_float2(y[8 * k + i], y[8 * k + i + 1]), make_float2(r, r));
            v[i] = p.x;
            v[i + 1] = p.y;
        }
        if (SSE) {
            float d[8];
            cw[k] = canonical_zero(e2m1x8_diff(v, d));
#pragma unroll
            for (int i = 0; i < 8; i += 2)
                sq = fma2_rn(make_float2(d[i], d[i + 1]), make_float2(d[i], d[i + 1]), sq);
        } else {
            cw[k] = canonical_zero(e2m1x8(v));
        }
    }
    if (SSE) sse = a > 0.0f ? (double)(sq.x + sq.y) * exp2i_f64(2 * e) : 0.0;   // 2e in [-254, 254]: exact
    sb_out = sb;
}

// ---------------------------------------------------------------------------
// Decoders (dequantize and error)
// ---------------------------------------------------------------------------

template <int FMT>
__device__ __forceinline__ void decode_nv16(uint32_t w0, uint32_t w1, uint32_t sb, float s_t, float* xh)
{
    constexpr bool RAZER = kRazer<FMT>;
    const float den = __fmul_rn(nv_scale_value<FMT>(sb), s_t);
    const float special = razer_special<FMT>(sb);
    float q[16];
    decode16(w0, w1, q);
    if (RAZER) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t nib = ((i < 8 ? w0 : w1) >> (4 * (i & 7))) & 0xFu;
            q[i] = nib == 8u ? special : q[i];
        }
    }
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const float2 p = mul2_rn(make_float2(q[i], q[i + 1]), make_float2(den, den));
        xh[i] = p.x;
        xh[i + 1] = p.y;
    }
}

__device__ __forceinline__ void decode_mx32(const uint32_t* cw, uint32_t sb, float* xh)
{
    const float s = exp2i((int)sb - 127);
    float q[32];
    decode16(cw[0], cw[1], q);
    decode16(cw[2], cw[3], q + 16);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        const float2 p = mul2_rn(make_float2(q[i], q[i + 1]), make_float2(s, s));
        xh[i] = p.x;
        xh[i + 1] = p.y;
    }
}

template <int FMT>
__device__ __forceinline__ void decode_unit(const uint32_t* cw, const uint32_t* sb, float s_t, float* xh)
{
    if (FMT == kMX) {
        decode_mx32(cw, sb[0], xh);
    } else {
        decode_nv16<FMT>(cw[0], cw[1], sb[0], s_t, xh);
        decode_nv16<FMT>(cw[2], cw[3], sb[1], s_t, xh + 16);
    }
}

// Read a unit's codes and scale bytes (dense layouts).
// With FP4Q_DEBUG, code_bytes and scale_bytes bound the two reads (an
// out-of-bounds read is recorded in err and reads zeros instead).
template <int FMT>
__device__ __forceinline__ void load_packed(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                            int64_t code_off, int64_t scale_off, bool full, bool a16, uint32_t* cw,
                                            uint32_t* sb, int64_t code_bytes = 0, int64_t scale_bytes = 0,
                                            unsigned* err = nullptr)
{
    constexpr int B = FMT == kMX ? 32 : 16;
    if (!in_bounds(code_off, full ? 16 : 8, code_bytes, kSiteCodesLoad, err) ||
        !in_bounds(scale_off, (FMT != kMX && full) ? 2 : 1, scale_bytes, kSiteScalesLoad, err)) {
        cw[0] = cw[1] = cw[2] = cw[3] = 0;
        sb[0] = sb[1] = 0;
        return;
    }
    (void)B;
    const uint8_t* cp = codes + code_off;
    if (full && a16) {
        const uint4 c = ldg_nc_v4(cp);
        cw[0] = c.x; cw[1] = c.y; cw[2] = c.z; cw[3] = c.w;
    } else {
        const uint2 c = __ldg(reinterpret_cast<const uint2*>(cp));
        cw[0] = c.x; cw[1] = c.y;
        if (full) {
            const uint2 d = __ldg(reinterpret_cast<const uint2*>(cp + 8));
            cw[2] = d.x; cw[3] = d.y;
        } else {
            cw[2] = 0; cw[3] = 0;
        }
    }
    sb[0] = __ldg(scales + scale_off);
    sb[1] = (FMT != kMX && full) ? (uint32_t)__ldg(scales + scale_off + 1) : 0u;
}

// ---------------------------------------------------------------------------
// The tile pipeline
// ---------------------------------------------------------------------------

// Shared memory of a pipelined CTA: kStages tiles (1024-byte aligned for the
// 128-byte swizzle), then a "full" and an "empty" mbarrier per stage.
// Dynamic shared memory of a pipeline of tiles of `tile_bytes`: the stages
// (1024-byte aligned), the alignment slack and the barriers.
constexpr int pipe_smem_bytes(int tile_bytes, int stages = kStages) { return stages * tile_bytes + 1024 + 128; }
constexpr int kPipeSmemBytes = pipe_smem_bytes(kTileBytes);
constexpr int kWarps = kThreads / 32;

// Stage s is "full" when its copy has landed (one arrival by thread 0 with the
// byte count, completed by the copy) and "empty" when every warp has finished
// reading it (one arrival per warp).  Warps consume tiles independently; only
// thread 0, which refills the stages, waits for a stage to become empty.
struct Pipe {
    uint32_t tiles;   // shared address of stage 0
    uint32_t full;    // shared address of the full barriers
    uint32_t empty;   // shared address of the empty barriers
};

template <int TILE_BYTES = kTileBytes, int WARPS = kWarps, int STAGES = kStages>
__device__ __forceinline__ Pipe pipe_setup(uint8_t* smem_raw)
{
    const uint32_t base = smem_u32(smem_raw);
    Pipe p;
    p.tiles = (base + 1023u) & ~1023u;
    p.full = p.tiles + STAGES * TILE_BYTES;
    p.empty = p.full + 8 * STAGES;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(p.full + 8 * s, 1);
            mbar_init(p.empty + 8 * s, WARPS);
        }
        mbar_init_fence();
    }
    __syncthreads();
    return p;
}

// Tiles of this CTA: blockIdx.x + j * gridDim.x, walked backwards when reverse.
struct Schedule {
    int64_t count, mine;
    bool reverse;
    __device__ int64_t tile(int64_t j) const
    {
        const int64_t i = (int64_t)blockIdx.x + j * gridDim.x;
        return reverse ? count - 1 - i : i;
    }
};

__device__ __forceinline__ Schedule make_schedule(int64_t count, bool reverse)
{
    Schedule s;
    s.count = count;
    s.reverse = reverse;
    s.mine = (int64_t)blockIdx.x < count ? (count - 1 - (int64_t)blockIdx.x) / gridDim.x + 1 : 0;
    return s;
}

// Thread 0: start the copy of the j-th tile of the schedule into its stage.
template <bool FLAT, int ROWS = kTileRows>
__device__ __forceinline__ void pipe_issue(const Pipe& p, const CUtensorMap* map, const Tiles& tl, const Schedule& sc,
                                           int64_t j)
{
    constexpr int kBytes = ROWS * 128;
    const int s = (int)(j % kStages);
    int x, y;
    tile_origin<FLAT, ROWS>(tl, sc.tile(j), x, y);
    mbar_arm(p.full + 8 * s, kBytes);
    tma_load_tile(p.tiles + s * kBytes, map, x, y, p.full + 8 * s);
}

// Every thread: wait (bounded) until the j-th tile has landed.
template <int STAGES = kStages>
__device__ __forceinline__ bool pipe_acquire(const Pipe& p, int64_t j)
{
    return mbar_wait(p.full + 8 * (int)(j % STAGES), (uint32_t)((j / STAGES) & 1));
}

// Every warp, after its last read of the j-th tile: release the stage.
template <int STAGES = kStages>
__device__ __forceinline__ void pipe_release(const Pipe& p, int64_t j)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(p.empty + 8 * (int)(j % STAGES)) : "memory");
}

// Thread 0: wait (bounded) until every warp has released the j-th tile's stage.
template <int STAGES = kStages>
__device__ __forceinline__ bool pipe_stage_free(const Pipe& p, int64_t j)
{
    return mbar_wait(p.empty + 8 * (int)(j % STAGES), (uint32_t)((j / STAGES) & 1));
}

// After a timeout: record it in the error words `err`; thread 0 waits
// (bounded) for the copies it issued that may still be in flight, tiles
// [from, to) of the schedule.
template <int STAGES = kStages>
__device__ __forceinline__ void pipe_fail(const Pipe& p, int64_t from, int64_t to, unsigned* err)
{
    if ((threadIdx.x & 31) == 0) atomicOr(err, kErrPipelineTimeout);
    if (threadIdx.x == 0)
        for (int64_t q = from; q < to; ++q) pipe_acquire<STAGES>(p, q);
}

__device__ __forceinline__ void load_unit_words(uint32_t tile, uint32_t r, uint32_t h, uint32_t* w)
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 v = lds128(tile_chunk(tile, r, 4 * h + c));
        w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
    }
}


// ---------------------------------------------------------------------------
// Per-tile work (shared by the single-tensor kernels and the batch scheduler)
// ---------------------------------------------------------------------------

// Block `half` of the unit (r, h) encoded again in the exact way from the tile
// (rotated again when ROT): codes, scale byte and the error in fp64, with
// division wherever RN(1 / den) overflowed.  Out of line and by value, so that
// the fast path keeps its registers; only blocks that path does not cover
// come here.
template <int FMT, bool ROT>
__device__ __noinline__ BlockOut nv_block_redo(uint32_t tile, uint32_t r, uint32_t h, uint32_t half, NvScale nsc)
{
    float y[32];
    {
        uint32_t w[16];
        load_unit_words(tile, r, h, w);
        if (ROT) {
            wht32_from_bf16(w, y);
        } else {
            unpack16(w, y);
            unpack16(w + 8, y + 16);
        }
    }
    const float* yb = half ? y + 16 : y;
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(yb[i]));
    const uint32_t sb = nv_scale_code<FMT>(nsc, a);
    const float2 dr = nv_den_rcp(nsc, sb);
    BlockOut o;
    nv_block_exact_f32<FMT, true, true>(yb, sb, dr.x, dr.y, o.w0, o.w1, o.sb, o.sse);
    return o;
}

// Q1-Q6 on the unit this thread owns in tile k (shared address `tile`):
// rotate, block scales, encode, RaZeR select, pack and store codes and scales.
// Returns the unit's squared error when SSE: in the original domain without
// rotation; with rotation in the rotated domain, which the orthonormal
// transform H / sqrt(32) maps onto the original one up to the fp32 rounding of
// the rotated values (about 2^-24 of each value, far inside the rotated
// paths' 1e-3 MSE tolerance).
template <int FMT, bool ROT, bool SSE, bool FLAT, int ROWS = kTileRows>
__device__ __forceinline__ double quantize_tile(uint32_t tile, const Tiles& tl, int64_t k, uint8_t* codes,
                                                uint8_t* scales, const NvScale& nsc, bool mx_ceil, unsigned* err)
{
    const int t = threadIdx.x;
    const bool a16 = FLAT || (tl.cols % 32) == 0;
    const uint32_t r = (uint32_t)t >> 1, h = (uint32_t)t & 1u;
    double acc = 0.0;
    const Unit u = unit_of<FLAT, ROWS>(tl, k, t);
    uint32_t cw[4] = {0, 0, 0, 0}, sb0 = 0, sb1 = 0;
    if (u.valid) {
        if (FMT != kMX && !ROT) {
            // two independent 16-element blocks, one after the other
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (half == 1 && !u.full) break;
                uint32_t w[8];
                const uint32_t a0 = tile_chunk(tile, r, 4 * h + 2 * half);
                const uint32_t a1 = tile_chunk(tile, r, 4 * h + 2 * half + 1);
                const uint4 v0 = lds128(a0), v1 = lds128(a1);
                w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
                w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
                uint32_t sbh;
                double e = 0.0;
                nv_block<FMT, SSE>(w, a0, a1, nsc, cw[2 * half], cw[2 * half + 1], sbh, e);
                if (half == 0) sb0 = sbh;
                else sb1 = sbh;
                if (SSE) acc += e;
            }
        } else {
            // rotated NVFP4 / RaZeR, and MXFP4: the error in the scaled (and rotated) domain
            float y[32];
            {
                uint32_t w[16];
                load_unit_words(tile, r, h, w);
                if (ROT) {
                    wht32_from_bf16(w, y);
                } else {
                    unpack16(w, y);
                    unpack16(w + 8, y + 16);
                }
            }
            if (FMT == kMX) {
                const float am = absmax_n<32>(y, 0.0f);
                double e = 0.0;
                mx_block<SSE>(y, am, mx_ceil, cw, sb0, e);
                if (SSE) acc += e;
            } else {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const float am = absmax_n<16>(y + 16 * half, 0.0f);
                    uint32_t c0 = 0, c1 = 0, sbh = 0;
                    double e = 0.0;
                    if (!nv_block_f32<FMT, SSE>(y + 16 * half, am, nsc, c0, c1, sbh, e)) {
                        const BlockOut o = nv_block_redo<FMT, ROT>(tile, r, h, (uint32_t)half, nsc);
                        c0 = o.w0;
                        c1 = o.w1;
                        sbh = o.sb;
                        e = o.sse;
                    }
                    cw[2 * half] = c0;
                    cw[2 * half + 1] = c1;
                    if (half == 0) sb0 = sbh;
                    else sb1 = sbh;
                    if (SSE) acc += e;
                }
            }
        }
        int64_t co, so;
        unit_offsets<FLAT, FMT>(tl, u, co, so);
        constexpr int B = FMT == kMX ? 32 : 16;
        const int64_t n = tl.rows * tl.cols;   // the bounds of the debug build's checks
        if (in_bounds(co, u.full ? 16 : 8, n / 2, kSiteCodesStore, err)) store_codes(codes + co, cw, u.full, a16);
        if (in_bounds(so, (FMT != kMX && u.full) ? 2 : 1, n / B, kSiteScalesStore, err)) {
            if (FMT == kMX) {
                scales[so] = (uint8_t)sb0;
            } else if (u.full && a16) {
                *reinterpret_cast<unsigned short*>(scales + so) = (unsigned short)(sb0 | (sb1 << 8));
            } else {
                scales[so] = (uint8_t)sb0;
                if (u.full) scales[so + 1] = (uint8_t)sb1;
            }
        }
    }
    return acc;
}

// Q0 on the unit this thread owns in a tile: max |x| (of |H x| when rotating).
// Out-of-range parts of a tile are zero-filled, so no validity test is needed.
template <bool ROT>
__device__ __forceinline__ float amax_tile(uint32_t tile)
{
    const int t = threadIdx.x;
    uint32_t w[16];
    load_unit_words(tile, (uint32_t)t >> 1, (uint32_t)t & 1u, w);
    float m = 0.0f;
    if (ROT) {
        float y[32];
        wht32_from_bf16(w, y);
        m = absmax_n<32>(y, 0.0f);
    } else {
        uint32_t mm = w[0];
#pragma unroll
        for (int i = 1; i < 16; ++i) mm = bf16x2_absmax(mm, w[i]);
        m = bf16x2_hmax_abs(mm);
    }
    return m;
}

}  // namespace fp4q
