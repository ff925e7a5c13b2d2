// Device helpers for the fp4q kernels (sm_100a).
//
// Number formats follow "RaZeR: Pushing the Limits of NVFP4 Quantization with
// Redundant Zero Remapping" (technical summary sect. 1: E2M1 elements
// {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit, FP8-E4M3 block scale; sect.
// 2.1 and 2.2: the 6-bit E3M3 block scale of its weight mode) and
// "TORQ: Two-Level Orthogonal Rotation for MXFP4 Quantization" (sect. 1:
// 32-element blocks with a shared power-of-two scale).  Conversions use the
// hardware cvt instructions of sm_100a: E2M1 and E4M3 encoding round to
// nearest even and saturate to the largest finite value, which is the
// element and scale rounding rule of this library.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace fp4q {

// RN_f32(1 / sqrt(32)), the normalisation of the 32-point Walsh-Hadamard transform.
__device__ __forceinline__ float wht_scale() { return __uint_as_float(0x3E3504F3u); }

// ---- bf16 -----------------------------------------------------------------

// A 32-bit word holds elements 2k (low half) and 2k+1 (high half); widening is exact.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Both halves widened with the mixed-precision add (x + -0 is exact for every
// finite x, zeros keep their sign), which runs on the FMA pipe rather than on
// the integer pipe.
__device__ __forceinline__ float2 bf16x2_to_f32(uint32_t w)
{
    float lo, hi;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "add.rn.f32.bf16 %0, l, 0f80000000;\n\tadd.rn.f32.bf16 %1, h, 0f80000000;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(w));
    return make_float2(lo, hi);
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// max(|a|, |b|) of two bf16 pairs at once (the sign bits of the result are the
// xor of the inputs' and carry no meaning here); exact.
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// |max| of the two bf16 halves of a word, as fp32.
__device__ __forceinline__ float bf16x2_hmax_abs(uint32_t w)
{
    return fmaxf(fabsf(bf16_lo(w)), fabsf(bf16_hi(w)));
}

// ---- packed fp32 pairs (IEEE round-to-nearest per lane, no flush to zero) ----

__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b)
{
    float2 r;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 sub2_rn(float2 a, float2 b)
{
    float2 r;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 add2_rn(float2 a, float2 b)
{
    float2 r;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

// a * b + c per lane, one rounding.
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c)
{
    float2 r;
    asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mov.b64 c, {%6, %7};\n\tfma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

// ---- E2M1 -----------------------------------------------------------------

// Eight fp32 values -> eight E2M1 nibbles (value i in bits 4i..4i+3), nearest
// even, saturating.  Negative values that round to zero come out as 0b1000.
__device__ __forceinline__ uint32_t e2m1x8(const float* v)
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// As e2m1x8, and e[i] = q_i - v[i] with q_i the grid value of nibble i (the
// codes are decoded back to f16 and subtracted in one mixed-precision
// rounding).  The difference is exact: q_i is the grid point nearest v[i],
// or +-6 when |v[i]| > 6, so q_i - v[i] is a multiple of ulp(v[i]) and no
// larger than max(|v[i]|, 1).
__device__ __forceinline__ uint32_t e2m1x8_diff(const float* v, float* e)
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 h0, h1, h2, h3;\n\t"
        ".reg .b16 l0, u0, l1, u1, l2, u2, l3, u3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %12, %11;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %14, %13;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %16, %15;\n\t"
        "cvt.rn.f16x2.e2m1x2 h0, b0;\n\tcvt.rn.f16x2.e2m1x2 h1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 h2, b2;\n\tcvt.rn.f16x2.e2m1x2 h3, b3;\n\t"
        "mov.b32 {l0, u0}, h0;\n\tmov.b32 {l1, u1}, h1;\n\t"
        "mov.b32 {l2, u2}, h2;\n\tmov.b32 {l3, u3}, h3;\n\t"
        "sub.rn.f32.f16 %1, l0, %9;\n\tsub.rn.f32.f16 %2, u0, %10;\n\t"
        "sub.rn.f32.f16 %3, l1, %11;\n\tsub.rn.f32.f16 %4, u1, %12;\n\t"
        "sub.rn.f32.f16 %5, l2, %13;\n\tsub.rn.f32.f16 %6, u2, %14;\n\t"
        "sub.rn.f32.f16 %7, l3, %15;\n\tsub.rn.f32.f16 %8, u3, %16;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out), "=f"(e[0]), "=f"(e[1]), "=f"(e[2]), "=f"(e[3]), "=f"(e[4]), "=f"(e[5]), "=f"(e[6]),
          "=f"(e[7])
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// Rewrite every -0 nibble (0b1000) as +0: a nibble keeps its sign bit only if
// its magnitude is nonzero.  (mag + 7) carries into bit 3 exactly when mag >= 1,
// and never into the next nibble.
__device__ __forceinline__ uint32_t canonical_zero(uint32_t w)
{
    uint32_t nz = (w & 0x77777777u) + 0x77777777u;
    return w & ((nz & 0x88888888u) | 0x77777777u);
}

// Eight E2M1 nibbles (one word, element i in bits 4i..4i+3) -> eight fp32
// values; the word is split into bytes inside the conversion block.
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t w, float* q)
{
    uint32_t h0, h1, h2, h3;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(w));
    const uint32_t h[4] = {h0, h1, h2, h3};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[k]));
        q[2 * k] = f.x;
        q[2 * k + 1] = f.y;
    }
}

// Two E2M1 nibbles (bits 0..3 element 2k, bits 4..7 element 2k+1) -> two fp32 values.
__device__ __forceinline__ float2 e2m1x2_to_f32(uint32_t byte)
{
    uint32_t h;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h) : "r"(byte));
    __half2 hh = *reinterpret_cast<__half2*>(&h);
    return __half22float2(hh);  // .x = low half = element 2k
}

// ---- E4M3 -----------------------------------------------------------------

// Non-negative fp32 -> E4M3 byte, nearest even, saturating at 448 (0x7E).
__device__ __forceinline__ uint32_t e4m3_rn_satfinite(float t)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
    return r & 0xFFu;
}

// E4M3 byte (sign included) -> fp32, exact.
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte)
{
    uint32_t h;
    uint16_t in = (uint16_t)(byte & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

// ---- E3M3 (block scale of the RaZeR weight mode) ---------------------------
//
// Unsigned; exponent field e (3 bits, bias 3) and mantissa m (3 bits):
// (1 + m/8) 2^(e-3) for e > 0, m 2^-5 for e = 0; largest value 30 (0x3F).

// Non-negative finite fp32 -> E3M3 code, nearest even, saturating at 30.  From
// 0.25 (the smallest normal) up to 30, E3M3 and E4M3 have the same values and
// the same 3-bit mantissa, so the E4M3 conversion of min(t, 30) is the E3M3
// code with 4 added to the exponent field; below 0.25 the quantum is 2^-5
// throughout and the code is RN_even(32 t), in [0, 8] (8 encodes 0.25).
__device__ __forceinline__ uint32_t e3m3_rn_sat(float t)
{
    const uint32_t lo = (uint32_t)__float2int_rn(t * 32.0f);
    const uint32_t hi = e4m3_rn_satfinite(fminf(t, 30.0f)) - 32u;
    return t < 0.25f ? lo : hi;
}

// E3M3 code (6 bits) -> fp32, exact.
__device__ __forceinline__ float e3m3_to_f32(uint32_t c)
{
    const uint32_t e = (c >> 3) & 7u, m = c & 7u;
    return e == 0u ? (float)m * 0x1p-5f : __uint_as_float(((e + 124u) << 23) | (m << 20));
}

// ---- E8M0 -----------------------------------------------------------------

// floor(log2 a) for a finite a > 0, from the binary32 fields (subnormals included).
__device__ __forceinline__ int floor_log2_f32(float a)
{
    uint32_t u = __float_as_uint(a);
    int ex = (int)((u >> 23) & 0xFFu);
    if (ex != 0) return ex - 127;
    return (31 - __clz((int)u)) - 149;
}

// 1 when the significand of a finite a > 0 exceeds 1.5 (a > 1.5 * 2^floor(log2 a)).
__device__ __forceinline__ int significand_above_1p5(float a)
{
    const uint32_t u = __float_as_uint(a);
    if ((u >> 23) & 0xFFu) return (u & 0x7FFFFFu) > 0x400000u ? 1 : 0;
    const int b = 31 - __clz((int)u);                    // subnormal: leading bit of u
    return b > 0 && (u & ((1u << b) - 1u)) > (1u << (b - 1)) ? 1 : 0;
}

// 2^k for k in [-127, 127] as fp32 (2^-127 is subnormal).
__device__ __forceinline__ float exp2i(int k)
{
    return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// 2^k for k in [-1022, 1023] as fp64, from its exponent field.
__device__ __forceinline__ double exp2i_f64(int k)
{
    return __longlong_as_double((long long)(k + 1023) << 52);
}

// max(|y_0|, ..., |y_{n-1}|, m) with three-input maxima.
template <int N>
__device__ __forceinline__ float absmax_n(const float* y, float m)
{
    int i = 0;
#pragma unroll
    for (; i + 1 < N; i += 2) {
        const float a = fabsf(y[i]), b = fabsf(y[i + 1]);
        asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(m), "f"(a), "f"(b));
    }
    if (i < N) m = fmaxf(m, fabsf(y[i]));
    return m;
}

// ---- 32-point Walsh-Hadamard, in registers ----------------------------------

// y <- H32 y (Sylvester order: H_ij = (-1)^popcount(i & j)), fp32 butterflies,
// then y <- RN(y * RN(1/sqrt 32)).  The transform is its own inverse.
// Stage h = 1 pairs neighbours and runs scalar; stages h = 2..16 pair whole
// pairs (y[i], y[i+1]) with (y[i+h], y[i+h+1]) and run two butterflies per
// packed add / sub.  Every lane rounds as the scalar operation would, so the
// result is the same bit for bit.
// Butterfly stages of stride 2..16 and the 1/sqrt(32) scale (the stride-1
// stage done).
__device__ __forceinline__ void wht32_rest(float* y)
{
#pragma unroll
    for (int h = 2; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            if ((i & h) == 0) {
                const float2 a = make_float2(y[i], y[i + 1]), b = make_float2(y[i + h], y[i + h + 1]);
                const float2 s = add2_rn(a, b), d = sub2_rn(a, b);
                y[i] = s.x;
                y[i + 1] = s.y;
                y[i + h] = d.x;
                y[i + h + 1] = d.y;
            }
        }
    }
    const float c = wht_scale();
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        const float2 p = mul2_rn(make_float2(y[i], y[i + 1]), make_float2(c, c));
        y[i] = p.x;
        y[i + 1] = p.y;
    }
}

__device__ __forceinline__ void wht32_inplace(float* y)
{
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        const float a = y[i], b = y[i + 1];
        y[i] = a + b;
        y[i + 1] = a - b;
    }
    wht32_rest(y);
}

// The same transform of the 32 bf16 values of w (element 2k in the low half
// of w[k]): the stride-1 stage adds and subtracts each word's two values
// straight from bf16 (add/sub.rn.f32.bf16 convert the bf16 operand exactly
// and round once, as the fp32 add of the unpacked values does), which saves
// unpacking the low halves.
__device__ __forceinline__ void wht32_from_bf16(const uint32_t* w, float* y)
{
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float hi = __uint_as_float(w[k] & 0xFFFF0000u);
        asm("{\n\t.reg .b16 lo, up;\n\tmov.b32 {lo, up}, %2;\n\t"
            "add.rn.f32.bf16 %0, lo, %3;\n\tsub.rn.f32.bf16 %1, lo, %3;\n\t}"
            : "=f"(y[2 * k]), "=f"(y[2 * k + 1])
            : "r"(w[k]), "f"(hi));
    }
    wht32_rest(y);
}

// ---- loads / stores -------------------------------------------------------

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ void stg_v4(void* p, uint4 v)
{
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__device__ __forceinline__ void stg_v2(void* p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(a), "r"(b) : "memory");
}

}  // namespace fp4q
