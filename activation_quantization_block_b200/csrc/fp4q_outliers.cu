// Sparse outlier separation ahead of block quantization, and the scatter that
// puts the outliers back into a reconstruction.
//
// "XFP: quality-targeted adaptive codebook quantization", technical summary
// sect. 2 (sparse outlier separation): weights with |w - mu| > k sigma (k = 4,
// at most 2 % of the weights) are kept apart as fp16 values at their
// positions, and the bulk, with the group mean in their place, is quantized.
// The group is a matrix row, handled by one warp (rows of up to 8192 elements)
// or one CTA, the row copied once into shared memory:
//   1. mu and sigma in one fp64 pass over the row (sums of x - c and of its
//      square around c, the row's first element; fixed-order reductions),
//      threshold T = k sigma;
//   2. one pass writes the bulk row (the mean, rounded to bf16, at every
//      outlier) and the outliers in column order, their slots from prefix
//      counts; |x - mu| > T is decided in fp32 outside a guard band that covers
//      the fp32 roundings, in fp64 inside it; a step in which no element of the
//      warp (or CTA) comes near the threshold copies the row and counts nothing;
//   3. only if that pass counted more than cap = floor(max_frac * n): T becomes
//      the cap-th largest deviation, found by bisection on the deviations' fp64
//      bit patterns (monotone for non-negative values), ties at T are taken
//      from the lowest columns up, and step 2 runs again.
// Each thread moves 16 bytes at a time.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fp4q_common.cuh"

namespace fp4q {

namespace {

constexpr int kOutThreads = 256;
constexpr int kOutTile = kOutThreads * 8;   // elements per tile: 8 per thread

struct OutlierArgs {
    const uint16_t* x;
    uint16_t* bulk;
    uint16_t* out_cols;
    uint16_t* out_vals;
    int32_t* out_count;
    int64_t ldx, ldb, cols, cap;
    double k;
    int64_t rows;
    unsigned* err;          // the library's device error words
};

// Sum over the CTA in a fixed order, result in every thread.
__device__ double cta_sum(double v, double* sh)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kOutThreads / 32 ? sh[lane] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if (lane == 0) sh[32] = v;
    }
    __syncthreads();
    return sh[32];
}

__device__ long long cta_count(long long v, long long* sh)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kOutThreads / 32 ? sh[lane] : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if (lane == 0) sh[32] = v;
    }
    __syncthreads();
    return sh[32];
}

// Exclusive prefix of v over the CTA in thread order; *total receives the sum.
__device__ int cta_exclusive_scan(int v, int* sh, int* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += n;
    }
    __syncthreads();
    if (lane == 31) sh[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kOutThreads / 32 ? sh[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < kOutThreads / 32) sh[lane] = wi - w;   // exclusive warp offsets
        if (lane == kOutThreads / 32 - 1) sh[32] = wi;
    }
    __syncthreads();
    *total = sh[32];
    return sh[warp] + inc - v;
}

// Copy n16 16-byte chunks from global to shared memory, `stride` threads
// taking chunk i, i + stride, ...: eight loads in flight per thread.
__device__ __forceinline__ void copy_row(uint4* dst, const uint4* src, int64_t n16, int64_t i, int64_t stride)
{
    for (; i < n16; i += 8 * stride) {
        uint4 r[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (i + q * stride < n16) r[q] = __ldg(src + i + q * stride);
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (i + q * stride < n16) dst[i + q * stride] = r[q];
    }
}

// Eight bf16 values of the row in shared memory (byte address srow) from
// column j (j % 8 == 0), as fp32.
__device__ __forceinline__ void load8(uint32_t srow, int64_t j, float* v)
{
    const uint4 w = lds128(srow + 2u * (uint32_t)j);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_lo(u[i]);
        v[2 * i + 1] = bf16_hi(u[i]);
    }
}

// binary64 -> bf16 bits, nearest even: truncate to binary32 and, if inexact,
// set its last bit (round to odd), then round to bf16; binary32 keeps 16 bits
// more than bf16, so the two roundings equal one.
__device__ __forceinline__ uint16_t f64_to_bf16_rn(double m)
{
    float f = __double2float_rz(m);
    if ((double)f != m) f = __uint_as_float(__float_as_uint(f) | 1u);
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Mean and population deviation of a row of n8 16-byte chunks of bf16 in
// shared memory, in one pass: the sums S1 = sum (x - c) and S2 = sum (x - c)^2
// around c, the row's first element, give mu = c + S1 / n and
// sigma^2 = S2 / n - (S1 / n)^2 (taken as 0 if rounding makes it negative).
// Every difference, square and sum is fp64, eight partial sums per thread
// combined in a fixed order and then by `reduce` (a fixed-order sum over the
// warp or the CTA).  Shifting by an element of the row keeps the cancellation
// in sigma^2 small: its relative rounding is about 2^-53 ((mu - c) / sigma)^2.
template <typename Reduce>
__device__ __forceinline__ void row_moments(uint32_t row, int64_t n8, int64_t first, int64_t stride, double c,
                                            Reduce reduce, double& mu, double& sigma)
{
    double p1[8] = {0, 0, 0, 0, 0, 0, 0, 0}, p2[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int64_t i = first; i < n8; i += stride) {
        float v[8];
        load8(row, 8 * i, v);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const double d = (double)v[q] - c;
            p1[q] += d;
            p2[q] = fma(d, d, p2[q]);
        }
    }
    const double n = (double)(8 * n8);
    const double s1 = reduce(((p1[0] + p1[1]) + (p1[2] + p1[3])) + ((p1[4] + p1[5]) + (p1[6] + p1[7])));
    const double s2 = reduce(((p2[0] + p2[1]) + (p2[2] + p2[3])) + ((p2[4] + p2[5]) + (p2[6] + p2[7])));
    const double m1 = s1 / n;
    mu = c + m1;
    sigma = sqrt(fmax(s2 / n - m1 * m1, 0.0));
}

__global__ void __launch_bounds__(kOutThreads) outlier_rows_kernel(OutlierArgs a)
{
    extern __shared__ uint4 srow_raw[];
    __shared__ double shd[33];
    __shared__ long long shl[33];
    __shared__ int shi[33];
    const int64_t r = blockIdx.x;
    const int t = threadIdx.x;
    const int64_t n = a.cols;
    const uint32_t row = smem_u32(srow_raw);
    if (!in_bounds(2 * r * a.ldx, 2 * n, 2 * ((a.rows - 1) * a.ldx + n), kSiteOutlierRowLoad, a.err)) return;
    copy_row(srow_raw, reinterpret_cast<const uint4*>(a.x + r * a.ldx), n / 8, t, kOutThreads);
    __syncthreads();

    // 1. mean and deviation, one pass over the row in shared memory
    double mu, thr;
    {
        float v0[8];
        load8(row, 0, v0);
        row_moments(row, n / 8, t, kOutThreads, (double)v0[0], [&](double v) { return cta_sum(v, shd); }, mu, thr);
        thr *= a.k;
    }

    // 2. bulk row and outliers in column order, speculatively with k sigma (the
    // count stays within the cap in the usual case); above the cap, the cap-th
    // largest deviation, its ties from the lowest column up, and the pass again.
    auto count_where = [&](auto pred) {
        long long c = 0;
        for (int64_t j = 8 * (int64_t)t; j < n; j += kOutTile) {
            float v[8];
            load8(row, j, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) c += pred(fabs((double)v[i] - mu)) ? 1 : 0;
        }
        return cta_count(c, shl);
    };
    const uint16_t mub = f64_to_bf16_rn(mu);
    uint16_t* brow = a.bulk + r * a.ldb;
    const int64_t bulk_bytes = 2 * ((a.rows - 1) * a.ldb + n);   // the debug build's bound of the bulk
    // d > t in fp32 outside a band covering the fp32 roundings of mu, t and d
    // (2^-20 of |mu| + t), in fp64 inside it; slots past the capacity are not written
    auto compact = [&](double t, long long tie_need, bool none) -> long long {
        const float mu32 = (float)mu, t32 = (float)t;
        const float band = 0x1p-20f * (fabsf(mu32) + t32);
        long long done = 0, ties_seen = 0;
        for (int64_t j0 = 0; j0 < n; j0 += kOutTile) {
            const int64_t j = j0 + 8 * (int64_t)threadIdx.x;
            const bool in = j < n;
            float v[8];
            uint4 w = make_uint4(0, 0, 0, 0);
            if (in) {
                w = lds128(row + 2u * (uint32_t)j);
                load8(row, j, v);
            }
            // the usual step: no element of the CTA's chunks near or above the
            // threshold, so the bulk is the row unchanged and nothing is counted
            float dm = 0.0f;
            if (in && !none) {
#pragma unroll
                for (int i = 0; i < 8; ++i) dm = fmaxf(dm, fabsf(v[i] - mu32));
            }
            if (__syncthreads_and(none || dm - t32 < -band)) {
                if (in && in_bounds(2 * (r * a.ldb + j), 16, bulk_bytes, kSiteBulkStore, a.err))
                    *reinterpret_cast<uint4*>(brow + j) = w;
                continue;
            }
            uint32_t gmask = 0, emask = 0;
            if (in && !none) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float d32 = fabsf(v[i] - mu32);
                    if (d32 - t32 > band && d32 <= 3.4e38f) {
                        gmask |= 1u << i;
                    } else if (!(d32 - t32 < -band)) {
                        const double d = fabs((double)v[i] - mu);
                        if (d > t) gmask |= 1u << i;
                        else if (d == t && tie_need > 0) emask |= 1u << i;
                    }
                }
            }
            int eq_total;
            int rank = (int)ties_seen + cta_exclusive_scan(__popc(emask), shi, &eq_total);
            uint32_t omask = gmask;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (emask & (1u << i)) {
                    if (rank < tie_need) omask |= 1u << i;
                    ++rank;
                }
            ties_seen += eq_total;
            int tot;
            long long slot = done + cta_exclusive_scan(__popc(omask), shi, &tot);
            if (in) {
                uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (omask & (1u << i)) {
                        const uint32_t sh = (i & 1) ? 16u : 0u;
                        u[i >> 1] = (u[i >> 1] & ~(0xFFFFu << sh)) | ((uint32_t)mub << sh);
                        if (slot < a.cap &&
                            in_bounds(2 * (r * a.cap + slot), 2, 2 * a.rows * a.cap, kSiteSlotStore, a.err)) {
                            a.out_cols[r * a.cap + slot] = (uint16_t)(j + i);
                            a.out_vals[r * a.cap + slot] =
                                __half_as_ushort(__float2half_rn(fminf(fmaxf(v[i], -65504.0f), 65504.0f)));
                        }
                        ++slot;
                    }
                if (in_bounds(2 * (r * a.ldb + j), 16, bulk_bytes, kSiteBulkStore, a.err))
                    *reinterpret_cast<uint4*>(brow + j) = make_uint4(u[0], u[1], u[2], u[3]);
            }
            done += tot;
        }
        return done;
    };
    long long total = compact(thr, 0, a.cap == 0);
    if (a.cap > 0 && total > a.cap) {
        unsigned long long lo = 0ull, hi = 0x7FF0000000000000ull;   // bits of 0 and of +inf
        while (hi - lo > 1ull) {
            const unsigned long long mid = lo + (hi - lo) / 2;
            const long long c = count_where([&](double d) { return (unsigned long long)__double_as_longlong(d) >= mid; });
            if (c >= a.cap) lo = mid;
            else hi = mid;
        }
        thr = __longlong_as_double((long long)lo);
        total = compact(thr, a.cap - count_where([&](double d) { return d > thr; }), false);
    }
    if (t == 0 && in_bounds(4 * r, 4, 4 * a.rows, kSiteCountStore, a.err)) a.out_count[r] = (int32_t)total;
}

// The same, one warp per row (rows of at most 8192 elements): warp w of CTA b
// takes row R b + w (R rows per CTA, 8 or as many as 48 KB of shared memory
// holds), its copy in shared memory at w * cols * 2 bytes.  Sums are
// xor-butterflies, so every lane holds the same, bit for bit.
constexpr int kRowsPerCta = 8;

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ int warp_sum_int(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Exclusive prefix over the warp's lanes; *total receives the sum.
__device__ __forceinline__ int warp_exclusive_scan(int v, int* total)
{
    const int lane = threadIdx.x & 31;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += n;
    }
    *total = __shfl_sync(0xFFFFFFFFu, inc, 31);
    return inc - v;
}

__global__ void __launch_bounds__(32 * kRowsPerCta) outlier_rows_warp_kernel(OutlierArgs a, int64_t rows)
{
    extern __shared__ uint4 srows_raw[];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + w;
    if (r >= rows) return;   // warp-uniform
    const int64_t n = a.cols, n8 = n / 8;
    uint4* srow = srows_raw + (int64_t)w * n8;
    const uint32_t row = smem_u32(srow);
    if (!in_bounds(2 * r * a.ldx, 2 * n, 2 * ((rows - 1) * a.ldx + n), kSiteOutlierRowLoad, a.err)) return;
    copy_row(srow, reinterpret_cast<const uint4*>(a.x + r * a.ldx), n8, lane, 32);
    __syncwarp();

    double mu, thr;
    {
        float v0[8];
        load8(row, 0, v0);
        row_moments(row, n8, lane, 32, (double)v0[0], [](double v) { return warp_sum(v); }, mu, thr);
        thr *= a.k;
    }

    auto count_where = [&](auto pred) {
        int c = 0;
        for (int64_t i = lane; i < n8; i += 32) {
            float v[8];
            load8(row, 8 * i, v);
            uint32_t m = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) m |= pred(fabs((double)v[q] - mu)) ? 1u << q : 0u;
            c += __popc(m);
        }
        return (long long)warp_sum_int(c);
    };
    const uint16_t mub = f64_to_bf16_rn(mu);
    uint16_t* brow = a.bulk + r * a.ldb;
    const int64_t bulk_bytes = 2 * ((a.rows - 1) * a.ldb + n);   // the debug build's bound of the bulk
    // One pass: bulk row and outlier slots for threshold t (and, when tie_need > 0,
    // the first tie_need elements with d == t).  d > t is decided in fp32 where
    // |d32 - t32| exceeds a band covering the fp32 roundings of mu, t and d (each
    // at most 2^-24 relative; the band is 2^-20 of |mu| + t), in fp64 elsewhere.
    // Slots past the capacity are not written.  Returns the row's count.
    auto compact = [&](double t, long long tie_need, bool none) -> long long {
        const float mu32 = (float)mu, t32 = (float)t;
        const float band = 0x1p-20f * (fabsf(mu32) + t32);
        long long done = 0, ties_seen = 0;
        for (int64_t i0 = 0; i0 < n8; i0 += 32) {
            const int64_t i = i0 + lane;
            const bool in = i < n8;
            float v[8];
            uint4 wd = make_uint4(0, 0, 0, 0);
            if (in) {
                wd = lds128(row + 16u * (uint32_t)i);
                load8(row, 8 * i, v);
            }
            // the usual step: no element of the warp's chunks near or above the
            // threshold, so the bulk is the row unchanged and nothing is counted
            float dm = 0.0f;
            if (in && !none) {
#pragma unroll
                for (int q = 0; q < 8; ++q) dm = fmaxf(dm, fabsf(v[q] - mu32));
            }
            if (__all_sync(0xFFFFFFFFu, none || dm - t32 < -band)) {
                if (in && in_bounds(2 * (r * a.ldb + 8 * i), 16, bulk_bytes, kSiteBulkStore, a.err))
                    *reinterpret_cast<uint4*>(brow + 8 * i) = wd;
                continue;
            }
            uint32_t gmask = 0, emask = 0;
            if (in && !none) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float d32 = fabsf(v[q] - mu32);
                    if (d32 - t32 > band && d32 <= 3.4e38f) {
                        gmask |= 1u << q;
                    } else if (!(d32 - t32 < -band)) {   // near the threshold (or non-finite): fp64
                        const double d = fabs((double)v[q] - mu);
                        if (d > t) gmask |= 1u << q;
                        else if (d == t && tie_need > 0) emask |= 1u << q;
                    }
                }
            }
            int eq_total;
            int rank = (int)ties_seen + warp_exclusive_scan(__popc(emask), &eq_total);
            uint32_t omask = gmask;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (emask & (1u << q)) {
                    if (rank < tie_need) omask |= 1u << q;
                    ++rank;
                }
            ties_seen += eq_total;
            int tot;
            long long slot = done + warp_exclusive_scan(__popc(omask), &tot);
            if (in) {
                uint32_t u[4] = {wd.x, wd.y, wd.z, wd.w};
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (omask & (1u << q)) {
                        const uint32_t sh = (q & 1) ? 16u : 0u;
                        u[q >> 1] = (u[q >> 1] & ~(0xFFFFu << sh)) | ((uint32_t)mub << sh);
                        if (slot < a.cap &&
                            in_bounds(2 * (r * a.cap + slot), 2, 2 * a.rows * a.cap, kSiteSlotStore, a.err)) {
                            a.out_cols[r * a.cap + slot] = (uint16_t)(8 * i + q);
                            a.out_vals[r * a.cap + slot] =
                                __half_as_ushort(__float2half_rn(fminf(fmaxf(v[q], -65504.0f), 65504.0f)));
                        }
                        ++slot;
                    }
                if (in_bounds(2 * (r * a.ldb + 8 * i), 16, bulk_bytes, kSiteBulkStore, a.err))
                    *reinterpret_cast<uint4*>(brow + 8 * i) = make_uint4(u[0], u[1], u[2], u[3]);
            }
            done += tot;
        }
        return done;
    };

    // Speculatively with k sigma (the usual case: the count stays within the cap);
    // otherwise the cap-th largest deviation, its ties, and the pass again.
    long long total = compact(thr, 0, a.cap == 0);
    if (a.cap > 0 && total > a.cap) {
        unsigned long long lo = 0ull, hi = 0x7FF0000000000000ull;   // bits of 0 and of +inf
        while (hi - lo > 1ull) {
            const unsigned long long mid = lo + (hi - lo) / 2;
            const long long c = count_where([&](double d) { return (unsigned long long)__double_as_longlong(d) >= mid; });
            if (c >= a.cap) lo = mid;
            else hi = mid;
        }
        thr = __longlong_as_double((long long)lo);
        total = compact(thr, a.cap - count_where([&](double d) { return d > thr; }), false);
    }
    if (lane == 0 && in_bounds(4 * r, 4, 4 * a.rows, kSiteCountStore, a.err)) a.out_count[r] = (int32_t)total;
}

struct ScatterArgs {
    const uint16_t* out_cols;
    const uint16_t* out_vals;
    const int32_t* out_count;
    uint16_t* y;
    int64_t rows, cols, cap, ldy;
    unsigned* err;          // the library's device error words
};

// One thread per (row, slot): the slot's fp16 value, as bf16, to its column.
// A column at or past cols is skipped, so that arrays not made by the
// separation can never write into y's padding columns [cols, ldy) (which may
// belong to another tensor) nor past the last row's cols elements.
__global__ void __launch_bounds__(256) outlier_scatter_kernel(ScatterArgs a)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.rows * a.cap) return;
    const int64_t r = i / a.cap, s = i - r * a.cap;
    if (s >= a.out_count[r]) return;
    const int64_t col = a.out_cols[i];
    if (col >= a.cols) return;
    if (!in_bounds(2 * (r * a.ldy + col), 2, 2 * ((a.rows - 1) * a.ldy + a.cols), kSiteScatterStore, a.err)) return;
    const float v = __half2float(__ushort_as_half(a.out_vals[i]));
    a.y[r * a.ldy + col] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

}  // namespace

int64_t outlier_capacity(int64_t cols, double max_frac) { return (int64_t)floor(max_frac * (double)cols); }

cudaError_t launch_separate_outliers(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx, double k, int64_t cap,
                                     uint16_t* bulk, int64_t ldb, uint16_t* out_cols, uint16_t* out_vals,
                                     int32_t* out_count, cudaStream_t st)
{
    if (rows == 0) return cudaSuccess;
    OutlierArgs a{x, bulk, out_cols, out_vals, out_count, ldx, ldb, cols, cap, k, rows, device_error_words()};
    if (a.err == nullptr) return cudaErrorInvalidSymbol;
    if (cols <= 8192) {   // one warp per row, at most 48 KB of rows per CTA
        int64_t rpc = (48 * 1024) / (cols * 2);
        rpc = rpc < 1 ? 1 : (rpc > kRowsPerCta ? kRowsPerCta : rpc);
        const int smem = (int)(rpc * cols * 2);
        const int64_t blocks = (rows + rpc - 1) / rpc;
        outlier_rows_warp_kernel<<<(unsigned)blocks, (unsigned)(32 * rpc), smem, st>>>(a, rows);
        return cudaGetLastError();
    }
    const int smem = (int)(cols * 2);   // the row, at most 128 KB
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(outlier_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   smem);
        if (e != cudaSuccess) return e;
    }
    outlier_rows_kernel<<<(unsigned)rows, kOutThreads, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_scatter_outliers(const uint16_t* out_cols, const uint16_t* out_vals, const int32_t* out_count,
                                    int64_t rows, int64_t cols, int64_t cap, uint16_t* y, int64_t ldy, cudaStream_t st)
{
    const int64_t n = rows * cap;
    if (n == 0) return cudaSuccess;
    const int64_t blocks = (n + 255) / 256;
    if (blocks >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    ScatterArgs a{out_cols, out_vals, out_count, y, rows, cols, cap, ldy, device_error_words()};
    if (a.err == nullptr) return cudaErrorInvalidSymbol;
    outlier_scatter_kernel<<<(unsigned)blocks, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace fp4q
