/*
 * fp4q -- block-scaled 4-bit quantization of bf16 matrices on NVIDIA B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only; every pointer argument to the tensor
 * entry points is a DEVICE pointer owned by the caller.  The library never
 * allocates, frees or synchronises inside these calls: each call validates its
 * arguments on the host, then enqueues kernels on `stream` and returns.
 *
 * Formats (element codes are 4-bit E2M1, sign in bit 3, magnitude index in
 * bits 0..2 over {0, 0.5, 1, 1.5, 2, 3, 4, 6} -- the FP4 value set of "RaZeR:
 * Pushing the Limits of NVFP4 Quantization with Redundant Zero Remapping",
 * technical summary sect. 1):
 *
 *  FP4Q_NVFP4        16-element blocks along a row.  Block scale: one FP8
 *                    E4M3 byte (the E4M3 block scale of RaZeR sect. 1).  Per
 *                    tensor: one fp32 scale s_t = RN(amax / (6 * 448)), so the
 *                    tensor maximum maps onto the largest code times the
 *                    largest E4M3 value.  Block b: sb = E4M3_RNE_sat(
 *                    RN(amax_b / RN(6 s_t))), den = RN(dec(sb) * s_t),
 *                    element code = nearest E2M1 to RN(x * RN(1 / den)),
 *                    ties to the even code, saturating at 6, zero as +0.
 *                    Reconstruction: RN(value(code) * den).
 *  FP4Q_NVFP4_RAZER  NVFP4 with redundant-zero remapping (RaZeR sect. 2.2):
 *                    code 0b1000 (the spare -0) means the special value +5,
 *                    or -5 when bit 7 of the scale byte (the spare sign bit of
 *                    the positive E4M3 scale) is set.  Per block the encoder
 *                    keeps the NVFP4 scale and codes, then picks the member of
 *                    {+5, -5} that lowers the block's squared error more (ties
 *                    and blocks with no gain keep +5 and bit 7 clear) and
 *                    recodes every element strictly closer to it than to its
 *                    regular value as 0b1000.  The scale magnitude is
 *                    bits 0..6.
 *  FP4Q_MXFP4        32-element blocks sharing one power-of-two scale ("TORQ:
 *                    Two-Level Orthogonal Rotation for MXFP4 Quantization",
 *                    technical summary sect. 1).  Scale byte E8M0 = e + 127
 *                    with e = clamp(floor(log2 amax_b) - 2, -127, 127);
 *                    element code = nearest E2M1 to x * 2^-e (exact scaling).
 *                    No tensor scale.
 *  FP4Q_NVFP4_RAZER_W  RaZeR weight mode (RaZeR sect. 2.1, 2.2): 16-element
 *                    blocks with a 6-bit unsigned E3M3 block scale (exponent
 *                    bias 3, exponent field 0 subnormal = m * 2^-5, largest
 *                    value 30) in bits 0..5 of the scale byte; bits 6..7 hold
 *                    the selector of the special value code 0b1000 stands
 *                    for: 0 -> +5, 1 -> -5, 2 -> +2.5, 3 -> -2.5 (the second
 *                    pair fixed offline by an error search over multiples of
 *                    0.5 on synthetic weights).  s_t = RN(amax / (6 * 30));
 *                    block scale E3M3_RNE_sat(RN(amax_b / RN(6 s_t))); codes
 *                    as NVFP4; per block the candidate with the largest
 *                    squared-error gain is chosen (ties: the lower selector)
 *                    and every element strictly closer to it than to its
 *                    regular value becomes 0b1000.
 *
 * rotate = 1 applies, before quantization, the orthonormal 32-point
 * Walsh-Hadamard transform y = RN(RN(H32 x) * RN(1/sqrt 32)) to every aligned
 * group of 32 elements of a row (H32 in Sylvester order; an orthogonal
 * intra-block rotation in the sense of TORQ sect. 2).  Quantization then acts
 * on y.  On dequantize and error, rotate = 1 means the codes hold rotated
 * values and the output is mapped back to the original domain with the same
 * (self-inverse) transform.  The butterfly is summed in fp32, so rotated
 * results can differ from an exact-sum reference by fp32 rounding.
 *
 * Layouts (all dense, row-major, caller-allocated, 16-byte aligned):
 *  x, y      bf16 [rows][ld], ld >= cols, ld a multiple of 8 elements.
 *  codes     uint8 [rows][cols/2]; element 2k in the low nibble of byte k.
 *  scales    uint8 [rows][cols/16] (NVFP4, NVFP4_RAZER, NVFP4_RAZER_W) or
 *            [rows][cols/32] (MXFP4).
 *  tensor_scale  one fp32 (NVFP4 formats; may be NULL for MXFP4).
 *  mse       one fp64: sum over all elements of (x - x^)^2 / (rows*cols),
 *            x^ the fp32 reconstruction (before any bf16 rounding) in the
 *            original domain, summed in fp64 in a fixed order.
 *
 * Shapes: cols must be a multiple of the block length (16 or 32) and of 32
 * when rotating.  rows * cols == 0 is allowed: nothing is launched except the
 * clearing of the scalar outputs (tensor_scale when computed, mse) to 0.
 *
 * Inputs must be finite.  NaN or infinity in x, a NaN scale byte (0x7F / 0xFF
 * in E4M3, 0xFF in E8M0) or a non-finite tensor scale are outside the
 * contract; the kernels do not fault on them, but the outputs are undefined.
 *
 * Errors: argument problems are reported before any launch as a status code,
 * and nothing is enqueued.  FP4Q_ERROR_CUDA reports a failed launch (the
 * library's own cudaGetLastError after its launches).  No call aborts,
 * throws, or falls back to the CPU.
 *
 * Thread safety: calls may come from any host thread.  A workspace buffer
 * must not be used by two calls that can run concurrently on the device.
 */
#ifndef FP4Q_H
#define FP4Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP4Q_ABI_VERSION 4

#if defined(__GNUC__)
#define FP4Q_API __attribute__((visibility("default")))
#else
#define FP4Q_API
#endif

typedef enum {
    FP4Q_NVFP4 = 0,
    FP4Q_NVFP4_RAZER = 1,
    FP4Q_MXFP4 = 2,
    FP4Q_NVFP4_RAZER_W = 3
} fp4q_format_t;

typedef enum {
    FP4Q_SUCCESS = 0,
    FP4Q_ERROR_INVALID_VALUE = 1,     /* null pointer, bad enum, bad flag, negative size */
    FP4Q_ERROR_SHAPE = 2,             /* cols not a multiple of the block / rotation group, ld < cols, size overflow */
    FP4Q_ERROR_MISALIGNED = 3,        /* pointer not 16-byte aligned, ld not a multiple of 8 */
    FP4Q_ERROR_WORKSPACE = 4,         /* workspace missing, misaligned or smaller than fp4q_workspace_size() */
    FP4Q_ERROR_UNSUPPORTED_DEVICE = 5,/* current device is not compute capability 10.0 (B200 / sm_100a) */
    FP4Q_ERROR_CUDA = 6               /* a CUDA runtime call or kernel launch failed */
} fp4q_status_t;

/* NVFP4 formats: *tensor_scale is an input; the tensor-absmax pass is skipped.
 * With *tensor_scale = 1 this is single-level NVFP4: the E4M3 block scale alone
 * carries the block's range (values whose block maximum / 6 falls below the
 * E4M3 normal range take subnormal scales). */
#define FP4Q_FLAG_TENSOR_SCALE_GIVEN 0x1u
/* MXFP4 only: the block exponent is the smallest e with amax_b <= 6 * 2^e (the
 * block maximum maps onto the largest code without clipping; "TORQ" sect. 2,
 * S-step) instead of floor(log2 amax_b) - 2, at most 125 so that no
 * reconstruction overflows fp32.  It differs exactly when amax_b's significand
 * exceeds 1.5.  Stored and decoded as MXFP4. */
#define FP4Q_FLAG_MX_CEIL_SCALE 0x2u

/* The stream type is CUDA's cudaStream_t (a CUstream_st*); NULL is the legacy default stream. */
typedef struct CUstream_st* fp4q_stream_t;

/* FP4Q_ABI_VERSION of the loaded library. */
FP4Q_API int fp4q_abi_version(void);

/* Static, NUL-terminated description of a status code. */
FP4Q_API const char* fp4q_status_string(fp4q_status_t status);

/* Bytes of device workspace fp4q_quantize and fp4q_error need for this shape
 * (per-CTA partial maxima and partial sums).  Independent of the data. */
FP4Q_API size_t fp4q_workspace_size(int64_t rows, int64_t cols, fp4q_format_t fmt, int rotate);

/* Quantize x (bf16 [rows][ldx]) into codes and scales.
 *  fmt, rotate    as above.
 *  flags          0 or FP4Q_FLAG_TENSOR_SCALE_GIVEN.
 *  codes, scales  outputs, layouts above.
 *  tensor_scale   NVFP4 formats: output (computed from the tensor absmax, of
 *                 the rotated values when rotate = 1), or input with the flag.
 *                 Ignored for MXFP4 (may be NULL).
 *  mse            nullable output; when NULL the error is not computed at all.
 *  workspace      device scratch of at least fp4q_workspace_size() bytes,
 *                 16-byte aligned; contents on entry are ignored.
 * Enqueues up to three kernels on `stream`: tensor absmax (NVFP4 formats
 * without the flag), the fused quantize pass, and the mse finaliser (when mse
 * is requested). */
FP4Q_API fp4q_status_t fp4q_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                            fp4q_format_t fmt, int rotate, uint32_t flags,
                            uint8_t* codes, uint8_t* scales, float* tensor_scale, double* mse,
                            void* workspace, size_t workspace_bytes, fp4q_stream_t stream);

/* Reconstruct y (bf16 [rows][ldy], round to nearest even from the fp32
 * reconstruction) from codes, scales and, for NVFP4 formats, *tensor_scale.
 * One kernel; no workspace. */
FP4Q_API fp4q_status_t fp4q_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                              int64_t rows, int64_t cols, fp4q_format_t fmt, int rotate,
                              void* y, int64_t ldy, fp4q_stream_t stream);

/* Mean squared error of the reconstruction of (codes, scales, tensor_scale)
 * against x (bf16 [rows][ldx]); *mse as in fp4q_quantize.  Two kernels. */
FP4Q_API fp4q_status_t fp4q_error(const void* x, int64_t ldx,
                         const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                         int64_t rows, int64_t cols, fp4q_format_t fmt, int rotate,
                         double* mse, void* workspace, size_t workspace_bytes, fp4q_stream_t stream);

/* The tensor scale alone: *tensor_scale = s_t of x (bf16 [rows][ldx]) for an
 * NVFP4 format, exactly the value fp4q_quantize computes and writes without
 * FP4Q_FLAG_TENSOR_SCALE_GIVEN (the absmax of the rotated values when
 * rotate = 1).
 *
 * Purpose: one tensor split by rows over several devices.  The map from the
 * absmax to s_t is monotone (a correctly rounded division by a positive
 * constant), so the largest s_t over the parts equals the s_t of the whole
 * tensor.  Each part calls this, the parts exchange the maximum, and each
 * part then calls fp4q_quantize with the flag; the codes and scales equal
 * those of the whole tensor quantized on one device.
 *  fmt            FP4Q_NVFP4, FP4Q_NVFP4_RAZER or FP4Q_NVFP4_RAZER_W; MXFP4
 *                 has no tensor scale (FP4Q_ERROR_INVALID_VALUE).
 *  tensor_scale   device output, 1 float, 4-byte aligned.  0 when rows or
 *                 cols is 0.
 *  workspace      as fp4q_quantize.
 * Validation as fp4q_quantize.  Enqueues two kernels: the absmax pass and a
 * one-CTA reduction of its per-CTA maxima. */
FP4Q_API fp4q_status_t fp4q_tensor_scale(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                         fp4q_format_t fmt, int rotate, float* tensor_scale,
                                         void* workspace, size_t workspace_bytes, fp4q_stream_t stream);

/* One tensor of a batch: as the arguments of fp4q_quantize (device pointers;
 * mse may be NULL, tensor_scale may be NULL for MXFP4). */
typedef struct fp4q_tensor_desc {
    const void* x;
    int64_t rows, cols, ldx;
    uint8_t* codes;
    uint8_t* scales;
    float* tensor_scale;
    double* mse;
} fp4q_tensor_desc_t;

/* Bytes of workspace fp4q_quantize_batch needs (independent of the tensors):
 * three rotating slots of per-CTA partial maxima and partial sums. */
FP4Q_API size_t fp4q_batch_workspace_size(int count, const fp4q_tensor_desc_t* tensors, fp4q_format_t fmt,
                                          int rotate);

/* Quantize `count` tensors, all in one format.  Results are those of calling
 * fp4q_quantize on each tensor in order with the same fmt, rotate and flags
 * (bit-identical codes, scales and tensor scales; each mse within fp64
 * summation order).  `tensors` is a HOST array read during the call.
 *
 * The call enqueues one persistent kernel per tensor (plus one), chained with
 * programmatic dependent launch: with the tensor scale computed, kernel j
 * runs the absmax pass of tensor j interleaved with the quantize pass of
 * tensor j-1 in the same SMs, so memory-bound and ALU-bound work overlap and
 * each kernel's start overlaps its predecessor's tail; kernel j also
 * finalises the MSE of tensor j-2.  The workspace (at least
 * fp4q_batch_workspace_size bytes, 16-byte aligned) needs no clearing; calls
 * sharing a workspace must not overlap on the device.  Errors as
 * fp4q_quantize; the first invalid tensor's status is returned before
 * anything is enqueued. */
FP4Q_API fp4q_status_t fp4q_quantize_batch(int count, const fp4q_tensor_desc_t* tensors, fp4q_format_t fmt,
                                           int rotate, uint32_t flags, void* workspace, size_t workspace_bytes,
                                           fp4q_stream_t stream);

/* Bits of the device error word (fp4q_device_errors). */
#define FP4Q_DEVICE_ERROR_PIPELINE_TIMEOUT 0x1u
#define FP4Q_DEVICE_ERROR_OUT_OF_BOUNDS 0x2u   /* only a library built with FP4Q_DEBUG sets it */

/* Read the device error word of the current CUDA context into *bits.  Every
 * kernel of the library records into one word per context.
 *  - Every wait of a kernel on its own copy pipeline gives up after 2 s.  A
 *    CTA that gives up sets FP4Q_DEVICE_ERROR_PIPELINE_TIMEOUT, waits (bounded)
 *    for its copies in flight and returns, so the outputs of that call are
 *    incomplete.
 *  - A library built with FP4Q_DEBUG checks every global-memory access its
 *    kernels make by hand (TMA copies are bounded by their tensor maps) against
 *    the extent its arguments give the buffer.  An access outside it is
 *    skipped and sets FP4Q_DEVICE_ERROR_OUT_OF_BOUNDS; the first one's site
 *    and offset are kept (fp4q_device_error_site).
 * This call is synchronous: it waits for the device, copies the word to the
 * host and, when clear != 0, resets the word and the kept site.  Returns
 * FP4Q_ERROR_INVALID_VALUE for a null bits, FP4Q_ERROR_CUDA if the copy fails. */
FP4Q_API fp4q_status_t fp4q_device_errors(uint32_t* bits, int clear);

/* The first out-of-bounds access a FP4Q_DEBUG library found since the word was
 * last cleared: *site names the access (a number fixed in the source, 0 when
 * there was none) and *offset is its byte offset into the buffer.  Synchronous,
 * like fp4q_device_errors; both pointers must be non-null. */
FP4Q_API fp4q_status_t fp4q_device_error_site(uint32_t* site, uint64_t* offset);

/* 1 when the loaded library was built with FP4Q_DEBUG, else 0. */
FP4Q_API int fp4q_debug_build(void);

/* Exercise the failure path above: one kernel arms a pipeline barrier that no
 * copy will complete and waits on it with the library's bounded wait.  After
 * 2 s the wait gives up and sets FP4Q_DEVICE_ERROR_PIPELINE_TIMEOUT; nothing
 * faults, traps or hangs, and the context stays usable.  Enqueues one kernel
 * on `stream`. */
FP4Q_API fp4q_status_t fp4q_selftest_timeout(fp4q_stream_t stream);

/* Bytes of device scratch held inside the library for fp4q_quantize_noalloc. */
#define FP4Q_NOALLOC_SCRATCH_BYTES 49152

/* fp4q_quantize for callers that cannot allocate device memory.
 *
 * No counterpart in the papers: this is a library convenience.  It exists for
 * code that must not call cudaMalloc (or any allocator) where it quantizes --
 * e.g. a plugin inside a program that owns all device memory, or a latency
 * path that cannot afford the synchronisation an allocation can imply -- and
 * so has no workspace to pass.  Arguments, outputs and results are those of
 * fp4q_quantize; the scratch comes from a static device array of
 * FP4Q_NOALLOC_SCRATCH_BYTES bytes that every GPU loading the library holds
 * until the process exits.  The call allocates nothing and frees nothing.
 *
 *  - The array's device address belongs to one CUDA context.  The first call
 *    in each context (the calling thread's current one; the device's primary
 *    context for a runtime-API program) looks it up with cudaGetSymbolAddress
 *    and caches it under that context's ID, so a call after cudaDeviceReset,
 *    or under a context the caller made current itself, gets that context's
 *    copy.  Make the first call in each context before any stream capture.
 *  - Every call on a device shares the one array, which keeps the previous
 *    call's contents.  Nothing in it needs clearing (each call writes every
 *    slot it reads), but calls that can overlap on the GPU -- on different
 *    streams without ordering between them -- race on it.  Order them on one
 *    stream or by events.
 *  - A shape whose scratch need (fp4q_workspace_size) exceeds the array is
 *    rejected with FP4Q_ERROR_WORKSPACE before anything is enqueued; with the
 *    present kernels every shape fits. */
FP4Q_API fp4q_status_t fp4q_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                             fp4q_format_t fmt, int rotate, uint32_t flags,
                                             uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                             double* mse, fp4q_stream_t stream);

/* ------------------------------------------------------------------------
 * Tensor-core operand form and the W4A4 product ("RaZeR", sect. 2.3: GEMMs on
 * existing tensor cores handle the remapped code in two passes).
 *
 * The operand form of a quantized NVFP4-family matrix (rows x cols, codes and
 * scales as fp4q_quantize writes them) is what the sm_100a block-scaled tensor
 * cores read:
 *  planes  uint8 [rows][P * cols/2], P = fp4q_mma_planes(fmt): P code planes
 *          per row, each cols/2 bytes in the codes layout.  NVFP4: the codes.
 *          RaZeR (both modes): plane 0 holds every code except 0b1000, which
 *          becomes the special value's base b -- the largest E2M1 magnitude
 *          below |s|, with the sign of s (+-4 for +-5, +-2 for +-2.5) -- and
 *          plane 1 holds s - b there (+-1, +-0.5) and +0 elsewhere, so the
 *          decoded planes add up to the reconstruction.
 *  sf      uint8 [fp4q_mma_sf_bytes(rows, cols)]: each block's scale
 *          magnitude as an E4M3 byte, bit 7 clear (weight mode: its E3M3 value,
 *          exact in E4M3), in 512-byte atoms of 128 rows x 4 blocks.  Atom
 *          (r / 128, kb / 4), row-major over ceil(rows/128) x ceil(cols/64)
 *          atoms, holds block kb of row r at byte
 *          (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4; padding is 0.
 * ------------------------------------------------------------------------ */

/* Code planes of a format's operand form: 1 (NVFP4), 2 (NVFP4_RAZER,
 * NVFP4_RAZER_W), 0 (MXFP4 or an invalid format: no operand form). */
FP4Q_API int fp4q_mma_planes(fp4q_format_t fmt);

/* Bytes of the scale atoms of a rows x cols operand (0 for negative sizes). */
FP4Q_API size_t fp4q_mma_sf_bytes(int64_t rows, int64_t cols);

/* Write the operand form of (codes, scales).  codes, scales, planes and sf are
 * device pointers, 16-byte aligned; cols a multiple of 16.  Enqueues one
 * kernel on `stream`.  FP4Q_ERROR_INVALID_VALUE for MXFP4, a bad format, a
 * null pointer or a negative size. */
FP4Q_API fp4q_status_t fp4q_mma_pack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                     fp4q_format_t fmt, uint8_t* planes, uint8_t* sf, fp4q_stream_t stream);

/* y = s_a * s_w * (A^ W^T) as bf16 (round to nearest even), A^ (M x K) and W^
 * (N x K) the reconstructions of two quantized matrices given in operand form:
 * a_planes / a_sf with a_np planes and tensor scale *a_scale, w_planes / w_sf
 * with w_np planes and *w_scale (device fp32 scalars).  The tensor cores
 * (tcgen05.mma kind::mxf4nvf4, 16-element E4M3 scales, fp32 accumulation)
 * run the a_np * w_np plane products as one accumulation of a_np * w_np * K
 * elements.  y is row-major [M][ldy] bf16.  Shapes: K > 0 a multiple of 256,
 * N a multiple of 8, ldy >= N a multiple of 8, a_np and w_np in {1, 2};
 * M, N, a_np * K / 2 and w_np * K / 2 below 2^31.  Pointers 16-byte aligned
 * (the scales 4).  M = 0 or N = 0 enqueues nothing.  The result equals the
 * exact product up to fp32 accumulation and the final bf16 rounding. */
FP4Q_API fp4q_status_t fp4q_gemm(const uint8_t* a_planes, const uint8_t* a_sf, int a_np, const float* a_scale,
                                 const uint8_t* w_planes, const uint8_t* w_sf, int w_np, const float* w_scale,
                                 int64_t M, int64_t N, int64_t K, void* y, int64_t ldy, fp4q_stream_t stream);

/* ------------------------------------------------------------------------
 * Sparse outlier separation ("XFP: quality-targeted adaptive codebook
 * quantization", sect. 2): per row r of a bf16 matrix, mu = mean and sigma =
 * population standard deviation (fp64); outliers are the elements with
 * |x - mu| > k sigma, at most cap = floor(max_frac * cols) of them (when more
 * qualify, the cap largest deviations, ties to the lower column).  They are
 * stored in column order as (column uint16, fp16 value -- nearest even,
 * saturating at 65504) in slots [r][0, count[r]) of [rows][cap] arrays, and
 * the bulk matrix is x with mu (rounded to bf16) at their positions, ready for
 * fp4q_quantize.  A reconstruction is fp4q_dequantize of the bulk's codes
 * followed by fp4q_scatter_outliers.  mu and sigma are reduced in a fixed
 * order on the GPU; an element whose deviation lies within a few fp64 ulps of
 * the threshold may be classified differently from a sequential sum.
 * ------------------------------------------------------------------------ */

/* floor(max_frac * cols), the outlier slots per row (0 for invalid arguments). */
FP4Q_API int64_t fp4q_outlier_capacity(int64_t cols, double max_frac);

/* x, bulk: bf16 [rows][ld], ld >= cols and a multiple of 8, 16-byte aligned;
 * cols a multiple of 8, at most 65536; k > 0 finite; 0 <= max_frac <= 1.
 * out_cols, out_vals: [rows][cap] uint16 (may be null when cap = 0); out_count:
 * [rows] int32.  One kernel on `stream`. */
FP4Q_API fp4q_status_t fp4q_separate_outliers(const void* x, int64_t rows, int64_t cols, int64_t ldx, double k,
                                              double max_frac, void* bulk, int64_t ldb, uint16_t* out_cols,
                                              uint16_t* out_vals, int32_t* out_count, fp4q_stream_t stream);

/* y[r][out_cols[r][s]] = bf16(out_vals[r][s]) for s < min(out_count[r], cap):
 * puts the outliers back into a bf16 reconstruction y [rows][ldy].  The arrays
 * are those fp4q_separate_outliers wrote (columns below cols); a slot whose
 * column is at or past cols is skipped, so no write lands in y's padding
 * columns [cols, ldy) or past element (rows-1)*ldy + cols - 1. */
FP4Q_API fp4q_status_t fp4q_scatter_outliers(const uint16_t* out_cols, const uint16_t* out_vals,
                                             const int32_t* out_count, int64_t rows, int64_t cols, int64_t cap,
                                             void* y, int64_t ldy, fp4q_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP4Q_H */
