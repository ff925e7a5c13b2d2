/*
 * fp4q oracle -- plain, slow, scalar CPU implementation of block-scaled 4-bit
 * quantize / dequantize / error (NVFP4, NVFP4 with RaZeR redundant-zero
 * remapping, MXFP4, each optionally after a 32-point Walsh-Hadamard rotation).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline and reference arm use it.  It shares no code, header, table or constant with the
 * CUDA library: every number below is restated here from the cited papers' text.
 *
 * Sources (title, section):
 *  [RaZeR]  "RaZeR: Pushing the Limits of NVFP4 Quantization with Redundant
 *           Zero Remapping", technical summary sect. 1 (E2M1 value set, E4M3
 *           block scale with an unused sign bit) and sect. 2.2 (the redundant
 *           -0 code remapped to a special value, chosen per block by minimum
 *           squared error; one free bit for activations = one pair; +-5).
 *  [TORQ]   "TORQ: Two-Level Orthogonal Rotation for MXFP4 Quantization",
 *           technical summary sect. 1 (32-element blocks sharing one exponent
 *           scale, e2m1 codebook) and sect. 2 (orthogonal intra-block rotation,
 *           "S-step" scale from the block maximum, rotations absorbed into the
 *           neighbouring weights).
 *
 * Readings where the papers are silent (each one restated where it is used):
 *  R1 element rounding: nearest E2M1 value, ties to the even code, |v| > 6
 *     saturates to 6, a zero result is always +0 (code 0b0000).
 *  R2 NVFP4 is two-level: a per-tensor fp32 scale s_t = RN(A / (6*448)) with A
 *     the tensor absmax, then per 16-block an E4M3 scale (round to nearest
 *     even, saturating at 448).  Elements are encoded as RN(y * r) with
 *     r = RN(1 / RN(dec(sb) * s_t)); where that reciprocal overflows to
 *     infinity (den below about 2^-128, which only a tensor whose absmax is
 *     below about 2^-107 can reach) they are encoded as RN(y / den) instead,
 *     so every element still goes to its nearest code and a zero stays +0.
 *  R3 MXFP4 scale: e = floor(log2(block absmax)) - 2, clamped to [-127, 127],
 *     stored as the E8M0 byte e + 127.
 *  R4 RaZeR (activation mode): the pair {+5, -5}; the scale sign bit selects
 *     -5; choose -5 only if it lowers the block's squared error strictly more
 *     than +5 does; the regular code wins ties between an element's regular
 *     value and the special value.
 *  R5 rotation: y = RN_f32(RN_f32(H32 x) * RN_f32(1/sqrt(32))) with H32 the
 *     Sylvester-ordered +-1 Hadamard matrix; the sum is taken in double.
 *  R6 layout: codes row-major, element 2k in the low nibble of byte k; scales
 *     dense row-major [rows][cols / block].
 *  R7 RaZeR weight mode [RaZeR sect. 2.1, 2.2: weights take a 6-bit E3M3 block
 *     scale, and the two freed bits choose among four special values, two
 *     pairs fixed offline, all multiples of 0.5]: E3M3 is unsigned, exponent
 *     bias 3, exponent field 0 subnormal (m * 2^-5), no NaN, largest value 30;
 *     the scale byte holds the E3M3 value in bits 0..5 and the selector in bits
 *     6..7 (0: +5, 1: -5, 2: +s2, 3: -s2); the first level is
 *     s_t = RN(A / (6 * 30)); per block the special value with the largest
 *     squared-error gain wins, ties going to the lower selector; s2 is the
 *     second pair found by the offline search in oracle/razer_weight_pair.py.
 *  R8 tensor-core operand form [RaZeR sect. 2.3: GEMMs on existing tensor
 *     cores handle the remapped code with two passes]: a quantized matrix
 *     becomes one code plane (NVFP4) or two (RaZeR, either mode) whose decoded
 *     sum is the reconstruction.  Plane 0 keeps every code except 0b1000, which
 *     becomes the special value's base b, the largest E2M1 magnitude below
 *     |s|, with the sign of s; plane 1 is +0 except at those elements, where it
 *     holds s - b (+-1 for +-5, +-0.5 for +-2.5).  Both planes use the block's
 *     scale magnitude as an E4M3 byte with bit 7 clear (weight mode: the E3M3
 *     value, which every E3M3 code has exactly in E4M3).  Plane p of row r
 *     occupies bytes [p * cols/2, (p+1) * cols/2) of the row.  The scale
 *     bytes are stored in 512-byte atoms, one per 128 rows x 4 blocks: rows
 *     padded to a multiple of 128 and blocks to a multiple of 4 with zeros,
 *     atom (r / 128, kb / 4) in row-major order, and inside it the byte
 *     (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4.
 *  R9 W4A4 product: Y = A^ W^T for A^ (M x K) and W^ (N x K) the fp32
 *     reconstructions of two quantized matrices, summed in binary64.
 *  R11 sparse outlier separation ["XFP: quality-targeted adaptive codebook
 *     quantization", technical summary sect. 2, sparse outlier separation:
 *     weights with |w - mu| > k sigma (k = 4 by default, at most 2 % of the
 *     weights) are kept apart in fp16 at their positions, and the bulk holds
 *     the group mean there before it is quantized]: the group is a row;
 *     mu = (sum of the row, in order) / n and sigma = sqrt(sum (x - mu)^2 / n)
 *     in binary64; with d = |x - mu| the candidates are d > k sigma; when more
 *     than cap = floor(max_frac * n) qualify, the cap largest d are kept, ties
 *     to the lower column; kept values are stored as fp16 (nearest even,
 *     saturating at 65504) in column order, and the bulk row is x with every
 *     kept position set to RN_bf16(mu).
 *  R10 MXFP4 exponent without clipping [TORQ sect. 2, S-step: the block
 *     scale maps the block maximum onto the largest code]: e is the smallest
 *     integer with a <= 6 * 2^e, clamped to [-127, 125] so that every
 *     reconstruction (at most 6 * 2^e) stays finite in binary32; below the
 *     clamp nothing saturates.
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -shared -fPIC
 * -pthread.  Floating point is IEEE binary32/binary64 with round-to-nearest
 * and no flush-to-zero, as on any x86-64 / aarch64 host without fast-math.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_NVFP4 0
#define ORC_NVFP4_RAZER 1
#define ORC_MXFP4 2
#define ORC_NVFP4_RAZER_W 3
#define ORC_MXFP4_CEIL 4      /* MXFP4 with the R10 exponent; stored and decoded as MXFP4 */
#define IS_MX(f) ((f) == ORC_MXFP4 || (f) == ORC_MXFP4_CEIL)

/* The second special-value pair of the RaZeR weight mode (R7): the winner of
 * the offline search over multiples of 0.5 (oracle/razer_weight_pair.py).
 * The search itself changes it through orc_set_razer_w_pair. */
static double razer_w_pair = 2.5;
void orc_set_razer_w_pair(double s2) { razer_w_pair = s2; }
double orc_razer_w_pair(void) { return razer_w_pair; }

/* ------------------------------------------------------------------------ */
/* bf16 and fp32 bit helpers                                                 */
/* ------------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the upper half of a binary32; widening is exact. */
float orc_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* binary32 -> bf16, round to nearest, ties to even (inputs are finite). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u = bits_from_f32(f);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------------ */
/* E2M1 element format  [RaZeR sect. 1: {+-0,+-0.5,+-1,+-1.5,+-2,+-3,+-4,+-6}] */
/* code bit 3 = sign, bits 0..2 = index into the magnitude list below.       */
/* ------------------------------------------------------------------------ */

static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(int code)
{
    double m = E2M1_MAGNITUDE[code & 7];
    return (code & 8) ? -m : m;
}

/* R1: nearest magnitude, ties to the even index, saturating at 6.  The
 * thresholds are the midpoints of neighbouring magnitudes; at a midpoint the
 * comparison sends the value to whichever neighbour has the even index
 * (0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4). */
int orc_e2m1_encode(float v)
{
    double a = fabs((double)v);
    int m;
    if (isnan(v)) return -1;           /* no E2M1 code is nearest to NaN */
    if (a <= 0.25) m = 0;
    else if (a < 0.75) m = 1;
    else if (a <= 1.25) m = 2;
    else if (a < 1.75) m = 3;
    else if (a <= 2.5) m = 4;
    else if (a < 3.5) m = 5;
    else if (a <= 5.0) m = 6;
    else m = 7;
    if (m == 0) return 0;              /* zero is always +0 */
    return (v < 0.0f) ? (8 | m) : m;
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 block scale  [RaZeR sect. 1: the block scale is an FP8-E4M3       */
/* value; it is always positive, so its sign bit is free]                    */
/* bias 7; exponent field 0 = subnormal (m * 2^-9); 0x7F / 0xFF are NaN.     */
/* ------------------------------------------------------------------------ */

double orc_e4m3_value(int byte)
{
    int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* R2: round a non-negative fp32 to E4M3, nearest, ties to even mantissa,
 * saturating at 448 (byte 0x7E); never produces NaN.  Direct arithmetic:
 * split t = f * 2^k with f in [1, 2), round (f - 1) * 8 to an integer. */
int orc_e4m3_encode(float t)
{
    double x = (double)t;
    if (!(x > 0.0)) return 0;
    if (x >= 448.0) return 0x7E;
    int k;
    double f = frexp(x, &k);       /* x = f * 2^k, f in [0.5, 1) */
    k -= 1;                        /* x = (2f) * 2^k, 2f in [1, 2) */
    if (k < -6) {                  /* subnormal range: quantum 2^-9 */
        double q = x / ldexp(1.0, -9);
        double r = floor(q);
        double frac = q - r;
        if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
        /* r == 8 is the smallest normal, exponent field 1, mantissa 0 */
        return (int)r;             /* r in [0, 8]; 8 encodes as 0x08 */
    }
    double q = (2.0 * f - 1.0) * 8.0;  /* mantissa in units of 1/8 */
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    int mant = (int)r, ex = k + 7;
    if (mant == 8) { mant = 0; ex += 1; }
    if (ex > 15 || (ex == 15 && mant > 6)) return 0x7E;
    return (ex << 3) | mant;
}

/* ------------------------------------------------------------------------ */
/* E3M3 block scale of the RaZeR weight mode (R7)                             */
/* ------------------------------------------------------------------------ */

double orc_e3m3_value(int byte6)
{
    int e = (byte6 >> 3) & 7, m = byte6 & 7;
    if (e == 0) return ldexp((double)m, -5);
    return ldexp(1.0 + m / 8.0, e - 3);
}

/* Round a non-negative fp32 to E3M3: nearest, ties to even mantissa,
 * saturating at 30 (0x3F).  As orc_e4m3_encode with bias 3. */
int orc_e3m3_encode(float t)
{
    double x = (double)t;
    if (!(x > 0.0)) return 0;
    if (x >= 30.0) return 0x3F;
    int k;
    double f = frexp(x, &k);       /* x = f * 2^k, f in [0.5, 1) */
    k -= 1;                        /* x = (2f) * 2^k, 2f in [1, 2) */
    if (k < -2) {                  /* subnormal range: quantum 2^-5 */
        double q = x / ldexp(1.0, -5);
        double r = floor(q);
        double frac = q - r;
        if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
        return (int)r;             /* r in [0, 8]; 8 encodes the smallest normal */
    }
    double q = (2.0 * f - 1.0) * 8.0;
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    int mant = (int)r, ex = k + 3;
    if (mant == 8) { mant = 0; ex += 1; }
    if (ex > 7) return 0x3F;
    return (ex << 3) | mant;
}

/* ------------------------------------------------------------------------ */
/* E8M0 shared exponent  [TORQ sect. 1: MXFP4 = 32-element blocks sharing an   */
/* exponent scale].  byte b stands for 2^(b - 127); 0xFF is NaN.             */
/* ------------------------------------------------------------------------ */

double orc_e8m0_value(int byte)
{
    if ((byte & 255) == 255) return NAN;
    return ldexp(1.0, (byte & 255) - 127);
}

/* R3: e = floor(log2 a) - 2 for a > 0 (2 = exponent of the largest E2M1
 * magnitude, 6 = 1.5 * 2^2), clamped to [-127, 127].  frexp is exact. */
int orc_mx_exponent(float a)
{
    int k;
    (void)frexp((double)a, &k);    /* a = f * 2^k, f in [0.5, 1) => floor(log2 a) = k - 1 */
    int e = (k - 1) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* R10: the smallest e with a <= 6 * 2^e (a > 0), by search upward from an
 * exponent known to be too small; 6 * 2^e is exact in binary64. */
int orc_mx_exponent_ceil(float a)
{
    int k;
    (void)frexp((double)a, &k);    /* a < 2^k */
    int e = k - 4;                 /* 6 * 2^(k-4) < 2^k / 2: too small */
    while ((double)a > 6.0 * ldexp(1.0, e)) ++e;
    if (e < -127) e = -127;
    if (e > 125) e = 125;
    return e;
}

/* ------------------------------------------------------------------------ */
/* 32-point Walsh-Hadamard rotation  [TORQ sect. 2: an orthogonal rotation     */
/* inside each block; R5 fixes it to the Sylvester Hadamard matrix / sqrt 32]  */
/* ------------------------------------------------------------------------ */

static int popcount5(int v) { int c = 0; for (int b = 0; b < 5; ++b) c += (v >> b) & 1; return c; }

/* entry (i, j) of the Sylvester-ordered 32x32 Hadamard matrix */
int orc_hadamard_entry(int i, int j) { return (popcount5(i & j) & 1) ? -1 : 1; }

float orc_wht_constant(void) { return (float)(1.0 / sqrt(32.0)); }

/* out_i = RN_f32( RN_f32( sum_j H_ij in_j ) * c ), the sum in double.
 * H / sqrt(32) is symmetric and orthogonal, so the same call inverts it. */
void orc_wht32(const float* in, float* out)
{
    const float c = orc_wht_constant();
    float tmp[32];
    for (int i = 0; i < 32; ++i) {
        double s = 0.0;
        for (int j = 0; j < 32; ++j)
            s += orc_hadamard_entry(i, j) * (double)in[j];
        tmp[i] = (float)s;
    }
    for (int i = 0; i < 32; ++i) out[i] = tmp[i] * c;
}

/* ------------------------------------------------------------------------ */
/* Row helpers                                                                */
/* ------------------------------------------------------------------------ */

/* Load one row as fp32, rotated in 32-groups when asked. */
static void load_row(const uint16_t* x, int64_t cols, int rotate, float* y)
{
    for (int64_t j = 0; j < cols; ++j) y[j] = orc_bf16_to_f32(x[j]);
    if (rotate)
        for (int64_t g = 0; g < cols; g += 32) {
            float t[32];
            orc_wht32(y + g, t);
            memcpy(y + g, t, sizeof t);
        }
}

static int block_size(int fmt) { return IS_MX(fmt) ? 32 : 16; }

/* ------------------------------------------------------------------------ */
/* Tensor absmax (NVFP4 first level, R2)                                      */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t* x; int64_t r0, r1, cols, ldx; int rotate; float amax;
} amax_job;

static void* amax_worker(void* p)
{
    amax_job* j = (amax_job*)p;
    float* y = (float*)malloc(sizeof(float) * (size_t)j->cols);
    float m = 0.0f;
    for (int64_t r = j->r0; r < j->r1; ++r) {
        load_row(j->x + r * j->ldx, j->cols, j->rotate, y);
        for (int64_t c = 0; c < j->cols; ++c) {
            float a = fabsf(y[c]);
            if (a > m) m = a;
        }
    }
    free(y);
    j->amax = m;
    return NULL;
}

float orc_tensor_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx,
                      int rotate, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > rows) nthreads = (int)rows;
    amax_job* jobs = (amax_job*)calloc((size_t)nthreads, sizeof(amax_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = (amax_job){x, rows * t / nthreads, rows * (t + 1) / nthreads, cols, ldx, rotate, 0.0f};
        pthread_create(&th[t], NULL, amax_worker, &jobs[t]);
    }
    float m = 0.0f;
    for (int t = 0; t < nthreads; ++t) {
        pthread_join(th[t], NULL);
        if (jobs[t].amax > m) m = jobs[t].amax;
    }
    free(jobs); free(th);
    return m;
}

/* R2: s_t maps the tensor maximum onto the largest E2M1 value (6) times the
 * largest E4M3 value (448). */
float orc_tensor_scale_from_amax(float amax) { return amax / 2688.0f; }

/* R7: the weight mode maps it onto 6 times the largest E3M3 value (30). */
float orc_tensor_scale_from_amax_w(float amax) { return amax / 180.0f; }

static float tensor_scale_for(int fmt, float amax)
{
    return fmt == ORC_NVFP4_RAZER_W ? orc_tensor_scale_from_amax_w(amax) : orc_tensor_scale_from_amax(amax);
}

/* ------------------------------------------------------------------------ */
/* Block decode: the fp32 reconstruction of one element                      */
/* ------------------------------------------------------------------------ */

/* NVFP4 / RaZeR: den = RN(dec(sb) * s_t); x^ = RN(value(code) * den).  Under
 * RaZeR the magnitude of the scale is the low 7 bits and code 0b1000 stands
 * for +5 (scale bit 7 clear) or -5 (bit 7 set)  [RaZeR sect. 2.2]. */
static float nv_den(int fmt, int sbyte, float s_t)
{
    double sv = fmt == ORC_NVFP4_RAZER_W ? orc_e3m3_value(sbyte & 0x3F)
                                         : orc_e4m3_value(fmt == ORC_NVFP4_RAZER ? (sbyte & 0x7F) : sbyte);
    return (float)sv * s_t;
}

/* The special value code 0b1000 stands for in a block with scale byte sbyte. */
static double special_value(int fmt, int sbyte)
{
    if (fmt == ORC_NVFP4_RAZER) return (sbyte & 0x80) ? -5.0 : 5.0;
    switch ((sbyte >> 6) & 3) {
        case 0: return 5.0;
        case 1: return -5.0;
        case 2: return razer_w_pair;
        default: return -razer_w_pair;
    }
}

static float nv_decode(int fmt, int code, int sbyte, float den)
{
    double q;
    if ((fmt == ORC_NVFP4_RAZER || fmt == ORC_NVFP4_RAZER_W) && code == 8) q = special_value(fmt, sbyte);
    else q = orc_e2m1_value(code);
    return (float)q * den;
}

static float mx_decode(int code, int sbyte)
{
    return (float)(orc_e2m1_value(code) * orc_e8m0_value(sbyte));
}

/* ------------------------------------------------------------------------ */
/* Quantize one row                                                           */
/* ------------------------------------------------------------------------ */

static void set_code(uint8_t* row_codes, int64_t j, int code)
{
    uint8_t* b = row_codes + (j >> 1);
    if (j & 1) *b = (uint8_t)((*b & 0x0F) | (code << 4));
    else       *b = (uint8_t)((*b & 0xF0) | code);
}

static int get_code(const uint8_t* row_codes, int64_t j)
{
    uint8_t b = row_codes[j >> 1];
    return (j & 1) ? (b >> 4) : (b & 0x0F);
}

/* RaZeR selection for one 16-block given the scaled values v[], the regular
 * codes q[] and the candidate special values sv[0..ns) (R4, R7).  Squared
 * errors are formed in double; every difference involved is exact in binary32
 * and every square and sum of the candidates is exact in binary64, so the
 * comparison is exact.  Returns the index of the candidate with the largest
 * total gain (ties: the lower index) and rewrites its winning elements, those
 * strictly closer to it than to their regular value, to 0b1000. */
static int razer_select(const float* v, int* q, int n, const double* sv, int ns)
{
    double best = 0.0;
    int pick = 0;
    for (int s = 0; s < ns; ++s) {
        double gain = 0.0;
        for (int i = 0; i < n; ++i) {
            double e_reg = (double)v[i] - orc_e2m1_value(q[i]);
            double e_sp = (double)v[i] - sv[s];
            if (fabs(e_sp) < fabs(e_reg))           /* strictly closer: remap */
                gain += e_reg * e_reg - e_sp * e_sp;
        }
        if (s == 0 || gain > best) { best = gain; pick = s; }
    }
    for (int i = 0; i < n; ++i) {
        double e_reg = (double)v[i] - orc_e2m1_value(q[i]);
        double e_sp = (double)v[i] - sv[pick];
        if (fabs(e_sp) < fabs(e_reg)) q[i] = 8;
    }
    return pick;
}

/* Quantize the row y[0..cols) (already rotated when asked).  Writes codes and
 * scales for the row; s_t is used for NVFP4 formats.  Returns 0, or -1 when an
 * element reached the E2M1 encoder as NaN (outside the finite-input contract). */
static int quantize_row(const float* y, int64_t cols, int fmt, float s_t,
                        uint8_t* row_codes, uint8_t* row_scales)
{
    int bad = 0;
    const int B = block_size(fmt);
    for (int64_t b0 = 0; b0 < cols; b0 += B) {
        float a = 0.0f;
        for (int i = 0; i < B; ++i) { float t = fabsf(y[b0 + i]); if (t > a) a = t; }
        float v[32];
        int q[32];
        int sbyte;
        if (IS_MX(fmt)) {
            /* TORQ sect. 1 / R3 */
            if (a == 0.0f) {
                sbyte = 0;
                for (int i = 0; i < B; ++i) q[i] = 0;
            } else {
                int e = fmt == ORC_MXFP4_CEIL ? orc_mx_exponent_ceil(a) : orc_mx_exponent(a);
                sbyte = e + 127;
                float r = (float)ldexp(1.0, -e);    /* exact power of two */
                for (int i = 0; i < B; ++i) { v[i] = y[b0 + i] * r; q[i] = orc_e2m1_encode(v[i]); }
            }
        } else {
            /* RaZeR sect. 1 / R2: block scale from the block absmax (R7: E3M3
             * for the weight mode) */
            float six_st = 6.0f * s_t;
            float t = (six_st > 0.0f) ? a / six_st : 0.0f;
            const int wmode = fmt == ORC_NVFP4_RAZER_W;
            sbyte = wmode ? orc_e3m3_encode(t) : orc_e4m3_encode(t);
            float den = (float)(wmode ? orc_e3m3_value(sbyte) : orc_e4m3_value(sbyte)) * s_t;
            if (sbyte == 0 || den == 0.0f) {
                /* a zero (or underflowed) scale decodes every element to 0 */
                for (int i = 0; i < B; ++i) q[i] = 0;
            } else {
                /* R2: scale by the reciprocal; by division where it overflows */
                float r = 1.0f / den;
                for (int i = 0; i < B; ++i) {
                    v[i] = isinf(r) ? y[b0 + i] / den : y[b0 + i] * r;
                    q[i] = orc_e2m1_encode(v[i]);
                }
                if (fmt == ORC_NVFP4_RAZER) {
                    const double pair[2] = {5.0, -5.0};
                    sbyte |= razer_select(v, q, B, pair, 2) << 7;
                } else if (wmode) {
                    const double four[4] = {5.0, -5.0, razer_w_pair, -razer_w_pair};
                    sbyte |= razer_select(v, q, B, four, 4) << 6;
                }
            }
        }
        for (int i = 0; i < B; ++i)
            if (q[i] < 0) { bad = 1; q[i] = 0; }
        row_scales[b0 / B] = (uint8_t)sbyte;
        for (int i = 0; i < B; ++i) set_code(row_codes, b0 + i, q[i]);
    }
    return bad ? -1 : 0;
}

/* Reconstruct the row in the original domain (inverse rotation when asked). */
static void dequant_row(const uint8_t* row_codes, const uint8_t* row_scales, int64_t cols,
                        int fmt, int rotate, float s_t, float* out)
{
    const int B = block_size(fmt);
    for (int64_t b0 = 0; b0 < cols; b0 += B) {
        int sbyte = row_scales[b0 / B];
        float den = IS_MX(fmt) ? 0.0f : nv_den(fmt, sbyte, s_t);
        for (int i = 0; i < B; ++i) {
            int code = get_code(row_codes, b0 + i);
            out[b0 + i] = IS_MX(fmt) ? mx_decode(code, sbyte)
                                             : nv_decode(fmt, code, sbyte, den);
        }
    }
    if (rotate)
        for (int64_t g = 0; g < cols; g += 32) {
            float t[32];
            orc_wht32(out + g, t);
            memcpy(out + g, t, sizeof t);
        }
}

static double row_sse(const uint16_t* x, const float* xhat, int64_t cols)
{
    double s = 0.0;
    for (int64_t j = 0; j < cols; ++j) {
        double d = (double)orc_bf16_to_f32(x[j]) - (double)xhat[j];
        s += d * d;
    }
    return s;
}

/* ------------------------------------------------------------------------ */
/* Whole-tensor entry points (rows split over pthreads; SSE summed in order) */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t* x; int64_t r0, r1, cols, ldx; int fmt, rotate; float s_t;
    uint8_t* codes; uint8_t* scales; const uint8_t* ccodes; const uint8_t* cscales;
    float* y_f32; uint16_t* y_bf16; int64_t ldy; int want_sse; double sse;
    int bad;   /* set when an element reached the E2M1 encoder as NaN */
} row_job;

static void* quant_worker(void* p)
{
    row_job* j = (row_job*)p;
    const int B = block_size(j->fmt);
    float* y = (float*)malloc(sizeof(float) * (size_t)j->cols);
    float* xh = (float*)malloc(sizeof(float) * (size_t)j->cols);
    double sse = 0.0;
    for (int64_t r = j->r0; r < j->r1; ++r) {
        uint8_t* rc = j->codes + r * (j->cols / 2);
        uint8_t* rs = j->scales + r * (j->cols / B);
        load_row(j->x + r * j->ldx, j->cols, j->rotate, y);
        if (quantize_row(y, j->cols, j->fmt, j->s_t, rc, rs) != 0) j->bad = 1;
        if (j->want_sse) {
            dequant_row(rc, rs, j->cols, j->fmt, j->rotate, j->s_t, xh);
            sse += row_sse(j->x + r * j->ldx, xh, j->cols);
        }
    }
    free(y); free(xh);
    j->sse = sse;
    return NULL;
}

static double run_rows(void* (*fn)(void*), row_job proto, int64_t rows, int nthreads, int* bad)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > rows) nthreads = (int)rows;
    row_job* jobs = (row_job*)calloc((size_t)nthreads, sizeof(row_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = proto;
        jobs[t].r0 = rows * t / nthreads;
        jobs[t].r1 = rows * (t + 1) / nthreads;
        pthread_create(&th[t], NULL, fn, &jobs[t]);
    }
    double sse = 0.0;
    for (int t = 0; t < nthreads; ++t) {
        pthread_join(th[t], NULL);
        sse += jobs[t].sse;
        if (bad && jobs[t].bad) *bad = 1;
    }
    free(jobs); free(th);
    return sse;
}

/* Quantize a rows x cols bf16 matrix (row stride ldx elements).
 *  scale_given != 0: *tensor_scale is read (NVFP4 formats), else computed
 *  and written.  sse (nullable) receives the sum of squared errors against
 *  the fp32 reconstruction in the original domain.  Returns 0, -1 on a
 *  shape the formats do not allow, or -2 when an element reached the E2M1
 *  encoder as NaN (non-finite input, outside the contract). */
int orc_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx,
                 int fmt, int rotate, int scale_given, float* tensor_scale,
                 uint8_t* codes, uint8_t* scales, double* sse, int nthreads)
{
    const int B = block_size(fmt);
    if (rows < 0 || cols % B || (rotate && cols % 32) || ldx < cols) return -1;
    float s_t = 0.0f;
    if (!IS_MX(fmt)) {
        if (scale_given) s_t = *tensor_scale;
        else {
            s_t = tensor_scale_for(fmt, orc_tensor_amax(x, rows, cols, ldx, rotate, nthreads));
            *tensor_scale = s_t;
        }
    }
    if (rows == 0 || cols == 0) { if (sse) *sse = 0.0; return 0; }
    row_job proto = {0};
    proto.x = x; proto.cols = cols; proto.ldx = ldx; proto.fmt = fmt; proto.rotate = rotate;
    proto.s_t = s_t; proto.codes = codes; proto.scales = scales; proto.want_sse = sse != NULL;
    int bad = 0;
    double s = run_rows(quant_worker, proto, rows, nthreads, &bad);
    if (sse) *sse = s;
    return bad ? -2 : 0;
}

static void* dequant_worker(void* p)
{
    row_job* j = (row_job*)p;
    const int B = block_size(j->fmt);
    float* xh = (float*)malloc(sizeof(float) * (size_t)j->cols);
    for (int64_t r = j->r0; r < j->r1; ++r) {
        dequant_row(j->ccodes + r * (j->cols / 2), j->cscales + r * (j->cols / B), j->cols,
                    j->fmt, j->rotate, j->s_t, xh);
        for (int64_t c = 0; c < j->cols; ++c) {
            if (j->y_f32) j->y_f32[r * j->ldy + c] = xh[c];
            if (j->y_bf16) j->y_bf16[r * j->ldy + c] = orc_f32_to_bf16(xh[c]);
        }
    }
    free(xh);
    j->sse = 0.0;
    return NULL;
}

/* Dequantize to fp32 (y_f32, nullable) and/or bf16 (y_bf16, nullable), both
 * with row stride ldy. */
int orc_dequantize(const uint8_t* codes, const uint8_t* scales, float tensor_scale,
                   int64_t rows, int64_t cols, int fmt, int rotate,
                   float* y_f32, uint16_t* y_bf16, int64_t ldy, int nthreads)
{
    const int B = block_size(fmt);
    if (rows < 0 || cols % B || (rotate && cols % 32) || ldy < cols) return -1;
    if (rows == 0 || cols == 0) return 0;
    row_job proto = {0};
    proto.cols = cols; proto.fmt = fmt; proto.rotate = rotate; proto.s_t = tensor_scale;
    proto.ccodes = codes; proto.cscales = scales; proto.y_f32 = y_f32; proto.y_bf16 = y_bf16;
    proto.ldy = ldy;
    run_rows(dequant_worker, proto, rows, nthreads, NULL);
    return 0;
}

static void* error_worker(void* p)
{
    row_job* j = (row_job*)p;
    const int B = block_size(j->fmt);
    float* xh = (float*)malloc(sizeof(float) * (size_t)j->cols);
    double sse = 0.0;
    for (int64_t r = j->r0; r < j->r1; ++r) {
        dequant_row(j->ccodes + r * (j->cols / 2), j->cscales + r * (j->cols / B), j->cols,
                    j->fmt, j->rotate, j->s_t, xh);
        sse += row_sse(j->x + r * j->ldx, xh, j->cols);
    }
    free(xh);
    j->sse = sse;
    return NULL;
}

/* Sum of squared errors between x and the reconstruction of (codes, scales). */
int orc_error(const uint16_t* x, int64_t ldx, const uint8_t* codes, const uint8_t* scales,
              float tensor_scale, int64_t rows, int64_t cols, int fmt, int rotate,
              double* sse, int nthreads)
{
    const int B = block_size(fmt);
    if (rows < 0 || cols % B || (rotate && cols % 32) || ldx < cols) return -1;
    if (rows == 0 || cols == 0) { *sse = 0.0; return 0; }
    row_job proto = {0};
    proto.x = x; proto.ldx = ldx; proto.cols = cols; proto.fmt = fmt; proto.rotate = rotate;
    proto.s_t = tensor_scale; proto.ccodes = codes; proto.cscales = scales;
    *sse = run_rows(error_worker, proto, rows, nthreads, NULL);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Tensor-core operand form (R8) and the W4A4 product (R9)                   */
/* ------------------------------------------------------------------------ */

int orc_mma_planes(int fmt) { return (fmt == ORC_NVFP4_RAZER || fmt == ORC_NVFP4_RAZER_W) ? 2 : 1; }

int64_t orc_mma_sf_bytes(int64_t rows, int64_t cols)
{
    return ((rows + 127) / 128) * ((cols / 16 + 3) / 4) * 512;
}

int64_t orc_mma_sf_offset(int64_t r, int64_t kb, int64_t cols)
{
    const int64_t atoms_per_row_block = (cols / 16 + 3) / 4;
    return ((r / 128) * atoms_per_row_block + kb / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4;
}

/* The block's scale magnitude as an E4M3 byte (bit 7 clear). */
int orc_mma_scale_byte(int fmt, int sbyte)
{
    if (fmt == ORC_NVFP4_RAZER_W) return orc_e4m3_encode((float)orc_e3m3_value(sbyte & 0x3F));
    if (fmt == ORC_NVFP4_RAZER) return sbyte & 0x7F;
    return sbyte;
}

/* Base of a special value s: the largest E2M1 magnitude below |s|, signed as s. */
static double special_base(double s)
{
    double b = 0.0;
    for (int c = 0; c < 8; ++c) {
        const double m = orc_e2m1_value(c);
        if (m < fabs(s) && m > b) b = m;
    }
    return s < 0.0 ? -b : b;
}

/* Codes (dense, rows x cols/2) and scales (rows x cols/16) of an NVFP4-family
 * matrix -> planes (rows x planes*cols/2) and scale atoms (orc_mma_sf_bytes). */
int orc_mma_pack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, int fmt,
                 uint8_t* planes, uint8_t* sf)
{
    if (IS_MX(fmt) || rows < 0 || cols % 16) return -1;
    const int np = orc_mma_planes(fmt);
    const int64_t half = cols / 2, nb = cols / 16;
    memset(sf, 0, (size_t)orc_mma_sf_bytes(rows, cols));
    memset(planes, 0, (size_t)(rows * np * half));
    for (int64_t r = 0; r < rows; ++r) {
        uint8_t* prow = planes + r * np * half;
        for (int64_t j = 0; j < cols; ++j) {
            const int code = get_code(codes + r * half, j);
            const int sbyte = scales[r * nb + j / 16];
            int c0 = code, c1 = 0;
            if (np == 2 && code == 8) {
                const double s = special_value(fmt, sbyte);
                const double b = special_base(s);
                c0 = orc_e2m1_encode((float)b);
                c1 = orc_e2m1_encode((float)(s - b));
            }
            set_code(prow, j, c0);
            if (np == 2) set_code(prow + half, j, c1);
        }
        for (int64_t kb = 0; kb < nb; ++kb)
            sf[orc_mma_sf_offset(r, kb, cols)] = (uint8_t)orc_mma_scale_byte(fmt, scales[r * nb + kb]);
    }
    return 0;
}

typedef struct {
    const float *a, *w;
    int64_t m0, m1, N, K;
    double *y, *yabs;
} gemm_job;

static void* gemm_worker(void* p)
{
    gemm_job* j = (gemm_job*)p;
    for (int64_t m = j->m0; m < j->m1; ++m)
        for (int64_t n = 0; n < j->N; ++n) {
            double s = 0.0, t = 0.0;
            for (int64_t k = 0; k < j->K; ++k) {
                const double prod = (double)j->a[m * j->K + k] * (double)j->w[n * j->K + k];
                s += prod;
                t += fabs(prod);
            }
            j->y[m * j->N + n] = s;
            if (j->yabs) j->yabs[m * j->N + n] = t;
        }
    return NULL;
}

/* R9: y = a w^T (a: M x K, w: N x K, row-major fp32), and yabs = |a| |w|^T. */
int orc_gemm(const float* a, const float* w, int64_t M, int64_t N, int64_t K, double* y, double* yabs,
             int nthreads)
{
    if (M < 0 || N < 0 || K < 0) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > M) nthreads = M > 0 ? (int)M : 1;
    gemm_job* jobs = (gemm_job*)calloc((size_t)nthreads, sizeof(gemm_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = (gemm_job){a, w, M * t / nthreads, M * (t + 1) / nthreads, N, K, y, yabs};
        pthread_create(&th[t], NULL, gemm_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(jobs); free(th);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Sparse outlier separation (R11)                                            */
/* ------------------------------------------------------------------------ */

/* Round |v| to a multiple of the quantum 2^qexp, nearest, ties to even multiple. */
static double round_to_quantum(double a, int qexp)
{
    double q = ldexp(a, -qexp);           /* exact: power-of-two scaling */
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    return ldexp(r, qexp);
}

/* binary64 -> bf16 bits, nearest even (8 significant bits, subnormal quantum 2^-133). */
uint16_t orc_f64_to_bf16(double v)
{
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    const double a = fabs(v);
    int k;
    (void)frexp(a, &k);                   /* a in [2^(k-1), 2^k) */
    const int e = k - 1;
    const double r = round_to_quantum(a, e < -126 ? -133 : e - 7);
    const uint16_t h = (uint16_t)(bits_from_f32((float)r) >> 16);   /* r is a bf16 value: exact in binary32 */
    return v < 0.0 ? (uint16_t)(h | 0x8000u) : h;
}

/* binary32 -> fp16 bits, nearest even (11 significant bits, subnormal quantum
 * 2^-24), magnitudes above 65504 saturating to 65504. */
uint16_t orc_f32_to_f16_sat(float f)
{
    const double v = (double)f;
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    const double a = fabs(v);
    int k;
    (void)frexp(a, &k);
    const int e = k - 1;
    double r = round_to_quantum(a, e < -14 ? -24 : e - 10);
    if (r > 65504.0) r = 65504.0;
    uint16_t h;
    if (r < ldexp(1.0, -14)) {
        h = (uint16_t)ldexp(r, 24);       /* subnormal: r / 2^-24 */
    } else {
        (void)frexp(r, &k);
        const int ex = k - 1;
        h = (uint16_t)(((ex + 15) << 10) | (int)(ldexp(r, 10 - ex) - 1024.0));
    }
    return v < 0.0 ? (uint16_t)(h | 0x8000u) : h;
}

double orc_f16_value(uint16_t h)
{
    const int ex = (h >> 10) & 31, m = h & 1023;
    double a;
    if (ex == 0) a = ldexp((double)m, -24);
    else if (ex == 31) a = m ? NAN : INFINITY;
    else a = ldexp(1.0 + m / 1024.0, ex - 15);
    return (h & 0x8000u) ? -a : a;
}

int64_t orc_outlier_capacity(int64_t cols, double max_frac) { return (int64_t)floor(max_frac * (double)cols); }

typedef struct { double d; int64_t j; } cand;

static int cand_order(const void* pa, const void* pb)
{
    const cand* a = (const cand*)pa; const cand* b = (const cand*)pb;
    if (a->d != b->d) return a->d > b->d ? -1 : 1;      /* larger deviation first */
    return a->j < b->j ? -1 : (a->j > b->j);             /* then the lower column */
}

static int col_order(const void* pa, const void* pb)
{
    const cand* a = (const cand*)pa; const cand* b = (const cand*)pb;
    return a->j < b->j ? -1 : (a->j > b->j);
}

/* R11 on a rows x cols bf16 matrix (row stride ldx): bulk (rows x cols bf16,
 * dense), outlier columns and fp16 values ([rows][cap], column order) and the
 * count per row.  Also returns each row's mu and k sigma when mu / thr are
 * non-null. */
int orc_separate_outliers(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx, double k, int64_t cap,
                          uint16_t* bulk, uint16_t* out_cols, uint16_t* out_vals, int32_t* out_count,
                          double* mu_out, double* thr_out)
{
    if (rows < 0 || cols <= 0 || ldx < cols || cap < 0 || cols > 65536) return -1;
    cand* c = (cand*)malloc(sizeof(cand) * (size_t)cols);
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + r * ldx;
        double s = 0.0;
        for (int64_t j = 0; j < cols; ++j) s += (double)orc_bf16_to_f32(xr[j]);
        const double mu = s / (double)cols;
        double v = 0.0;
        for (int64_t j = 0; j < cols; ++j) {
            const double t = (double)orc_bf16_to_f32(xr[j]) - mu;
            v += t * t;
        }
        const double thr = k * sqrt(v / (double)cols);
        int64_t n = 0;
        for (int64_t j = 0; j < cols; ++j) {
            const double d = fabs((double)orc_bf16_to_f32(xr[j]) - mu);
            if (d > thr) c[n++] = (cand){d, j};
        }
        if (n > cap) {
            qsort(c, (size_t)n, sizeof(cand), cand_order);
            n = cap;
        }
        qsort(c, (size_t)n, sizeof(cand), col_order);
        const uint16_t mub = orc_f64_to_bf16(mu);
        for (int64_t j = 0; j < cols; ++j) bulk[r * cols + j] = xr[j];
        for (int64_t i = 0; i < n; ++i) {
            bulk[r * cols + c[i].j] = mub;
            out_cols[r * cap + i] = (uint16_t)c[i].j;
            out_vals[r * cap + i] = orc_f32_to_f16_sat(orc_bf16_to_f32(xr[c[i].j]));
        }
        out_count[r] = (int32_t)n;
        if (mu_out) mu_out[r] = mu;
        if (thr_out) thr_out[r] = thr;
    }
    free(c);
    return 0;
}
