/*
 * wq_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow CPU model of the INT4 / INT2 weight-quantized matmul
 *     C[M,N] = A[M,K] x dequant(Wq[N,K])^T
 * written so that each step can be checked by eye against the two pages it
 * follows.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg call it; the CUDA library never links it and it shares no code,
 * header or table with the CUDA library.
 *
 * Sources (cited by short tag below):
 *   [CG]  "Accelerating LLM inference with CUDA Graph and INT4 quantization"
 *         (cnblogs, JCpeng), part 1 "quantized compute with the T4 INT4
 *         instruction set (DP4A)":
 *           step 1 weight quantization   -- symmetric absmax scale, round,
 *                                           clip; two INT4 values per byte;
 *           step 2 activation quantization -- q = round(a / a_scale);
 *           step 3 INT4 GEMM computation flow -- unpack each byte into two
 *                                           INT4 values, DP4A dot product
 *                                           c += a0*b0 + a1*b1 + a2*b2 + a3*b3,
 *                                           INT32 accumulation;
 *           step 4 dequantization         -- multiply the INT32 result by
 *                                           (weight_scale * activation_scale),
 *                                           optionally add a bias, emit FP16.
 *   [BB]  "BitBLAS practical guide: mixed-precision compute in vLLM" (mlqm):
 *           "What is BitBLAS"             -- C[M,N] = A[M,K] x W[N,K];
 *           "Advanced features 1"         -- MatmulConfig with layout "nt";
 *           "Advanced features 2"         -- group_size=128, with_scaling,
 *                                           with_zeros, zeros_mode "original";
 *           "Core advantages 2"           -- FP16xINT4, FP16xINT2, INT8xINT2;
 *           "Core advantages 3"           -- INT4 / INT2 = 1/4 / 1/8 of FP16 bytes;
 *           "Real-world case"             -- BitNet-b1.58 ternary weights.
 *
 * Readings taken where the pages are silent or garbled (the INT4 passage of
 * [CG] step 1 prints the INT8 range 127 / [-127,127]):
 *   - symmetric INT4: scale = absmax / 7, codes clipped to [-7, 7], stored as
 *     the offset-binary nibble q + 8;
 *   - asymmetric INT4 ("original" zeros): range widened to include 0,
 *     scale = (max - min) / 15, zero = round(-min / scale) in [0, 15],
 *     q = clip(round(w / scale) + zero, 0, 15), w ~ (q - zero) * scale;
 *   - scales are computed in binary32, stored as binary16 (round to nearest
 *     even), and the STORED value is the one used to quantize;
 *   - "round" is round-half-to-even (C rintf in the default rounding mode);
 *     divisions are IEEE binary32 divisions;
 *   - activations: per-token a_scale = absmax / 127 in binary32, codes clipped
 *     to [-127, 127];
 *   - ternary (BitNet-b1.58) weights: one binary32 scale per tensor equal to
 *     mean |w| (exact sum rounded once to binary64, divided by the element
 *     count in binary64, rounded to binary32); q = clip(round(w / s), -1, 1);
 *     stored as 2-bit two's complement fields, four per byte;
 *   - packing: byte j of a row holds element 2j in bits 0..3 and element 2j+1
 *     in bits 4..7 (INT2: element 4j+i in bits 2i..2i+1);
 *   - degenerate groups (scale 0) quantize to code 0 (nibble 8 when symmetric).
 *
 * The other weight types of [BB] "Main features" (FP16 x FP8 / FP4 / INT1 and
 * INT8 x INT1; "Core advantages 3": INT1 is 1/16 of the FP16 bytes).  The page
 * names the types only; the readings are:
 *   - FP4 = e2m1 (1 sign, 2 exponent bits with bias 1, 1 mantissa bit; values
 *     0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives), FP8 = e4m3 (1 sign,
 *     4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest
 *     finite 448);  per group of gs elements along K: scale = binary16 of
 *     absmax / 6 (e2m1) or absmax / 448 (e4m3), the stored value used; code =
 *     the format's value nearest to w / scale (binary32 quotient, clipped to
 *     the largest finite value), ties to the even last mantissa bit; a
 *     magnitude that rounds to 0 is the code +0; scale 0 gives code 0.  FP4
 *     packs like INT4, FP8 is one byte per element;
 *   - INT1 = binary weights: one binary32 scale per tensor equal to mean |w|
 *     (as for ternary), code c = 1 when w >= 0 else 0, value (2c - 1) * scale;
 *     element 8j+i in bit i of byte j.
 * The page's data-type table also lists FP8_E4M3 x FP8_E4M3 -> FP32 -> FP16: FP8
 * activations with FP8 weights.  Reading: the activations are quantized per token
 * like the INT8 ones, scale = absmax / 448 in binary32, code = e4m3 of a / scale
 * (the weight rounding above); the products of code values are summed per weight
 * group, times the group's weight scale, and the token's scale is applied last:
 *     C[m,n] = fp16( a_scale[m] * sum_g s[n,g] * sum_{k in g} v(Aq[m,k]) v(Wq[n,k])  (+ bias) ).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared -pthread
 * (IEEE binary32 / binary64 arithmetic on SSE, round to nearest even).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_OVERFLOW 2

enum { ORC_F16 = 1, ORC_BF16 = 2 };
/* weight formats: integer codes (INT4 / INT2 / INT1 by `bits`), e2m1, e4m3 */
enum { ORC_FMT_INT = 0, ORC_FMT_E2M1 = 1, ORC_FMT_E4M3 = 2 };

/* ------------------------------------------------------------------------ */
/* binary16 / bfloat16 rounding, from the IEEE 754 definition                */
/* ------------------------------------------------------------------------ */

/* Round finite x to the nearest number of a binary format with p significand
 * bits (implicit bit counted) and smallest normal 2^emin; ties to even; with
 * gradual underflow; results above max_finite become +-inf, which is what
 * round-to-nearest-even gives for them. */
static double round_to_format(double x, int p, int emin, double max_finite)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);                               /* |x| in [2^(e-1), 2^e) */
    int top = (e - 1 > emin) ? e - 1 : emin;    /* binade, clamped at subnormals */
    int ulp_exp = top - (p - 1);
    double r = ldexp(rint(ldexp(x, -ulp_exp)), ulp_exp);
    if (fabs(r) > max_finite) r = copysign(INFINITY, x);
    return r;
}

uint16_t orc_f64_to_f16(double x)
{
    if (isnan(x)) return 0x7e00;
    double r = round_to_format(x, 11, -14, 65504.0);
    uint16_t sign = signbit(r) ? 0x8000 : 0;
    double a = fabs(r);
    if (isinf(a)) return sign | 0x7c00;
    if (a < 0x1p-14) return sign | (uint16_t)(a * 0x1p24);   /* a = m * 2^-24 */
    int e;
    double f = frexp(a, &e);                    /* a = (2f) * 2^(e-1), 2f in [1,2) */
    uint16_t man = (uint16_t)((2.0 * f - 1.0) * 1024.0);
    return sign | (uint16_t)((e - 1 + 15) << 10) | man;
}

double orc_f16_to_f64(uint16_t h)
{
    int sign = h >> 15, ex = (h >> 10) & 0x1f, man = h & 0x3ff;
    double v;
    if (ex == 0) v = ldexp((double)man, -24);
    else if (ex == 31) v = man ? NAN : INFINITY;
    else v = ldexp((double)(1024 + man), ex - 25);
    return sign ? -v : v;
}

uint16_t orc_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7fc0;
    double r = round_to_format(x, 8, -126, 0x1.fep127);
    float f = (float)r;                         /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

double orc_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* e2m1 / e4m3 (sign | exponent | mantissa, the layouts of the readings above):
 * value of a code from the definition of a binary format with a subnormal
 * binade, and the code of a value the format holds (searched in the code
 * table, so that encode and decode cannot disagree). */
double orc_minifloat_value(int fmt, int code)
{
    int eb = fmt == ORC_FMT_E2M1 ? 2 : 4, mb = fmt == ORC_FMT_E2M1 ? 1 : 3;
    int bias = fmt == ORC_FMT_E2M1 ? 1 : 7;
    int sign = (code >> (eb + mb)) & 1, e = (code >> mb) & ((1 << eb) - 1), m = code & ((1 << mb) - 1);
    if (fmt == ORC_FMT_E4M3 && e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp((double)m, 1 - bias - mb)                    /* subnormal: m * 2^(1-bias-mb) */
                      : ldexp((double)((1 << mb) + m), e - bias - mb);     /* (1 + m / 2^mb) * 2^(e-bias) */
    return sign ? -v : v;
}

static double minifloat_max(int fmt) { return fmt == ORC_FMT_E2M1 ? 6.0 : 448.0; }

/* Round x (|x| <= the format's largest finite value) to the format: nearest,
 * ties to even (the generic binary rounding above with p = mantissa bits + 1
 * and the smallest normal 2^(1-bias)); returns the code, +0 for a zero result. */
int orc_minifloat_encode(int fmt, double x)
{
    int p = fmt == ORC_FMT_E2M1 ? 2 : 4, emin = fmt == ORC_FMT_E2M1 ? 0 : -6;
    int ncode = fmt == ORC_FMT_E2M1 ? 16 : 256;
    double r = round_to_format(x, p, emin, minifloat_max(fmt));
    if (r == 0.0) return 0;
    for (int c = 0; c < ncode; ++c)
        if (orc_minifloat_value(fmt, c) == r) return c;
    return -1;                                      /* not reached for |x| <= max */
}

static double act_value(const uint16_t *A, int dt, int64_t i)
{
    return dt == ORC_BF16 ? orc_bf16_to_f64(A[i]) : orc_f16_to_f64(A[i]);
}

static uint16_t round_out(double x, int dt)
{
    return dt == ORC_BF16 ? orc_f64_to_bf16(x) : orc_f64_to_f16(x);
}

/* ------------------------------------------------------------------------ */
/* packing ([CG] step 1 "storage": two INT4 values in one byte)              */
/* ------------------------------------------------------------------------ */

/* fields: unsigned field values [N,K] (0..15 for INT4, 0..3 for INT2). */
int orc_pack(const uint8_t *fields, int64_t N, int64_t K, int bits, uint8_t *out)
{
    if (bits == 4) {
        if (K % 2) return ORC_ERR_ARG;
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < K / 2; ++j) {
                uint8_t lo = fields[n * K + 2 * j] & 15, hi = fields[n * K + 2 * j + 1] & 15;
                out[n * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
            }
        return ORC_OK;
    }
    if (bits == 2) {
        if (K % 4) return ORC_ERR_ARG;
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < K / 4; ++j) {
                uint8_t b = 0;
                for (int i = 0; i < 4; ++i) b |= (uint8_t)((fields[n * K + 4 * j + i] & 3) << (2 * i));
                out[n * (K / 4) + j] = b;
            }
        return ORC_OK;
    }
    if (bits == 1) {
        if (K % 8) return ORC_ERR_ARG;
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < K / 8; ++j) {
                uint8_t b = 0;
                for (int i = 0; i < 8; ++i) b |= (uint8_t)((fields[n * K + 8 * j + i] & 1) << i);
                out[n * (K / 8) + j] = b;
            }
        return ORC_OK;
    }
    if (bits == 8) {
        memcpy(out, fields, (size_t)(N * K));
        return ORC_OK;
    }
    return ORC_ERR_ARG;
}

/* Field value of element k of row n. */
static int field_at(const uint8_t *Wq, int64_t K, int bits, int64_t n, int64_t k)
{
    if (bits == 8) return Wq[n * K + k];
    if (bits == 4) {
        uint8_t b = Wq[n * (K / 2) + k / 2];
        return (k & 1) ? (b >> 4) : (b & 15);
    }
    if (bits == 1) return (Wq[n * (K / 8) + k / 8] >> (k & 7)) & 1;
    uint8_t b = Wq[n * (K / 4) + k / 4];
    return (b >> (2 * (k & 3))) & 3;
}

/* Signed code of an integer field: symmetric INT4 nibble - 8, asymmetric INT4
 * nibble unchanged, INT2 two's complement, INT1 2c - 1. */
static int code_of(int field, int bits, int symmetric)
{
    if (bits == 4) return symmetric ? field - 8 : field;
    if (bits == 1) return 2 * field - 1;
    return field >= 2 ? field - 4 : field;
}

/* Bits per element of a weight format, 0 if the pair is not one. */
static int format_bits(int fmt, int bits)
{
    if (fmt == ORC_FMT_INT) return (bits == 4 || bits == 2 || bits == 1) ? bits : 0;
    if (fmt == ORC_FMT_E2M1) return bits == 4 ? 4 : 0;
    if (fmt == ORC_FMT_E4M3) return bits == 8 ? 8 : 0;
    return 0;
}

/* Integer formats: the signed codes; e2m1 / e4m3: the raw codes (as bytes). */
int orc_unpack(const uint8_t *Wq, int64_t N, int64_t K, int bits, int fmt, int symmetric, int8_t *q)
{
    if (!format_bits(fmt, bits) || K % (8 / (bits < 8 ? bits : 8))) return ORC_ERR_ARG;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int f = field_at(Wq, K, bits, n, k);
            q[n * K + k] = (int8_t)(fmt == ORC_FMT_INT ? code_of(f, bits, symmetric) : f);
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* weight quantization ([CG] step 1, [BB] advanced features 2)               */
/* ------------------------------------------------------------------------ */

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Symmetric INT4 per group of gs elements along K. scales: binary16 bits [N, K/gs]. */
int orc_quant_int4_sym(const float *W, int64_t N, int64_t K, int64_t gs, uint8_t *Wq, uint16_t *scales)
{
    if (gs <= 0 || K % gs || K % 2) return ORC_ERR_ARG;
    int64_t G = K / gs;
    uint8_t *fields = (uint8_t *)malloc((size_t)(N * K));
    if (!fields) return ORC_ERR_ARG;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + n * K + g * gs;
            float amax = 0.0f;
            for (int64_t i = 0; i < gs; ++i) amax = fmaxf(amax, fabsf(w[i]));
            float s32 = amax / 7.0f;
            uint16_t sh = orc_f64_to_f16((double)s32);
            float s = (float)orc_f16_to_f64(sh);       /* quantize with the stored scale */
            scales[n * G + g] = sh;
            for (int64_t i = 0; i < gs; ++i) {
                float q = 0.0f;
                if (s != 0.0f) q = clampf(rintf(w[i] / s), -7.0f, 7.0f);
                fields[n * K + g * gs + i] = (uint8_t)((int)q + 8);
            }
        }
    int rc = orc_pack(fields, N, K, 4, Wq);
    free(fields);
    return rc;
}

/* Asymmetric INT4 ("original" zero points) per group. scales, zeros: binary16 [N, K/gs]. */
int orc_quant_int4_asym(const float *W, int64_t N, int64_t K, int64_t gs, uint8_t *Wq,
                        uint16_t *scales, uint16_t *zeros)
{
    if (gs <= 0 || K % gs || K % 2) return ORC_ERR_ARG;
    int64_t G = K / gs;
    uint8_t *fields = (uint8_t *)malloc((size_t)(N * K));
    if (!fields) return ORC_ERR_ARG;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + n * K + g * gs;
            float mn = 0.0f, mx = 0.0f;                 /* range always includes 0 */
            for (int64_t i = 0; i < gs; ++i) {
                mn = fminf(mn, w[i]);
                mx = fmaxf(mx, w[i]);
            }
            float s32 = (mx - mn) / 15.0f;
            uint16_t sh = orc_f64_to_f16((double)s32);
            float s = (float)orc_f16_to_f64(sh);
            float z = 0.0f;
            /* + 0.0f: a zero point is an integer in [0,15]; -0 (from -mn when mn == 0) becomes +0 */
            if (s != 0.0f) z = clampf(rintf(-mn / s), 0.0f, 15.0f) + 0.0f;
            scales[n * G + g] = sh;
            zeros[n * G + g] = orc_f64_to_f16((double)z);
            for (int64_t i = 0; i < gs; ++i) {
                float q = 0.0f;
                if (s != 0.0f) q = clampf(rintf(w[i] / s) + z, 0.0f, 15.0f);
                fields[n * K + g * gs + i] = (uint8_t)(int)q;
            }
        }
    int rc = orc_pack(fields, N, K, 4, Wq);
    free(fields);
    return rc;
}

/* Exact sum of |x[i]| over binary32 inputs, rounded once to binary64.
 * Every finite |x| equals m * 2^(E - 149) with an integer m < 2^24 and
 * E = max(biased exponent, 1) - 1 in [0, 253].  The exact sum is therefore the
 * integer sum(m << E) times 2^-149, held here in 12 limbs of 32 bits. */
double orc_exact_abs_sum_f32(const float *x, int64_t count)
{
    uint64_t limb[13];
    memset(limb, 0, sizeof limb);
    for (int64_t i = 0; i < count; ++i) {
        uint32_t u;
        memcpy(&u, &x[i], 4);
        uint32_t be = (u >> 23) & 0xff, frac = u & 0x7fffff;
        if (be == 0xff) return NAN;
        uint64_t m = be ? (frac | 0x800000u) : frac;
        int E = (be ? (int)be : 1) - 1;
        uint64_t v = m << (E % 32);                 /* < 2^55 */
        limb[E / 32] += v & 0xffffffffu;
        limb[E / 32 + 1] += v >> 32;
        if ((i & 0xffffff) == 0xffffff) {           /* keep carries bounded */
            for (int j = 0; j < 12; ++j) { limb[j + 1] += limb[j] >> 32; limb[j] &= 0xffffffffu; }
        }
    }
    for (int j = 0; j < 12; ++j) { limb[j + 1] += limb[j] >> 32; limb[j] &= 0xffffffffu; }
    /* highest set bit */
    int top = -1;
    for (int j = 12; j >= 0 && top < 0; --j)
        if (limb[j]) for (int b = 31; b >= 0; --b) if ((limb[j] >> b) & 1) { top = 32 * j + b; break; }
    if (top < 0) return 0.0;
#define BIT(p) ((p) >= 0 ? (int)((limb[(p) / 32] >> ((p) % 32)) & 1) : 0)
    uint64_t mant = 0;
    int lo = top - 52;                              /* lowest kept bit */
    for (int p = top; p >= lo && p >= 0; --p) mant = (mant << 1) | (uint64_t)BIT(p);
    if (lo < 0) return ldexp((double)mant, -149);   /* fewer than 54 bits: exact */
    int round_bit = BIT(lo - 1), sticky = 0;
    for (int p = lo - 2; p >= 0; --p) sticky |= BIT(p);
#undef BIT
    if (round_bit && (sticky || (mant & 1))) ++mant;   /* ties to even; 2^53 is still exact */
    return ldexp((double)mant, lo - 149);
}

/* Ternary (BitNet-b1.58) quantization with one binary32 scale per tensor.
 * scale_out[0] = mean |w|; 2-bit two's complement fields, four per byte. */
int orc_quant_ternary(const float *W, int64_t N, int64_t K, uint8_t *Wq, float *scale_out)
{
    if (K % 4) return ORC_ERR_ARG;
    double sum = orc_exact_abs_sum_f32(W, N * K);
    float s = (float)(sum / (double)(N * K));
    scale_out[0] = s;
    uint8_t *fields = (uint8_t *)malloc((size_t)(N * K));
    if (!fields) return ORC_ERR_ARG;
    for (int64_t i = 0; i < N * K; ++i) {
        float q = 0.0f;
        if (s != 0.0f) q = clampf(rintf(W[i] / s), -1.0f, 1.0f);
        fields[i] = (uint8_t)((int)q & 3);
    }
    int rc = orc_pack(fields, N, K, 2, Wq);
    free(fields);
    return rc;
}

/* e2m1 / e4m3 per group of gs elements along K ([BB] "Main features", with
 * the group scheme of "Advanced features 2"). scales: binary16 bits [N, K/gs]. */
int orc_quant_minifloat(const float *W, int64_t N, int64_t K, int64_t gs, int fmt, uint8_t *Wq, uint16_t *scales)
{
    if ((fmt != ORC_FMT_E2M1 && fmt != ORC_FMT_E4M3) || gs <= 0 || K % gs || K % 2) return ORC_ERR_ARG;
    int64_t G = K / gs;
    float fmax = (float)minifloat_max(fmt);
    uint8_t *fields = (uint8_t *)malloc((size_t)(N * K));
    if (!fields) return ORC_ERR_ARG;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + n * K + g * gs;
            float amax = 0.0f;
            for (int64_t i = 0; i < gs; ++i) amax = fmaxf(amax, fabsf(w[i]));
            uint16_t sh = orc_f64_to_f16((double)(amax / fmax));
            float s = (float)orc_f16_to_f64(sh);
            scales[n * G + g] = sh;
            for (int64_t i = 0; i < gs; ++i) {
                int c = 0;
                if (s != 0.0f) c = orc_minifloat_encode(fmt, (double)clampf(w[i] / s, -fmax, fmax));
                if (c < 0) { free(fields); return ORC_ERR_ARG; }
                fields[n * K + g * gs + i] = (uint8_t)c;
            }
        }
    int rc = orc_pack(fields, N, K, fmt == ORC_FMT_E2M1 ? 4 : 8, Wq);
    free(fields);
    return rc;
}

/* Binary (INT1) quantization with one binary32 scale per tensor:
 * scale_out[0] = mean |w| (as for ternary); bit 1 for w >= 0, eight per byte. */
int orc_quant_binary(const float *W, int64_t N, int64_t K, uint8_t *Wq, float *scale_out)
{
    if (K % 8) return ORC_ERR_ARG;
    double sum = orc_exact_abs_sum_f32(W, N * K);
    scale_out[0] = (float)(sum / (double)(N * K));
    uint8_t *fields = (uint8_t *)malloc((size_t)(N * K));
    if (!fields) return ORC_ERR_ARG;
    for (int64_t i = 0; i < N * K; ++i) fields[i] = W[i] >= 0.0f ? 1 : 0;
    int rc = orc_pack(fields, N, K, 1, Wq);
    free(fields);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* activation quantization ([CG] step 2), per token                          */
/* ------------------------------------------------------------------------ */

int orc_act_quant_int8(const uint16_t *A, int a_dt, int64_t M, int64_t K, int8_t *Aq, float *a_scale)
{
    if (a_dt != ORC_F16 && a_dt != ORC_BF16) return ORC_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) amax = fmaxf(amax, fabsf((float)act_value(A, a_dt, m * K + k)));
        float sc = amax / 127.0f;
        a_scale[m] = sc;
        for (int64_t k = 0; k < K; ++k) {
            float q = 0.0f;
            if (sc != 0.0f) q = clampf(rintf((float)act_value(A, a_dt, m * K + k) / sc), -127.0f, 127.0f);
            Aq[m * K + k] = (int8_t)(int)q;
        }
    }
    return ORC_OK;
}

/* FP8 activations per token ([BB] data-type table, FP8_E4M3 x FP8_E4M3):
 * a_scale[m] = absmax / 448 (binary32), Aq = e4m3 code of clip(a / a_scale, -448, 448). */
int orc_act_quant_e4m3(const uint16_t *A, int a_dt, int64_t M, int64_t K, uint8_t *Aq, float *a_scale)
{
    if (a_dt != ORC_F16 && a_dt != ORC_BF16) return ORC_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) amax = fmaxf(amax, fabsf((float)act_value(A, a_dt, m * K + k)));
        float sc = amax / 448.0f;
        a_scale[m] = sc;
        for (int64_t k = 0; k < K; ++k) {
            int c = 0;
            if (sc != 0.0f) c = orc_minifloat_encode(ORC_FMT_E4M3, (double)clampf((float)act_value(A, a_dt, m * K + k) / sc, -448.0f, 448.0f));
            if (c < 0) return ORC_ERR_ARG;
            Aq[m * K + k] = (uint8_t)c;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* reference matmuls ([BB] "What is BitBLAS"; [CG] steps 3-4)                */
/* ------------------------------------------------------------------------ */

typedef struct {
    /* problem */
    const uint16_t *A; int a_dt;                 /* A16 */
    const int8_t *Aq; const float *a_scale;      /* A8 */
    int64_t M, N, K;
    const uint8_t *Wq; int bits, fmt, symmetric; int64_t gs;
    const uint16_t *scales16; const float *scale32; const uint16_t *zeros; const uint16_t *bias;
    /* selection */
    const int64_t *m_idx; int64_t m_cnt;
    const int64_t *n_idx; int64_t n_cnt;
    /* outputs, [m_cnt, n_cnt] */
    double *C_exact; uint16_t *C_out; int32_t *acc_out;
    /* thread slice over the selected n */
    int64_t j0, j1; int status;
} job_t;

static int64_t sel(const int64_t *idx, int64_t j) { return idx ? idx[j] : j; }

/* Dequantized weight w[n,k] = (q - z) * s, or value(code) * s for e2m1 / e4m3,
 * exact in binary64 (|q - z| <= 15, a code value has at most 4 significant bits,
 * s a binary16 or binary32 value). */
static double dequant_weight(const job_t *J, int64_t n, int64_t k)
{
    int f = field_at(J->Wq, J->K, J->bits, n, k);
    if (J->fmt != ORC_FMT_INT) {
        int64_t G = J->K / J->gs;
        return orc_minifloat_value(J->fmt, f) * orc_f16_to_f64(J->scales16[n * G + k / J->gs]);
    }
    int c = code_of(f, J->bits, J->symmetric);
    if (J->bits <= 2) return (double)c * (double)J->scale32[0];
    int64_t G = J->K / J->gs, g = k / J->gs;
    double s = orc_f16_to_f64(J->scales16[n * G + g]);
    double z = (J->symmetric || !J->zeros) ? 0.0 : orc_f16_to_f64(J->zeros[n * G + g]);
    return ((double)c - z) * s;
}

static void *run_a16(void *arg)
{
    job_t *J = (job_t *)arg;
    double *w = (double *)malloc((size_t)J->K * sizeof(double));
    if (!w) { J->status = ORC_ERR_ARG; return NULL; }
    for (int64_t j = J->j0; j < J->j1; ++j) {
        int64_t n = sel(J->n_idx, j);
        for (int64_t k = 0; k < J->K; ++k) w[k] = dequant_weight(J, n, k);
        for (int64_t i = 0; i < J->m_cnt; ++i) {
            int64_t m = sel(J->m_idx, i);
            double acc = 0.0;
            for (int64_t k = 0; k < J->K; ++k) acc += act_value(J->A, J->a_dt, m * J->K + k) * w[k];
            if (J->bias) acc += act_value(J->bias, J->a_dt, n);
            if (J->C_exact) J->C_exact[i * J->n_cnt + j] = acc;
            if (J->C_out) J->C_out[i * J->n_cnt + j] = round_out(acc, J->a_dt);
        }
    }
    free(w);
    return NULL;
}

static void *run_a8(void *arg)
{
    job_t *J = (job_t *)arg;
    int64_t G = J->bits <= 2 ? 1 : J->K / J->gs;
    int64_t glen = J->bits <= 2 ? J->K : J->gs;
    int32_t *qz = (int32_t *)malloc((size_t)J->K * sizeof(int32_t));
    if (!qz) { J->status = ORC_ERR_ARG; return NULL; }
    for (int64_t j = J->j0; j < J->j1; ++j) {
        int64_t n = sel(J->n_idx, j);
        /* integer weight codes minus integer zero point */
        for (int64_t k = 0; k < J->K; ++k) {
            int c = code_of(field_at(J->Wq, J->K, J->bits, n, k), J->bits, J->symmetric);
            int z = 0;
            if (J->bits == 4 && !J->symmetric && J->zeros) {
                double zd = orc_f16_to_f64(J->zeros[n * G + k / J->gs]);
                if (zd != floor(zd)) { J->status = ORC_ERR_ARG; free(qz); return NULL; }
                z = (int)zd;
            }
            qz[k] = c - z;
        }
        for (int64_t i = 0; i < J->m_cnt; ++i) {
            int64_t m = sel(J->m_idx, i);
            double total = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t acc = 0;                         /* DP4A: sum of int8 x int products */
                for (int64_t k = g * glen; k < (g + 1) * glen; ++k)
                    acc += (int64_t)J->Aq[m * J->K + k] * (int64_t)qz[k];
                if (acc > INT32_MAX || acc < INT32_MIN) J->status = ORC_ERR_OVERFLOW;
                if (J->acc_out) J->acc_out[(i * J->n_cnt + j) * G + g] = (int32_t)acc;
                double s = J->bits <= 2 ? (double)J->scale32[0] : orc_f16_to_f64(J->scales16[n * G + g]);
                total += s * (double)acc;
            }
            double c = (double)J->a_scale[m] * total;   /* (w_scale * a_scale) dequantization */
            if (J->bias) c += orc_f16_to_f64(J->bias[n]);
            if (J->C_exact) J->C_exact[i * J->n_cnt + j] = c;
            if (J->C_out) J->C_out[i * J->n_cnt + j] = orc_f64_to_f16(c);
        }
    }
    free(qz);
    return NULL;
}

/* FP8 x FP8: per group, the sum of products of the code values (binary64), times the
 * weight group scale; the token scale last. */
static void *run_f8(void *arg)
{
    job_t *J = (job_t *)arg;
    int64_t G = J->K / J->gs;
    const uint8_t *Aq = (const uint8_t *)J->Aq;
    double *w = (double *)malloc((size_t)J->K * sizeof(double));
    if (!w) { J->status = ORC_ERR_ARG; return NULL; }
    for (int64_t j = J->j0; j < J->j1; ++j) {
        int64_t n = sel(J->n_idx, j);
        for (int64_t k = 0; k < J->K; ++k) w[k] = orc_minifloat_value(ORC_FMT_E4M3, J->Wq[n * J->K + k]);
        for (int64_t i = 0; i < J->m_cnt; ++i) {
            int64_t m = sel(J->m_idx, i);
            double total = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                double acc = 0.0;
                for (int64_t k = g * J->gs; k < (g + 1) * J->gs; ++k)
                    acc += orc_minifloat_value(ORC_FMT_E4M3, Aq[m * J->K + k]) * w[k];
                total += orc_f16_to_f64(J->scales16[n * G + g]) * acc;
            }
            double c = (double)J->a_scale[m] * total;
            if (J->bias) c += orc_f16_to_f64(J->bias[n]);
            if (J->C_exact) J->C_exact[i * J->n_cnt + j] = c;
            if (J->C_out) J->C_out[i * J->n_cnt + j] = orc_f64_to_f16(c);
        }
    }
    free(w);
    return NULL;
}

static int run_threads(job_t *proto, void *(*fn)(void *), int threads)
{
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    if (threads > proto->n_cnt) threads = proto->n_cnt > 0 ? (int)proto->n_cnt : 1;
    job_t jobs[256];
    pthread_t tid[256];
    for (int t = 0; t < threads; ++t) {
        jobs[t] = *proto;
        jobs[t].j0 = proto->n_cnt * t / threads;
        jobs[t].j1 = proto->n_cnt * (t + 1) / threads;
        jobs[t].status = ORC_OK;
    }
    for (int t = 1; t < threads; ++t) pthread_create(&tid[t], NULL, fn, &jobs[t]);
    fn(&jobs[0]);
    for (int t = 1; t < threads; ++t) pthread_join(tid[t], NULL);
    int rc = ORC_OK;
    for (int t = 0; t < threads; ++t) if (jobs[t].status != ORC_OK) rc = jobs[t].status;
    return rc;
}

static int check_weights(int64_t K, int bits, int fmt, int64_t gs)
{
    if (!format_bits(fmt, bits)) return ORC_ERR_ARG;
    if (fmt != ORC_FMT_INT || bits == 4) return (gs > 0 && K % gs == 0 && K % 2 == 0) ? ORC_OK : ORC_ERR_ARG;
    return K % (8 / bits) == 0 ? ORC_OK : ORC_ERR_ARG;
}

/* W4A16 / W2A16 / W1A16:  C[m,n] = sum_k A[m,k] * (q[n,k] - z[n,g(k)]) * s[n,g(k)]  (+ bias[n])
 * accumulated in binary64 in k order, then rounded once to A's dtype; for e2m1 / e4m3
 * weights (q - z) is the code's value.
 * scales: binary16 [N, K/gs] (INT4, e2m1, e4m3) or one binary32 (INT2, INT1).
 * zeros: binary16 or NULL.  m_idx / n_idx select the computed rows / columns (NULL = all);
 * outputs are [m_cnt, n_cnt]. */
int orc_gemm_a16(const uint16_t *A, int a_dt, int64_t M, int64_t K,
                 const uint8_t *Wq, int64_t N, int bits, int fmt, int symmetric, int64_t gs,
                 const void *scales, const uint16_t *zeros, const uint16_t *bias,
                 const int64_t *m_idx, int64_t m_cnt, const int64_t *n_idx, int64_t n_cnt,
                 double *C_exact, uint16_t *C_out, int threads)
{
    if ((a_dt != ORC_F16 && a_dt != ORC_BF16) || check_weights(K, bits, fmt, gs) || M < 0 || N < 0)
        return ORC_ERR_ARG;
    job_t J;
    memset(&J, 0, sizeof J);
    J.A = A; J.a_dt = a_dt; J.M = M; J.N = N; J.K = K;
    J.Wq = Wq; J.bits = bits; J.fmt = fmt; J.symmetric = symmetric; J.gs = gs;
    J.scales16 = (const uint16_t *)scales; J.scale32 = (const float *)scales;
    J.zeros = zeros; J.bias = bias;
    J.m_idx = m_idx; J.m_cnt = m_idx ? m_cnt : M;
    J.n_idx = n_idx; J.n_cnt = n_idx ? n_cnt : N;
    J.C_exact = C_exact; J.C_out = C_out;
    return run_threads(&J, run_a16, threads);
}

/* W4A8 / W2A8 / W1A8:  acc_g[m,n] = sum_{k in group g} Aq[m,k] * (q[n,k] - z[n,g])   (exact integer)
 *               C[m,n] = fp16( a_scale[m] * sum_g s[n,g] * acc_g[m,n]  (+ bias[n]) )
 * The integer dot product is the DP4A definition; the float scale is applied
 * after integer accumulation.  INT2 and INT1 weights have one group spanning all
 * of K and one binary32 scale.  acc_out (optional): int32 [m_cnt, n_cnt, G].
 * Returns ORC_ERR_OVERFLOW if some group sum leaves the int32 range. */
int orc_gemm_a8(const int8_t *Aq, const float *a_scale, int64_t M, int64_t K,
                const uint8_t *Wq, int64_t N, int bits, int symmetric, int64_t gs,
                const void *scales, const uint16_t *zeros, const uint16_t *bias,
                const int64_t *m_idx, int64_t m_cnt, const int64_t *n_idx, int64_t n_cnt,
                double *C_exact, uint16_t *C_out, int32_t *acc_out, int threads)
{
    if (check_weights(K, bits, ORC_FMT_INT, gs) || M < 0 || N < 0) return ORC_ERR_ARG;
    job_t J;
    memset(&J, 0, sizeof J);
    J.Aq = Aq; J.a_scale = a_scale; J.M = M; J.N = N; J.K = K;
    J.Wq = Wq; J.bits = bits; J.symmetric = symmetric; J.gs = gs;
    J.scales16 = (const uint16_t *)scales; J.scale32 = (const float *)scales;
    J.zeros = zeros; J.bias = bias;
    J.m_idx = m_idx; J.m_cnt = m_idx ? m_cnt : M;
    J.n_idx = n_idx; J.n_cnt = n_idx ? n_cnt : N;
    J.C_exact = C_exact; J.C_out = C_out; J.acc_out = acc_out;
    return run_threads(&J, run_a8, threads);
}

/* W8A8 FP8 (e4m3 weights with binary16 group scales, e4m3 activations with per-token
 * binary32 scales):
 *   C[m,n] = fp16( a_scale[m] * sum_g s[n,g] * sum_{k in g} v(Aq[m,k]) * v(Wq[n,k])  (+ bias[n]) )
 * summed in binary64.  Wq [N,K] and Aq [M,K] are e4m3 codes (bytes). */
int orc_gemm_f8(const uint8_t *Aq, const float *a_scale, int64_t M, int64_t K,
                const uint8_t *Wq, int64_t N, int64_t gs, const uint16_t *scales, const uint16_t *bias,
                const int64_t *m_idx, int64_t m_cnt, const int64_t *n_idx, int64_t n_cnt,
                double *C_exact, uint16_t *C_out, int threads)
{
    if (gs <= 0 || K % gs || M < 0 || N < 0) return ORC_ERR_ARG;
    job_t J;
    memset(&J, 0, sizeof J);
    J.Aq = (const int8_t *)Aq; J.a_scale = a_scale; J.M = M; J.N = N; J.K = K;
    J.Wq = Wq; J.bits = 8; J.fmt = ORC_FMT_E4M3; J.symmetric = 1; J.gs = gs;
    J.scales16 = scales; J.bias = bias;
    J.m_idx = m_idx; J.m_cnt = m_idx ? m_cnt : M;
    J.n_idx = n_idx; J.n_cnt = n_idx ? n_cnt : N;
    J.C_exact = C_exact; J.C_out = C_out;
    return run_threads(&J, run_f8, threads);
}
