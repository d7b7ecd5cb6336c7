/*
 * fp4_oracle.c -- plain, slow, obviously-correct CPU oracle for block-scaled
 * FP4 (E2M1) quantisation: NVFP4 (16-element blocks, E4M3 block scale, FP32
 * global scale), MXFP4 (32-element blocks, E8M0 power-of-two scale), nibble
 * packing, dequantisation and the per-block MSE scale search.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no source, header, table or helper
 * with the CUDA library; the two meet only through the seeded inputs.
 *
 * Sources (web pages; cited by title and section):
 *   [NVMX]  "NVFP4 与 MXFP4 格式" (charlestar.github.io, nvfp4-mxfp4-format):
 *           S1 "E2M1 的十六种编码究竟表示什么"; S2 shared scales (E8M0, E4M3);
 *           S3 "NVFP4 的两个 scale 怎样完成一次量化"; S4 "scale 量化误差会再次
 *           改变元素格点" (E4M3 codec, reconstruct, MSE, NV reference);
 *           S5 "MXFP4 也不是只有一种 scale 选择算法"; S6 grouping / transpose;
 *           S8 storage cost.
 *   [MATH]  "FP4 / NVFP4 数学总结" (devpress.csdn.net): S3 NVFP4 formula,
 *           S7-S8 max/6 scale worked example, S9 Loss(s), S10 quantise /
 *           dequantise formulas.
 *   [TJ]    "FP4、FP8 与 INT8/INT4：数值范围、块缩放与推理计算精度"
 *           (tom-jerr.github.io): S4 "Scale 怎么选" (four over six).
 *
 * Arithmetic: double for every step the pages write as real arithmetic;
 * IEEE single (C `float`, FLT_EVAL_METHOD == 0, no contraction) for the
 * steps the contract fixes in fp32: the global scale g, the element
 * quotient x / fl32(s_b * g) and the dequant product fl32(fl32(p*s_b)*g).
 *
 * Readings of the pages taken here (each is listed with its reason in the
 * design notes of the repository):
 *   - E2M1 rounding: nearest value, ties to the code with the even low bit;
 *     sign taken from the sign bit (so -0 and tiny negatives give code 8);
 *     magnitudes clamp to 6 ([NVMX] S1).
 *   - NVFP4 block scale: E4M3 code nearest to the exact rational
 *     A_b / (6 g), ties to the even code, clamped at 448 ([NVMX] S3, S4).
 *     The page forms that quotient in double; since A_b has 24 significant
 *     bits and 6 g at most 27, a nonzero distance to any E4M3 midpoint is
 *     at least 2^-33 relative, far above double rounding, so the double
 *     quotient selects the same code as the exact rational.
 *   - A block whose scale rounds to E4M3 zero (including an all-zero block)
 *     gets scale byte 0x00 and all-zero codes: the fixed convention "a zero
 *     scale gives all-zero codes" replaces the page's rejection / b = 1.
 *   - Element quotient v = fl32(x / fl32(s_b * g)) (IEEE single division).
 *   - MXFP4: e = floor(log2 A_b) - 2 (OCP rounding-down rule, [NVMX] S5),
 *     via frexp, clamped to [-127, 127]; an all-zero block clamps to -127.
 *   - Scale search: 64 candidates m_k * A_b / (6 g), m_k = (147 + k) / 210,
 *     k = 0..63 (0.70 .. 1.00 inclusive); loss of the emitted artefact,
 *     summed in double; exact ties go to the larger scale.  The grid form
 *     takes m_k = (p + k) / q, k = 0..n-1, for any n, p, q up to 2^20.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs single-precision operations evaluated in single precision"
#endif

/* Status values returned by the oracle (its own numbering). */
enum {
    ORACLE_OK = 0,
    ORACLE_ERR_ARG = 1,       /* bad argument (NULL pointer, code out of range) */
    ORACLE_ERR_SHAPE = 2,     /* incomplete block or odd length */
    ORACLE_ERR_NONFINITE = 4, /* NaN or Inf in the input */
    ORACLE_ERR_RANGE = 5      /* global scale rounds to zero in fp32 */
};

/* Input element types. */
enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* The eight E2M1 magnitudes, codes 0..7 ([NVMX] S1 table). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* NVFP4 global-scale divisor 6 * 448 ([NVMX] S3). */
#define NV_GLOBAL_DIV 2688.0

/* Scale-search candidate grid: m_k = (147 + k) / 210, k = 0..63. */
#define SEARCH_N 64
#define SEARCH_NUM0 147
#define SEARCH_DEN 210

/* ------------------------------------------------------------------ */
/* Element access: bf16 is the upper half of an fp32 bit pattern.      */
/* ------------------------------------------------------------------ */

static float load_elem(const void *x, int dtype, int64_t i)
{
    if (dtype == ORACLE_F32)
        return ((const float *)x)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)x)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even on the upper 16 bits. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (isnan(f))
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* E2M1 element codec ([NVMX] S1).                                     */
/* ------------------------------------------------------------------ */

/* Value of a four-bit code: sign bit 3, magnitude index bits 0..2.  Code 8
 * is negative zero. */
double oracle_e2m1_decode(int code)
{
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? copysign(m, -1.0) : m;
}

/* Nearest E2M1 code to a finite value.  The magnitude is clamped to 6; the
 * nearest of the eight magnitudes wins and an exact midpoint goes to the
 * code whose low bit is even; the sign bit of the input becomes bit 3. */
int oracle_e2m1_encode(double value, int *code)
{
    if (!isfinite(value))
        return ORACLE_ERR_NONFINITE;
    int sign = signbit(value) ? 8 : 0;
    double m = fabs(value);
    if (m > E2M1_MAG[7])
        m = E2M1_MAG[7];
    int best = 0;
    double best_dist = fabs(E2M1_MAG[0] - m);
    for (int c = 1; c < 8; ++c) {
        double dist = fabs(E2M1_MAG[c] - m);
        if (dist < best_dist || (dist == best_dist && (c & 1) < (best & 1))) {
            best = c;
            best_dist = dist;
        }
    }
    *code = sign | best;
    return ORACLE_OK;
}

/* Codes of n fp32 values; a non-finite value yields 0xFF. */
void oracle_e2m1_encode_f32(const float *v, uint8_t *codes, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        int c;
        codes[i] = oracle_e2m1_encode((double)v[i], &c) == ORACLE_OK ? (uint8_t)c : 0xFF;
    }
}

/* Two codes per byte: element 2i in the low nibble, 2i+1 in the high one. */
int oracle_pack4(const uint8_t *codes, int64_t n, uint8_t *out)
{
    if (n % 2)
        return ORACLE_ERR_SHAPE;
    for (int64_t i = 0; i < n; ++i)
        if (codes[i] > 15)
            return ORACLE_ERR_ARG;
    for (int64_t j = 0; j < n / 2; ++j)
        out[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
    return ORACLE_OK;
}

void oracle_unpack4(const uint8_t *bytes, int64_t nbytes, uint8_t *codes)
{
    for (int64_t j = 0; j < nbytes; ++j) {
        codes[2 * j] = bytes[j] & 15;
        codes[2 * j + 1] = bytes[j] >> 4;
    }
}

/* ------------------------------------------------------------------ */
/* Scale formats ([NVMX] S2, S4).                                       */
/* ------------------------------------------------------------------ */

/* Positive finite E4M3 (FN) code 0..126: exponent field e = code / 8,
 * fraction f = code % 8; e == 0 is subnormal f * 2^-9, otherwise
 * 2^(e-7) * (1 + f/8).  Returns NaN for a code outside 0..126. */
double oracle_e4m3_value(int code)
{
    if (code < 0 || code > 126)
        return NAN;
    int e = code / 8, f = code % 8;
    return e == 0 ? f * ldexp(1.0, -9) : ldexp(1.0 + f / 8.0, e - 7);
}

/* Any E4M3 byte: bit 7 is the sign; 0x7F and 0xFF are NaN. */
double oracle_e4m3_decode_byte(int byte)
{
    int mag = byte & 0x7F;
    if (mag == 0x7F)
        return NAN;
    double v = oracle_e4m3_value(mag);
    return (byte & 0x80) ? -v : v;
}

/* Nearest positive E4M3 code to a finite non-negative value, after
 * saturation to 448; an exact midpoint goes to the even code. */
int oracle_e4m3_encode(double value)
{
    if (!(value >= 0.0) || !isfinite(value))
        return -1;
    double top = oracle_e4m3_value(126);
    if (value > top)
        value = top;
    int best = 0;
    double best_dist = fabs(oracle_e4m3_value(0) - value);
    for (int c = 1; c <= 126; ++c) {
        double dist = fabs(oracle_e4m3_value(c) - value);
        if (dist < best_dist || (dist == best_dist && (c & 1) < (best & 1))) {
            best = c;
            best_dist = dist;
        }
    }
    return best;
}

/* E8M0 byte c: 2^(c-127); 255 is NaN. */
double oracle_e8m0_value(int byte)
{
    if (byte == 255)
        return NAN;
    return ldexp(1.0, byte - 127);
}

/* ------------------------------------------------------------------ */
/* NVFP4 ([NVMX] S3-S4; [MATH] S3, S10).                                */
/* ------------------------------------------------------------------ */

/* A = max |x| over the tensor; any NaN/Inf -> NONFINITE. */
int oracle_tensor_amax(const void *x, int dtype, int64_t n, float *amax)
{
    float a = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float v = load_elem(x, dtype, i);
        if (!isfinite(v))
            return ORACLE_ERR_NONFINITE;
        float m = fabsf(v);
        if (m > a)
            a = m;
    }
    *amax = a;
    return ORACLE_OK;
}

/* g = fl32(A / (6 * 448)), the page's double quotient rounded once to fp32
 * (equal to the IEEE single quotient: 53 >= 2*24 + 2, so the double
 * rounding is innocuous).  An all-zero tensor uses g = 1 ([NVMX] S3,
 * "全零张量").  The page rejects a g that is not finite and positive; with
 * the element quotient fixed in fp32, a subnormal g lets fl32(s_b * g) lose
 * its precision or vanish, so a g below the smallest normal fp32 is
 * rejected too (only tensors with 0 < A < 2688 * 2^-126 reach this). */
int oracle_nv_global_scale(float amax, float *g)
{
    if (!isfinite(amax) || amax < 0.0f)
        return ORACLE_ERR_ARG;
    if (amax == 0.0f) {
        *g = 1.0f;
        return ORACLE_OK;
    }
    float a = (float)((double)amax / NV_GLOBAL_DIV);
    if (!(a >= FLT_MIN) || !isfinite(a))
        return ORACLE_ERR_RANGE;
    *g = a;
    return ORACLE_OK;
}

/* E4M3 block-scale code for block maximum A_b under global scale g:
 * nearest E4M3 to A_b / (6 g) ([NVMX] S3 b* = A_g / (6a), b = Q_E4M3(b*)). */
int oracle_nv_block_scale_code(float amax_b, float g)
{
    double t = (double)amax_b / (6.0 * (double)g);
    return oracle_e4m3_encode(t);
}

/* Codes of one block of n elements at E4M3 scale code sc and global g:
 * zero scale -> all codes 0; else v = fl32(x / fl32(s_b * g)), E2M1. */
static void nv_block_codes(const float *xb, int n, int sc, float g, uint8_t *codes)
{
    double sb = oracle_e4m3_value(sc);
    if (sb == 0.0) {
        for (int i = 0; i < n; ++i)
            codes[i] = 0;
        return;
    }
    float d = (float)sb * g;
    for (int i = 0; i < n; ++i) {
        float v = xb[i] / d;
        int c = 0;
        oracle_e2m1_encode((double)v, &c); /* v is finite: |x| <= ~6.1 d */
        codes[i] = (uint8_t)c;
    }
}

/* NVFP4 dequantised value of one code: fl32(fl32(p * s_b) * g). */
static float nv_dequant_value(int code, double sb, float g)
{
    float ps = (float)(oracle_e2m1_decode(code) * sb); /* exact product */
    return ps * g;
}

/* Quantise with a given global scale g.  x: rows*cols elements row-major,
 * cols % 16 == 0.  packed: rows*cols/2 bytes; scales: rows*cols/16 bytes.
 * The caller guarantees finiteness (the tensor-level call checks it). */
int oracle_nvfp4_quantize_with_g(const void *x, int dtype, int64_t rows, int64_t cols,
                                 float g, uint8_t *packed, uint8_t *scales)
{
    if (cols % 16 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    int64_t nblocks = rows * cols / 16;
    for (int64_t b = 0; b < nblocks; ++b) {
        float xb[16];
        float ab = 0.0f;
        for (int i = 0; i < 16; ++i) {
            xb[i] = load_elem(x, dtype, b * 16 + i);
            if (!isfinite(xb[i]))
                return ORACLE_ERR_NONFINITE;
            if (fabsf(xb[i]) > ab)
                ab = fabsf(xb[i]);
        }
        int sc = oracle_nv_block_scale_code(ab, g);
        uint8_t codes[16];
        nv_block_codes(xb, 16, sc, g, codes);
        scales[b] = (uint8_t)sc;
        oracle_pack4(codes, 16, packed + b * 8);
    }
    return ORACLE_OK;
}

/* Full NVFP4 quantisation: amax -> g -> blocks ([NVMX] S4 NV reference). */
int oracle_nvfp4_quantize(const void *x, int dtype, int64_t rows, int64_t cols,
                          uint8_t *packed, uint8_t *scales, float *g_out)
{
    if (cols % 16 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    float amax, g;
    int st = oracle_tensor_amax(x, dtype, rows * cols, &amax);
    if (st)
        return st;
    st = oracle_nv_global_scale(amax, &g);
    if (st)
        return st;
    *g_out = g;
    return oracle_nvfp4_quantize_with_g(x, dtype, rows, cols, g, packed, scales);
}

/* NVFP4 dequantisation to fp32: y = fl32(fl32(p * s_b) * g), [MATH] S3
 * x_hat = q * s_b * g in that order.  Scale bytes decode as signed E4M3
 * (0x7F / 0xFF -> NaN). */
void oracle_nvfp4_dequantize(const uint8_t *packed, const uint8_t *scales, float g,
                             int64_t rows, int64_t cols, float *y)
{
    int64_t n = rows * cols;
    for (int64_t i = 0; i < n; ++i) {
        int code = (i & 1) ? packed[i / 2] >> 4 : packed[i / 2] & 15;
        double sb = oracle_e4m3_decode_byte(scales[i / 16]);
        y[i] = nv_dequant_value(code, sb, g);
    }
}

/* ------------------------------------------------------------------ */
/* MXFP4 ([NVMX] S2, S5, S6).                                           */
/* ------------------------------------------------------------------ */

/* Shared exponent of a 32-block: floor(log2 A_b) - 2, clamped to the
 * E8M0 range; A_b = 0 clamps to -127.  frexp gives A_b = m 2^E with
 * m in [0.5, 1), so floor(log2 A_b) = E - 1. */
int oracle_mx_block_exponent(float amax_b)
{
    if (amax_b == 0.0f)
        return -127;
    int E;
    frexp((double)amax_b, &E);
    int e = E - 3;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/* Shared exponent of a 32-block under the ceil rule of the page's
 * `mx_scale` helper ([NVMX] S5-S6: the ModelOpt-style 2^ceil(log2(A_b/6))):
 * an all-zero block gets scale 1 (e = 0); otherwise e = max(-127, E - 3)
 * with frexp(A_b) = m 2^E, then e + 1 if A_b > 6 * 2^e (the threshold
 * compare avoids rounding log2 near integers); e > 127 is rejected. */
int oracle_mx_block_exponent_ceil(float amax_b, int *e_out)
{
    if (amax_b == 0.0f) {
        *e_out = 0;
        return ORACLE_OK;
    }
    int E;
    frexp((double)amax_b, &E);
    int e = E - 3;
    if (e < -127)
        e = -127;
    if ((double)amax_b > 6.0 * ldexp(1.0, e))
        e += 1;
    if (e > 127)
        return ORACLE_ERR_RANGE;
    *e_out = e;
    return ORACLE_OK;
}

/* MXFP4 with the scale rule chosen: rule 0 = OCP rounding-down (floor),
 * rule 1 = the ceil rule above. */
int oracle_mxfp4_quantize_rule(const void *x, int dtype, int64_t rows, int64_t cols, int rule,
                               uint8_t *packed, uint8_t *scales)
{
    if (cols % 32 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    if (rule != 0 && rule != 1)
        return ORACLE_ERR_ARG;
    int64_t n = rows * cols;
    for (int64_t i = 0; i < n; ++i)
        if (!isfinite(load_elem(x, dtype, i)))
            return ORACLE_ERR_NONFINITE;
    int64_t nblocks = n / 32;
    for (int64_t b = 0; b < nblocks; ++b) {
        float ab = 0.0f;
        for (int i = 0; i < 32; ++i) {
            float m = fabsf(load_elem(x, dtype, b * 32 + i));
            if (m > ab)
                ab = m;
        }
        int e;
        if (rule == 0) {
            e = oracle_mx_block_exponent(ab);
        } else {
            int st = oracle_mx_block_exponent_ceil(ab, &e);
            if (st)
                return st;
        }
        double scale = ldexp(1.0, e);
        uint8_t codes[32];
        for (int i = 0; i < 32; ++i) {
            int c = 0;
            oracle_e2m1_encode((double)load_elem(x, dtype, b * 32 + i) / scale, &c);
            codes[i] = (uint8_t)c;
        }
        scales[b] = (uint8_t)(e + 127);
        oracle_pack4(codes, 32, packed + b * 16);
    }
    return ORACLE_OK;
}

int oracle_mxfp4_quantize(const void *x, int dtype, int64_t rows, int64_t cols,
                          uint8_t *packed, uint8_t *scales)
{
    if (cols % 32 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    int64_t n = rows * cols;
    for (int64_t i = 0; i < n; ++i)
        if (!isfinite(load_elem(x, dtype, i)))
            return ORACLE_ERR_NONFINITE;
    int64_t nblocks = n / 32;
    for (int64_t b = 0; b < nblocks; ++b) {
        float ab = 0.0f;
        for (int i = 0; i < 32; ++i) {
            float m = fabsf(load_elem(x, dtype, b * 32 + i));
            if (m > ab)
                ab = m;
        }
        int e = oracle_mx_block_exponent(ab);
        double scale = ldexp(1.0, e);
        uint8_t codes[32];
        for (int i = 0; i < 32; ++i) {
            int c = 0;
            oracle_e2m1_encode((double)load_elem(x, dtype, b * 32 + i) / scale, &c);
            codes[i] = (uint8_t)c;
        }
        scales[b] = (uint8_t)(e + 127);
        oracle_pack4(codes, 32, packed + b * 16);
    }
    return ORACLE_OK;
}

/* MXFP4 dequantisation to fp32: y = p * 2^(c - 127) (exact for every
 * scale a quantiser emits); byte 255 -> NaN. */
void oracle_mxfp4_dequantize(const uint8_t *packed, const uint8_t *scales,
                             int64_t rows, int64_t cols, float *y)
{
    int64_t n = rows * cols;
    for (int64_t i = 0; i < n; ++i) {
        int code = (i & 1) ? packed[i / 2] >> 4 : packed[i / 2] & 15;
        double s = oracle_e8m0_value(scales[i / 32]);
        y[i] = (float)(oracle_e2m1_decode(code) * s);
    }
}

/* ------------------------------------------------------------------ */
/* Scale search ([MATH] S9 Loss(s); [NVMX] S4 max-based vs better scale) */
/* ------------------------------------------------------------------ */

/* Loss of the emitted artefact for one 16-block at scale code sc:
 * sum over i of (x_i - x_hat_i)^2 in double, x_hat the NVFP4 dequantised
 * value of the code the quantiser emits. */
double oracle_nv_block_loss(const float *xb, int sc, float g)
{
    uint8_t codes[16];
    nv_block_codes(xb, 16, sc, g, codes);
    double sb = oracle_e4m3_value(sc);
    double loss = 0.0;
    for (int i = 0; i < 16; ++i) {
        double diff = (double)xb[i] - (double)nv_dequant_value(codes[i], sb, g);
        loss += diff * diff;
    }
    return loss;
}

/* Raw candidate of numerator num over the grid denominator q: the E4M3
 * code nearest to num A_b / (6 q g), the quotient rounded once to double.
 * With num, q <= 2^20 the numerator (<= 44 bits) and the denominator
 * (<= 47 bits) are exact in double. */
int oracle_search_grid_code(float amax_b, float g, int num, int q)
{
    double t = ((double)num * (double)amax_b) / (6.0 * (double)q * (double)g);
    return oracle_e4m3_encode(t);
}

/* Raw candidate k of the fixed grid: m_k = (147 + k) / 210, i.e. the code
 * nearest to (147 + k) A_b / (1260 g) = m_k * A_b / (6 g). */
int oracle_search_candidate_code(float amax_b, float g, int k)
{
    return oracle_search_grid_code(amax_b, g, SEARCH_NUM0 + k, SEARCH_DEN);
}

/* Brute-force search over the n candidates m_k = (p + k) / q, k = 0..n-1,
 * of every block at a given global scale g: the scale with the smallest
 * loss wins, exact ties go to the larger scale.  Emits packed codes, scale
 * codes and (optionally) the winning loss per block.  The fixed search is
 * n = 64, p = 147, q = 210. */
int oracle_nvfp4_scale_search_grid_with_g(const void *x, int dtype, int64_t rows, int64_t cols,
                                          float g, int n, int p, int q, uint8_t *packed,
                                          uint8_t *scales, double *block_loss)
{
    if (cols % 16 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    if (n < 1 || p < 1 || q < 1 || p + (int64_t)n - 1 > (1 << 20) || q > (1 << 20))
        return ORACLE_ERR_ARG;
    int64_t nblocks = rows * cols / 16;
    for (int64_t b = 0; b < nblocks; ++b) {
        float xb[16];
        float ab = 0.0f;
        for (int i = 0; i < 16; ++i) {
            xb[i] = load_elem(x, dtype, b * 16 + i);
            if (!isfinite(xb[i]))
                return ORACLE_ERR_NONFINITE;
            if (fabsf(xb[i]) > ab)
                ab = fabsf(xb[i]);
        }
        int best = -1;
        double best_loss = 0.0;
        for (int k = 0; k < n; ++k) {
            int c = oracle_search_grid_code(ab, g, p + k, q);
            double loss = oracle_nv_block_loss(xb, c, g);
            if (best < 0 || loss < best_loss ||
                (loss == best_loss && oracle_e4m3_value(c) > oracle_e4m3_value(best))) {
                best = c;
                best_loss = loss;
            }
        }
        uint8_t codes[16];
        nv_block_codes(xb, 16, best, g, codes);
        scales[b] = (uint8_t)best;
        oracle_pack4(codes, 16, packed + b * 8);
        if (block_loss)
            block_loss[b] = best_loss;
    }
    return ORACLE_OK;
}

int oracle_nvfp4_scale_search_with_g(const void *x, int dtype, int64_t rows, int64_t cols,
                                     float g, uint8_t *packed, uint8_t *scales,
                                     double *block_loss)
{
    return oracle_nvfp4_scale_search_grid_with_g(x, dtype, rows, cols, g, SEARCH_N, SEARCH_NUM0,
                                                 SEARCH_DEN, packed, scales, block_loss);
}

/* The full search over the grid (n, p, q): tensor amax -> g (as for
 * NVFP4) -> per-block search. */
int oracle_nvfp4_scale_search_grid(const void *x, int dtype, int64_t rows, int64_t cols, int n,
                                   int p, int q, uint8_t *packed, uint8_t *scales, float *g_out,
                                   double *block_loss)
{
    if (cols % 16 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    float amax, g;
    int st = oracle_tensor_amax(x, dtype, rows * cols, &amax);
    if (st)
        return st;
    st = oracle_nv_global_scale(amax, &g);
    if (st)
        return st;
    *g_out = g;
    return oracle_nvfp4_scale_search_grid_with_g(x, dtype, rows, cols, g, n, p, q, packed, scales,
                                                 block_loss);
}

/* The full search: tensor amax -> g (as for NVFP4) -> per-block search. */
int oracle_nvfp4_scale_search(const void *x, int dtype, int64_t rows, int64_t cols,
                              uint8_t *packed, uint8_t *scales, float *g_out,
                              double *block_loss)
{
    if (cols % 16 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    float amax, g;
    int st = oracle_tensor_amax(x, dtype, rows * cols, &amax);
    if (st)
        return st;
    st = oracle_nv_global_scale(amax, &g);
    if (st)
        return st;
    *g_out = g;
    return oracle_nvfp4_scale_search_with_g(x, dtype, rows, cols, g, packed, scales, block_loss);
}

/* NVFP4 "four over six" ([TJ] S4: mapping the block maximum to 4 instead
 * of 6 can place the other values on better grid points; neither rule wins
 * on every block).  Per 16-block the two candidate scales are the E4M3
 * codes nearest to A_b / (6g) (the max-based scale) and A_b / (4g); the
 * second is taken only when its artefact loss is strictly smaller.  g as
 * for NVFP4.  Emits codes, scale codes, g and the chosen loss. */
int oracle_nvfp4_quantize_four_over_six_with_g(const void *x, int dtype, int64_t rows,
                                               int64_t cols, float g, uint8_t *packed,
                                               uint8_t *scales, double *block_loss)
{
    if (cols % 16 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    int64_t nblocks = rows * cols / 16;
    for (int64_t b = 0; b < nblocks; ++b) {
        float xb[16];
        float ab = 0.0f;
        for (int i = 0; i < 16; ++i) {
            xb[i] = load_elem(x, dtype, b * 16 + i);
            if (!isfinite(xb[i]))
                return ORACLE_ERR_NONFINITE;
            if (fabsf(xb[i]) > ab)
                ab = fabsf(xb[i]);
        }
        int c6 = oracle_e4m3_encode((double)ab / (6.0 * (double)g));
        int c4 = oracle_e4m3_encode((double)ab / (4.0 * (double)g));
        double l6 = oracle_nv_block_loss(xb, c6, g);
        double l4 = oracle_nv_block_loss(xb, c4, g);
        int best = l4 < l6 ? c4 : c6;
        uint8_t codes[16];
        nv_block_codes(xb, 16, best, g, codes);
        scales[b] = (uint8_t)best;
        oracle_pack4(codes, 16, packed + b * 8);
        if (block_loss)
            block_loss[b] = l4 < l6 ? l4 : l6;
    }
    return ORACLE_OK;
}

int oracle_nvfp4_quantize_four_over_six(const void *x, int dtype, int64_t rows, int64_t cols,
                                        uint8_t *packed, uint8_t *scales, float *g_out,
                                        double *block_loss)
{
    if (cols % 16 || rows < 0 || cols < 0)
        return ORACLE_ERR_SHAPE;
    float amax, g;
    int st = oracle_tensor_amax(x, dtype, rows * cols, &amax);
    if (st)
        return st;
    st = oracle_nv_global_scale(amax, &g);
    if (st)
        return st;
    *g_out = g;
    return oracle_nvfp4_quantize_four_over_six_with_g(x, dtype, rows, cols, g, packed, scales,
                                                      block_loss);
}

/* Per-block loss of given (packed, scale) artefacts against x, for
 * checking another implementation's choice. */
int oracle_nvfp4_artefact_loss(const void *x, int dtype, int64_t rows, int64_t cols,
                               const uint8_t *packed, const uint8_t *scales, float g,
                               double *block_loss)
{
    if (cols % 16)
        return ORACLE_ERR_SHAPE;
    int64_t nblocks = rows * cols / 16;
    for (int64_t b = 0; b < nblocks; ++b) {
        double sb = oracle_e4m3_decode_byte(scales[b]);
        double loss = 0.0;
        for (int i = 0; i < 16; ++i) {
            int64_t j = b * 16 + i;
            int code = (j & 1) ? packed[j / 2] >> 4 : packed[j / 2] & 15;
            double diff = (double)load_elem(x, dtype, j) - (double)nv_dequant_value(code, sb, g);
            loss += diff * diff;
        }
        block_loss[b] = loss;
    }
    return ORACLE_OK;
}

/* Storage of a complete-block tensor ([NVMX] S8): n/2 payload bytes, one
 * scale byte per block, plus the bytes of any tensor-level scale. */
int64_t oracle_storage_bytes(int64_t elements, int64_t group, int64_t global_bytes)
{
    if (elements <= 0 || (group != 16 && group != 32) || global_bytes < 0 || elements % group)
        return -1;
    return elements / 2 + elements / group + global_bytes;
}

/* ------------------------------------------------------------------ */
/* Ragged rows and the other grouping axis ([NVMX] S6, S7, S8).        */
/* ------------------------------------------------------------------ */

/* Blocks of a row-padded [rows, cols] matrix, B = rows * ceil(cols / G)
 * ([NVMX] S8: padding each row gives this count, not ceil(rows*cols/G)). */
int64_t oracle_padded_blocks(int64_t rows, int64_t cols, int64_t group)
{
    if (rows < 0 || cols < 0 || group <= 0)
        return -1;
    return rows * ((cols + group - 1) / group);
}

/* Storage of a row-padded matrix ([NVMX] S8): B (G/2 + 1) bytes of payload
 * and block scales, plus the bytes of any tensor-level scale. */
int64_t oracle_padded_storage_bytes(int64_t rows, int64_t cols, int64_t group,
                                    int64_t global_bytes)
{
    if ((group != 16 && group != 32) || global_bytes < 0)
        return -1;
    int64_t b = oracle_padded_blocks(rows, cols, group);
    if (b < 0)
        return -1;
    return b * (group / 2 + 1) + global_bytes;
}

/* Pads every row of x [rows, cols] to padded_cols >= cols elements with +0
 * (the pad value is not given on the page; +0 leaves every block maximum as
 * it was).  out holds rows * padded_cols elements of x's type. */
int oracle_pad_rows(const void *x, int dtype, int64_t rows, int64_t cols, int64_t padded_cols,
                    void *out)
{
    if (rows < 0 || cols < 0 || padded_cols < cols || (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < padded_cols; ++c) {
            if (dtype == ORACLE_F32)
                ((float *)out)[r * padded_cols + c] = c < cols ? ((const float *)x)[r * cols + c] : 0.0f;
            else
                ((uint16_t *)out)[r * padded_cols + c] =
                    c < cols ? ((const uint16_t *)x)[r * cols + c] : (uint16_t)0;
        }
    return ORACLE_OK;
}

/* Keeps the first cols of every padded row ([NVMX] S7: decode the padded
 * layout, then cut each row back to the original shape). */
int oracle_crop_rows(const float *y_padded, int64_t rows, int64_t padded_cols, int64_t cols,
                     float *y)
{
    if (rows < 0 || cols < 0 || padded_cols < cols)
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            y[r * cols + c] = y_padded[r * padded_cols + c];
    return ORACLE_OK;
}

/* out [cols, rows] = x [rows, cols] transposed ([NVMX] S6: grouping the
 * transposed matrix by rows groups the original by columns). */
int oracle_transpose(const void *x, int dtype, int64_t rows, int64_t cols, void *out)
{
    if (rows < 0 || cols < 0 || (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            if (dtype == ORACLE_F32)
                ((float *)out)[c * rows + r] = ((const float *)x)[r * cols + c];
            else
                ((uint16_t *)out)[c * rows + r] = ((const uint16_t *)x)[r * cols + c];
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* The consumer of the quantised operands: a block-scaled matrix       */
/* product ([NVMX] S6: Y = X W with both operands blocked along K; the */
/* block scales can only be taken out of the dot product of one block).*/
/* ------------------------------------------------------------------ */

/* D[m][n] = g_a g_b sum over 16-blocks kb of s_a[m][kb] s_b[n][kb]
 * sum_{k in kb} p_a[m][k] p_b[n][k], for A = (packed_a [M, K/2], scales_a
 * [M, K/16] E4M3, g_a) and B = (packed_b [N, K/2], scales_b [N, K/16], g_b),
 * both blocked along K (B is stored N x K, the weight's K-grouping of
 * [NVMX] S6).  Every product p s p s is exact in double, and the block sums
 * are exact; the total is summed in double in k order.  Also returns, per
 * output, the sum of the magnitudes of the terms (for error bounds). */
int oracle_nvfp4_gemm(const uint8_t *packed_a, const uint8_t *scales_a, float g_a,
                      const uint8_t *packed_b, const uint8_t *scales_b, float g_b, int64_t M,
                      int64_t N, int64_t K, double *d, double *mag)
{
    if (M < 0 || N < 0 || K < 0 || K % 16)
        return ORACLE_ERR_SHAPE;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, abs_acc = 0.0;
            for (int64_t kb = 0; kb < K / 16; ++kb) {
                double sa = oracle_e4m3_decode_byte(scales_a[m * (K / 16) + kb]);
                double sb = oracle_e4m3_decode_byte(scales_b[n * (K / 16) + kb]);
                double dot = 0.0, dot_abs = 0.0;
                for (int64_t k = kb * 16; k < kb * 16 + 16; ++k) {
                    int64_t ia = m * K + k, ib = n * K + k;
                    int ca = (ia & 1) ? packed_a[ia / 2] >> 4 : packed_a[ia / 2] & 15;
                    int cb = (ib & 1) ? packed_b[ib / 2] >> 4 : packed_b[ib / 2] & 15;
                    double t = oracle_e2m1_decode(ca) * oracle_e2m1_decode(cb);
                    dot += t;
                    dot_abs += fabs(t);
                }
                acc += sa * sb * dot;
                abs_acc += fabs(sa * sb) * dot_abs;
            }
            d[m * N + n] = acc * (double)g_a * (double)g_b;
            if (mag)
                mag[m * N + n] = abs_acc * fabs((double)g_a * (double)g_b);
        }
    return ORACLE_OK;
}

/* Scale bytes [rows, nb] (one per 16-block, row-major) in the blocked
 * layout the block-scaled tensor-core MMA reads (not on the pages; it is
 * the layout of the sm100 block-scaled MMA's scale factors): rows grouped
 * in tiles of 128, blocks in tiles of 4, tiles in row-tile-major order with
 * the block tiles contiguous; inside a 512-byte tile, row r = r0 + 32 r1
 * (r0 < 32, r1 < 4) and block j (< 4) sit at byte 16 r0 + 4 r1 + j.  Rows
 * and blocks past the matrix hold 0.  out has ceil(rows/128) * 128 *
 * ceil(nb/4) * 4 bytes. */
int oracle_scales_mma_layout(const uint8_t *scales, int64_t rows, int64_t nb, uint8_t *out)
{
    if (rows < 0 || nb < 0)
        return ORACLE_ERR_ARG;
    int64_t rt = (rows + 127) / 128, kt = (nb + 3) / 4;
    memset(out, 0, (size_t)(rt * kt * 512));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < nb; ++j) {
            int64_t tile = (r / 128) * kt + j / 4;
            int64_t rr = r % 128;
            out[tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + j % 4] = scales[r * nb + j];
        }
    return ORACLE_OK;
}
