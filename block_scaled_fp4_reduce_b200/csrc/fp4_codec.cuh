// fp4_codec.cuh -- device-side codecs for block-scaled FP4 (sm_100a).
//
// E2M1 element codes, E4M3 (FN) and E8M0 block scales, and the NVFP4
// element quotient.  Definitions follow "NVFP4 与 MXFP4 格式"
// (charlestar.github.io): section 1 (E2M1 codes, nearest value with ties to
// the even code, saturation at 6, the sign bit kept, even element in the low
// nibble), section 2 (E8M0 2^(c-127), E4M3 max 448 / min subnormal 2^-9),
// section 3 (b* = A_g / (6a) rounded to E4M3 before the elements are
// quantised) and section 5 (OCP rounding-down E8M0 rule).
//
// The file is compiled with -fmad=false: every product and sum below is
// rounded exactly as written; fused multiply-adds appear only as explicit
// fmaf / fma calls.
#pragma once

#include <cstdint>

namespace fp4 {

// ---------------------------------------------------------------------------
// E2M1 encode: eight fp32 values -> eight packed codes in one u32.
// Byte j holds element 2j in its low nibble and 2j+1 in its high nibble.
// `cvt.rn.satfinite.e2m1x2.f32 d, a, b` rounds to nearest even, saturates
// to +-6 and puts `a` in the high nibble, `b` in the low one.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4,
                                           float v5, float v6, float v7)
{
    uint32_t out;
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t"
        "}"
        : "=r"(out)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return out;
}

__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8])
{
    return e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
}

// ---------------------------------------------------------------------------
// E2M1 decode: eight packed codes -> eight fp32 values (code 8 = -0).
// `cvt.rn.f16x2.e2m1x2` widens a byte of two codes to f16x2 exactly (high
// nibble -> high half); the f16 -> f32 widening is exact too.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t packed, uint32_t (&h)[4])
{
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t"
        "}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(packed));
}

__device__ __forceinline__ void f16x2_to_f32(uint32_t h, float &lo, float &hi)
{
    asm("{\n\t"
        ".reg .f16 l, u;\n\t"
        "mov.b32 {l, u}, %2;\n\t"
        "cvt.f32.f16 %0, l;\n\t"
        "cvt.f32.f16 %1, u;\n\t"
        "}"
        : "=f"(lo), "=f"(hi)
        : "r"(h));
}

__device__ __forceinline__ void e2m1x8_decode(uint32_t packed, float (&p)[8])
{
    uint32_t h[4];
    e2m1x8_to_f16x2(packed, h);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        f16x2_to_f32(h[j], p[2 * j], p[2 * j + 1]);
}

// ---------------------------------------------------------------------------
// E4M3 (FN) block scale.
// ---------------------------------------------------------------------------

// Value of an E4M3 byte (sign in bit 7, 0x7F / 0xFF = NaN), exact in fp32.
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte)
{
    uint32_t h;
    uint16_t b = (uint16_t)(byte & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(b));
    float lo, hi;
    f16x2_to_f32(h, lo, hi);
    return lo;
}

// E4M3 code nearest to a finite t >= 0 given in double (ties to the even
// code), after saturation to 448.  The double must be the correctly rounded
// value of the exact rational the scale is defined from: a nonzero distance
// from that rational to an E4M3 midpoint is at least 2^-33 relative (A_b has
// 24 significant bits, the midpoints 5, the divisor 6g at most 27), so one
// double rounding never moves it across or onto a midpoint.
//   t < 2^-6 : subnormal grid, code = rint(t * 2^9)            (0..8)
//   otherwise: t in [2^E, 2^(E+1)), m = rint(t * 2^(3-E)) in [8, 16],
//              code = (E + 6) * 8 + m   (m = 16 carries into the next
//              binade with a zero fraction, which is again the even code)
// rint rounds half to even, and the code's low bit is the low bit of m.
__device__ __forceinline__ uint32_t e4m3_code_from_f64(double t)
{
    if (t >= 448.0)
        return 126u;
    if (t < 0x1p-6)
        return (uint32_t)rint(t * 512.0);
    int E = (int)((__double_as_longlong(t) >> 52) & 0x7FF) - 1023;   // -6 .. 8
    double scale = __longlong_as_double((long long)(1023 + 3 - E) << 52); // 2^(3-E)
    uint32_t m = (uint32_t)rint(t * scale);
    return (uint32_t)((E + 6) * 8) + m;
}

// NVFP4 block-scale code: E4M3 nearest to the exact rational A_b / (6 g).
// Fast path: t = RN(A_b * RN(1/(6g))) is within 2^-23 relative of the
// rational, i.e. a few units in its last place, and `cvt.rn.satfinite.e4m3x2`
// rounds t once to E4M3 (saturating at 448).  Every E4M3 midpoint, and every
// E4M3 value, is an fp32 pattern whose 19 low fraction bits are zero; when t
// lies more than 16 units from such a pattern, t and the rational round to
// the same code.  Otherwise (and never for t < 2^-11, which is always code
// 0) the rational is formed as one correctly rounded double quotient.
__device__ __forceinline__ uint32_t nv_scale_code(float amax_b, float inv6g, double six_g)
{
    float t = __fmul_rn(amax_b, inv6g);
    uint32_t tb = __float_as_uint(t);
    if (tb > 0x3A000000u && ((tb + 16u) & 0x7FFFFu) < 32u)
        return e4m3_code_from_f64(__ddiv_rn((double)amax_b, six_g));
    uint16_t c;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(0.0f), "f"(t));
    return (uint32_t)(c & 0xFFu);
}

// ---------------------------------------------------------------------------
// E8M0 block scale (OCP rounding-down rule): e = floor(log2 A_b) - 2,
// clamped to [-127, 127]; byte = e + 127.  For a finite A_b >= 0 with
// exponent field f: floor(log2 A_b) = f - 127 for normal values, and every
// subnormal or zero A_b clamps to e = -127 (byte 0).  Finite fp32 inputs
// give at most f = 254, i.e. e = 125, so the upper clamp never binds.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e8m0_byte_floor(uint32_t amax_bits)
{
    int f = (int)(amax_bits >> 23);
    return (uint32_t)max(f - 2, 0);
}

// 2^-e as fp32 for the E8M0 byte b = e + 127 (b <= 252 from finite input):
// biased exponent 127 - e = 254 - b, always normal.
__device__ __forceinline__ float e8m0_inverse(uint32_t byte)
{
    return __uint_as_float((254u - byte) << 23);
}

// 2^e as fp32 for any E8M0 byte: 0 -> 2^-127 (subnormal), 255 -> NaN.
__device__ __forceinline__ float e8m0_to_f32(uint32_t byte)
{
    if (byte == 0u)
        return __uint_as_float(0x00400000u);
    if (byte == 255u)
        return __uint_as_float(0x7FC00000u);
    return __uint_as_float(byte << 23);
}

// ---------------------------------------------------------------------------
// NVFP4 element quotient v = fl32(x / d) followed by E2M1 rounding, for
// eight elements sharing d = fl32(s_b * g) > 0.
//
// Bracketing instead of dividing: with r = RN(1/d) (IEEE reciprocal) the
// neighbours r_lo = pred(r) and r_hi = succ(r) satisfy r_lo <= 1/d <= r_hi
// exactly, so x*r_lo and x*r_hi bracket x/d, and since rounding to nearest
// is monotone, RN(x*r_lo) and RN(x*r_hi) bracket v = RN(x/d) in magnitude,
// all three with the sign of x.  The E2M1 code is a monotone function of
// the magnitude, so when both brackets give the same code, v has it too.
// Only when a midpoint of the E2M1 grid falls inside the two-ulp bracket
// (about one element in a million for random data, and exact ties) do the
// eight elements take the IEEE single division.  A d below the smallest
// normal fp32 (1/d could overflow) always takes the division.
// ---------------------------------------------------------------------------
struct NvRecip {
    float d, lo, hi;
    bool exact_only;
};

__device__ __forceinline__ NvRecip nv_recip(float d)
{
    NvRecip q;
    q.d = d;
    q.exact_only = !(d >= 0x1p-126f);
    float r = __frcp_rn(q.exact_only ? 1.0f : d);
    q.lo = __uint_as_float(__float_as_uint(r) - 1u);
    q.hi = __uint_as_float(__float_as_uint(r) + 1u);
    return q;
}

__device__ __forceinline__ uint32_t nv_encode8(const float (&x)[8], const NvRecip &q)
{
    float a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        a[i] = __fmul_rn(x[i], q.lo);
        b[i] = __fmul_rn(x[i], q.hi);
    }
    uint32_t ca = e2m1x8(a);
    uint32_t cb = e2m1x8(b);
    if (ca != cb || q.exact_only) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            a[i] = __fdiv_rn(x[i], q.d);
        ca = e2m1x8(a);
    }
    return ca;
}

// NVFP4 dequantised value fl32(fl32(p * s_b) * g); p * s_b is exact.
__device__ __forceinline__ float nv_dequant(float p, float sb, float g)
{
    return __fmul_rn(__fmul_rn(p, sb), g);
}

// ---------------------------------------------------------------------------
// Loads: eight consecutive input elements as fp32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bf16x8_to_f32(const uint4 &w, float (&x)[8])
{
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[2 * j] = __uint_as_float(ws[j] << 16);
        x[2 * j + 1] = __uint_as_float(ws[j] & 0xFFFF0000u);
    }
}

// max over eight bf16 of the |x| bit pattern, as an fp32 bit pattern.
// Non-negative floats order like their bit patterns; NaN / Inf patterns
// (>= 0x7F80 in bf16) sort above every finite value.
__device__ __forceinline__ uint32_t bf16x8_absmax_bits(const uint4 &w)
{
    uint32_t m = __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                          __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu));
    return max(m & 0xFFFFu, m >> 16) << 16;
}

__device__ __forceinline__ uint32_t f32x4_absmax_bits(const uint4 &w)
{
    return max(max(w.x & 0x7FFFFFFFu, w.y & 0x7FFFFFFFu),
               max(w.z & 0x7FFFFFFFu, w.w & 0x7FFFFFFFu));
}

__device__ __forceinline__ uint4 ldg_stream(const void *p)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Store one 16-byte vector without keeping it in L1 / with streaming hint.
__device__ __forceinline__ void stg_stream(void *p, const uint4 &v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// Eight fp32 -> eight bf16 (round to nearest even) packed in a uint4.
__device__ __forceinline__ uint4 f32x8_to_bf16x8(const float (&y)[8])
{
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
    return make_uint4(o[0], o[1], o[2], o[3]);
}

} // namespace fp4
