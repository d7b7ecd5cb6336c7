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
// to +-6 and puts `a` in the high nibble, `b` in the low one; the four bytes
// are packed with one vector move.
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
// `cvt.rn.f16x2.e2m1x2` widens one byte of two codes to f16x2 exactly (high
// nibble -> high half); the f16 -> f32 widening is exact too.  Each byte is
// shifted down in a 32-bit register and narrowed on its own (cvt.u8.u32):
// unpacking a word with one vector move into four 8-bit registers straight
// after the encoder packed it was seen to return wrong upper bytes.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low_bits)
{
    uint32_t h;
    asm("{\n\t"
        ".reg .b8 q;\n\t"
        "cvt.u8.u32 q, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, q;\n\t"
        "}"
        : "=r"(h)
        : "r"(byte_in_low_bits));
    return h;
}

__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t packed, uint32_t (&h)[4])
{
#pragma unroll
    for (int j = 0; j < 4; ++j)
        h[j] = e2m1x2_to_f16x2(packed >> (8 * j));
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

// Round eight fp32 values to the E2M1 grid and return the grid values
// (quantise-dequantise), each pair converted to codes and back inside one
// asm block so that the codes never leave their 8-bit registers: the codes
// are not needed, and a packed word built from `cvt ... e2m1x2` results that
// is unpacked again straight away was seen to lose its upper two bytes.
__device__ __forceinline__ void e2m1x8_qdq(const float (&v)[8], float (&p)[8])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t h;
        asm("{\n\t"
            ".reg .b8 q;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 q, %2, %1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, q;\n\t"
            "}"
            : "=r"(h)
            : "f"(v[2 * j]), "f"(v[2 * j + 1]));
        f16x2_to_f32(h, p[2 * j], p[2 * j + 1]);
    }
}

// Rounding error of eight fp32 values on the E2M1 grid: e[i] = p_i - v[i]
// (p_i the grid value of v[i]), each pair rounded to codes, widened to f16
// and subtracted from the fp32 value by the mixed-precision
// `sub.rn.f32.f16` (sm_100) inside one asm block.  One rounding per
// element, so |e| is the magnitude of the correctly rounded v - p.
__device__ __forceinline__ void e2m1x8_error(const float (&v)[8], float (&e)[8])
{
#pragma unroll
    for (int j = 0; j < 4; ++j)
        asm("{\n\t"
            ".reg .b8 q;\n\t"
            ".reg .b32 h;\n\t"
            ".reg .b16 l, u;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 q, %3, %2;\n\t"
            "cvt.rn.f16x2.e2m1x2 h, q;\n\t"
            "mov.b32 {l, u}, h;\n\t"
            "sub.rn.f32.f16 %0, l, %2;\n\t"
            "sub.rn.f32.f16 %1, u, %3;\n\t"
            "}"
            : "=f"(e[2 * j]), "=f"(e[2 * j + 1])
            : "f"(v[2 * j]), "f"(v[2 * j + 1]));
}

// sqrt.approx.f32: relative error below 2^-21 (for bounds only).
__device__ __forceinline__ float sqrt_approx(float x)
{
    float r;
    asm("sqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
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

// Block-scale code: E4M3 nearest to the exact rational num * A_b / den
// (NVFP4: num = 1, den = 6g; the search's smallest candidate: num = 147,
// den = 1260 g), given inv = RN32(num / den).
// Fast path: t = RN(A_b * inv) is within 2^-23 relative of the rational, a
// few units in its last place, and `cvt.rn.satfinite.e4m3x2` rounds t once
// to E4M3 (saturating at 448).  Every E4M3 midpoint, and every E4M3 value,
// is an fp32 pattern whose 19 low fraction bits are zero; when t lies more
// than 16 units from such a pattern, t and the rational round to the same
// code.  Otherwise (never for t < 2^-11, which is always code 0) the rational
// is formed as one correctly rounded double quotient (num * A_b and den are
// exact in double).
__device__ __forceinline__ uint32_t e4m3_rn(float t)
{
    uint16_t c;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(0.0f), "f"(t));
    return (uint32_t)(c & 0xFFu);
}

__device__ __forceinline__ uint32_t nv_scale_code(float amax_b, float inv, double num, double den)
{
    const float t = __fmul_rn(amax_b, inv);
    const uint32_t tb = __float_as_uint(t);
    if (tb > 0x3A000000u && ((tb + 16u) & 0x7FFFFu) < 32u)
        return e4m3_code_from_f64(__ddiv_rn(num * (double)amax_b, den));
    return e4m3_rn(t);
}

// The same for t = amax_b / (m g) with m = 6 (the max-based scale) or 4,
// inv = RN32(1 / (m g)), den = m g (exact in double), without the double
// division where t lies near a grid point P with five significant bits in
// the normal E4M3 range.  An E4M3 value P: t is within 18 ulps of it and
// 2^19 ulps from either midpoint, so the conversion of t is right.  A
// midpoint P: the sign of amax_b - P m g decides exactly -- P m is exact
// (eight significant bits), P m g = hi + lo exactly (one fma), amax_b - hi
// is exact (Sterbenz: amax_b is within 2^-18 of hi) -- and an exact tie
// takes the even code.  The double path rounds the quotient to double
// first, which makes no false tie: a nonzero amax_b - P m g is at least
// ~2^-31 of it, far above double's 2^-53.
__device__ __forceinline__ uint32_t nv_scale_code_mg(float amax_b, float inv, float g, float m, double den)
{
    const float t = __fmul_rn(amax_b, inv);
    const uint32_t tb = __float_as_uint(t);
    if (tb > 0x3A000000u && ((tb + 16u) & 0x7FFFFu) < 32u) {
        const uint32_t pb = (tb + 16u) & ~0x7FFFFu;
        const float P = __uint_as_float(pb);
        if (P >= 0x1p-6f && g >= 0x1p-100f) {
            if (!(pb & 0x80000u) && P <= 448.0f)
                return e4m3_rn(t);
            if ((pb & 0x80000u) && P < 448.0f) {
                const float pm = __fmul_rn(P, m);
                const float hi = __fmul_rn(pm, g);
                const float lo = __fmaf_rn(pm, g, -hi);
                const float d = __fsub_rn(amax_b, hi);
                const uint32_t c_lo = e4m3_rn(__uint_as_float(pb & ~0x80000u));
                if (d > lo)
                    return c_lo + 1u;
                if (d < lo)
                    return c_lo;
                return c_lo + (c_lo & 1u);
            }
        }
        return e4m3_code_from_f64(__ddiv_rn((double)amax_b, den));
    }
    return e4m3_rn(t);
}

// Value of an E4M3 byte as f16 bits: every E4M3 value (2^-9 .. 448, NaN)
// is exact in f16.
__device__ __forceinline__ uint16_t e4m3_to_f16(uint32_t byte)
{
    uint16_t r;
    const uint16_t b = (uint16_t)(byte & 0xFFu);
    asm("{\n\t"
        ".reg .b32 h;\n\t"
        ".reg .b16 u;\n\t"
        "cvt.rn.f16x2.e4m3x2 h, %1;\n\t"
        "mov.b32 {%0, u}, h;\n\t"
        "}"
        : "=h"(r)
        : "h"(b));
    return r;
}

// Value of a positive E4M3 code 0..126 as fp32 (exact): the E4M3 -> f16
// conversion, then f16 -> fp32.
__device__ __forceinline__ float e4m3_pos_to_f32(uint32_t c)
{
    float r;
    asm("cvt.f32.f16 %0, %1;" : "=f"(r) : "h"(e4m3_to_f16(c)));
    return r;
}

// The two f16 halves of h, each times the f16 s, as fp32 with one rounding
// (mixed-precision `fma.rn.f32.f16`, sm_100): a * s + (-0).  Adding -0 keeps
// the sign of a zero product and changes nothing else.
__device__ __forceinline__ void f16x2_mul_f16_to_f32(uint32_t h, uint16_t s, float &lo, float &hi)
{
    asm("{\n\t"
        ".reg .b16 l, u;\n\t"
        "mov.b32 {l, u}, %2;\n\t"
        "fma.rn.f32.f16 %0, l, %3, 0f80000000;\n\t"
        "fma.rn.f32.f16 %1, u, %3, 0f80000000;\n\t"
        "}"
        : "=f"(lo), "=f"(hi)
        : "r"(h), "h"(s));
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

// E8M0 block scale, ceil rule (the NVFP4/MXFP4 format page's `mx_scale`,
// ModelOpt-style 2^ceil(log2(A_b/6))): an all-zero block gets e = 0 (scale
// 1); otherwise e = max(E - 3, -127) with A_b = m 2^E, m in [0.5, 1), then
// e + 1 if A_b > 6 * 2^e, so that A_b never exceeds 6 * 2^e.  For finite
// fp32 input E <= 128, so e <= 126 and the E8M0 range is never exceeded.
__device__ __forceinline__ uint32_t e8m0_byte_ceil(uint32_t amax_bits)
{
    if (amax_bits == 0u)
        return 127u;
    const int E = amax_bits >= 0x00800000u ? (int)(amax_bits >> 23) - 126
                                           : (32 - __clz((int)amax_bits)) - 149;
    int e = max(E - 3, -127);
    const float p2 = e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23)
                               : __uint_as_float(0x00400000u); // 2^-127
    if (__uint_as_float(amax_bits) > __fmul_rn(6.0f, p2))
        ++e;
    return (uint32_t)(e + 127);
}

// 2^-e as fp32 for the E8M0 byte b = e + 127 (b <= 253 from finite input):
// biased exponent 127 - e = 254 - b, always normal.
__device__ __forceinline__ float e8m0_inverse(uint32_t byte)
{
    return __uint_as_float((254u - byte) << 23);
}

// 2^e as f16 bits for an E8M0 byte b = e + 127 with -24 <= e <= 15:
// normal 2^e (e >= -14) has exponent field e + 15; below that the
// subnormal 2^e = 2^(e + 24) units of 2^-24.
__device__ __forceinline__ uint16_t e8m0_to_f16(uint32_t byte)
{
    const int e = (int)byte - 127;
    return e >= -14 ? (uint16_t)((e + 15) << 10) : (uint16_t)(1u << (e + 24));
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
// Bracketing instead of dividing: with r_lo <= 1/d <= r_hi (exact reals,
// see nv_recip), x*r_lo and x*r_hi bracket x/d, and since rounding to
// nearest is monotone, RN(x*r_lo) and RN(x*r_hi) bracket v = RN(x/d) in
// magnitude, all three with the sign of x.  The E2M1 code is a monotone
// function of the magnitude, so when both brackets give the same code, v
// has it too.  Only when a midpoint of the E2M1 grid falls inside the
// eight-ulp bracket (a few elements in a million for random data, and exact
// ties) do the eight elements take the IEEE single division.  A d below the
// smallest normal fp32 always takes the division.
// ---------------------------------------------------------------------------
struct NvRecip {
    float d, lo, hi;
    bool exact_only;
};

__device__ __forceinline__ float rcp_approx(float d)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

// Reciprocal bracket of d.  r0 = rcp.approx(d) has a relative error far
// below 2^-12; one Newton step r1 = r0 + r0 (1 - d r0) (two FMAs) leaves
// |r1 d - 1| <= delta^2 + delta u + u < 2^-23 (u = 2^-24), i.e. at most two
// units in the last place of r1, four bit patterns when 1/d sits just below a
// power of two.  So r1 - 4 and r1 + 4 (as bit patterns) bracket 1/d exactly.
// d is normal here (>= 2^-126) and at most 2^125.5 (448 g, g <= FLT_MAX/2688),
// so 1/d and its neighbours are normal.
__device__ __forceinline__ NvRecip nv_recip(float d)
{
    NvRecip q;
    q.d = d;
    q.exact_only = !(d >= 0x1p-126f);
    const float dd = q.exact_only ? 1.0f : d;
    const float r0 = rcp_approx(dd);
    const float e = fmaf(-dd, r0, 1.0f);
    const float r1 = fmaf(r0, e, r0);
    q.lo = __uint_as_float(__float_as_uint(r1) - 4u);
    q.hi = __uint_as_float(__float_as_uint(r1) + 4u);
    return q;
}

// Packed fp32 pairs (sm_100): two IEEE single operations, each rounded to
// nearest, per instruction.  pack2 / unpack2 only name a register pair.
__device__ __forceinline__ uint64_t pack2(float lo, float hi)
{
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}

__device__ __forceinline__ void unpack2(uint64_t d, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}

__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// The bracket step alone: the codes of RN(x r_lo), and `exact` set when
// they are not known to be v's (the brackets' codes differ, or d is
// subnormal), i.e. when the eight IEEE quotients are needed.
__device__ __forceinline__ uint32_t nv_bracket8(const float (&x)[8], const NvRecip &q, bool &exact)
{
    float a[8], b[8];
    const uint64_t rlo = pack2(q.lo, q.lo), rhi = pack2(q.hi, q.hi);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint64_t xp = pack2(x[2 * j], x[2 * j + 1]);
        unpack2(mul2(xp, rlo), a[2 * j], a[2 * j + 1]);
        unpack2(mul2(xp, rhi), b[2 * j], b[2 * j + 1]);
    }
    const uint32_t ca = e2m1x8(a);
    const uint32_t cb = e2m1x8(b);
    exact = ca != cb || q.exact_only;
    return ca;
}

// E2M1 code (low nibble) of one value.
__device__ __forceinline__ uint32_t e2m1_nibble(float v)
{
    uint32_t out;
    asm("{\n\t"
        ".reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\t"
        "cvt.u32.u8 %0, b;\n\t"
        "}"
        : "=r"(out)
        : "f"(v), "f"(0.0f));
    return out & 15u;
}

__device__ __forceinline__ uint32_t nv_encode8(const float (&x)[8], const NvRecip &q)
{
    bool exact;
    uint32_t c = nv_bracket8(x, q, exact);
    if (exact) {
        float a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            a[i] = __fdiv_rn(x[i], q.d);
        c = e2m1x8(a);
    }
    return c;
}

// NVFP4 dequantised value fl32(fl32(p * s_b) * g); p * s_b is exact.
__device__ __forceinline__ float nv_dequant(float p, float sb, float g)
{
    return __fmul_rn(__fmul_rn(p, sb), g);
}

// ---------------------------------------------------------------------------
// 32-byte (256-bit) vector load / store, sm_100 and later.  Loads are
// cached in L2 only (.cg): data is streamed once, and with launch chaining a
// kernel may start while its predecessor still runs, so inputs are never
// read through the non-coherent path.
__device__ __forceinline__ void ldg_v8(const void *p, uint32_t *w)
{
    asm volatile("ld.global.cg.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
          "=r"(w[7])
        : "l"(p));
}

__device__ __forceinline__ void stg_v8(void *p, const uint32_t *w)
{
    asm volatile("st.global.cs.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                 "r"(w[7])
                 : "memory");
}

} // namespace fp4
