// fp4_kernels.cuh -- sm_100a kernels of the block-scaled FP4 path.
//
//   amax_kernel           tensor amax ("NVFP4 与 MXFP4 格式" section 3: A, the
//                         tensor absolute maximum): per-CTA maxima, folded by
//                         the last CTA to finish, in one launch
//   nvfp4_quantize_kernel block amax, E4M3 scale, element quotient, E2M1
//                         rounding and nibble packing in one pass (section 3)
//   mxfp4_quantize_kernel the same for 32-blocks with an E8M0 scale (section 5;
//                         OCP rounding-down rule, or the page's ceil rule)
//   dequantize_kernel     x_hat = q * s_b * g (NVFP4) or q * 2^e (MXFP4)
//   scale_search_kernel   per-block MSE-minimising E4M3 scale
//                         ("FP4 / NVFP4 数学总结" section 9)
//
// Layout of the work: one thread owns one whole block (16 elements for
// NVFP4 and the search, 32 for MXFP4) and reads it with 256-bit loads
// (`ld.global.cg.v8`, new on sm_100), so consecutive lanes
// read consecutive 32-byte sectors and every per-block step (amax, scale,
// reciprocal) runs once per block.  Grids are persistent: SMs x resident
// CTAs, grid-striding over the blocks, two blocks in flight per thread.
// Everything is HBM-bound streaming except the scale search (issue-bound).
//
// Launch chaining: every kernel is launched with programmatic stream
// serialisation and waits for the previous kernel on the stream
// (griddepcontrol.wait) before its first global memory access.  No kernel
// triggers its dependents early (griddepcontrol.launch_dependents): the
// persistent grids here leave room on the SMs, and a dependent grid launched
// at the start of its predecessor parks CTAs there for the predecessor's
// whole run, which measured slower -- 18.1 against 16.0 ms per step on the
// 7B weight set, 79.5 against 72.4 us on the 4096 x 4096 weight.  The
// dependent grid is launched as the previous one's CTAs exit.  Loads after
// the wait go through L2 (.cg / coherent), never the non-coherent path.
#pragma once

#include <cstdint>

#include "fp4_codec.cuh"

namespace fp4 {

constexpr int kThreads = 256;
constexpr int kMaxPartials = 1024;
constexpr uint32_t kNonFiniteBits = 0x7F800000u;

// Status values written to the caller's device status word (fp4.h).
constexpr int32_t kStatusNonFinite = 4;
constexpr int32_t kStatusRange = 5;

__device__ __forceinline__ void raise_status(int32_t *status, int32_t code)
{
    atomicCAS(status, 0, code);
}

// Max of one value over the CTA (all threads must call; result broadcast).
__device__ __forceinline__ uint32_t cta_max_u32(uint32_t v)
{
    __shared__ uint32_t s_part[kThreads / 32];
    __shared__ uint32_t s_res;
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        s_part[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < (int)(blockDim.x >> 5) ? s_part[lane] : 0u;
        w = __reduce_max_sync(0xFFFFFFFFu, w);
        if (lane == 0)
            s_res = w;
    }
    __syncthreads();
    return s_res;
}

// ---------------------------------------------------------------------------
// A block of N input elements of type T (float, or uint16_t = bf16 bits) as
// raw 32-bit words, loaded with 256-bit vectors.
// ---------------------------------------------------------------------------
template <typename T, int N> struct Blk {
    static constexpr int kWords = N * (int)sizeof(T) / 4;
    static_assert(kWords % 8 == 0, "blocks are whole 32-byte vectors");
    uint32_t w[kWords];
};

template <typename T, int N, typename I>
__device__ __forceinline__ void load_blk(const T *x, I b, Blk<T, N> &k)
{
    const char *p = reinterpret_cast<const char *>(x) + (int64_t)b * (int64_t)(N * sizeof(T));
#pragma unroll
    for (int j = 0; j < Blk<T, N>::kWords; j += 8)
        ldg_v8(p + 4 * j, &k.w[j]);
}

// max |x| over the block as an fp32 bit pattern, with packed
// `max.NaN.xorsign.abs` (sm_86+): the magnitude of the result is the larger
// magnitude, its sign is garbage and masked off at the end; a NaN operand
// makes the result NaN.  bf16 pairs take one instruction per two elements.
// Finite values order like their bit patterns, and NaN / Inf patterns sort
// above every finite value.
template <typename T, int N>
__device__ __forceinline__ uint32_t absmax_bits(const Blk<T, N> &k)
{
    constexpr int W = Blk<T, N>::kWords;
    uint32_t m[W];
#pragma unroll
    for (int j = 0; j < W; ++j)
        m[j] = k.w[j];
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int s = W / 2; s >= 1; s /= 2)
#pragma unroll
            for (int j = 0; j < s; ++j)
                asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[j]) : "r"(m[j]), "r"(m[j + s]));
        uint32_t r;
        asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;"
            : "=r"(r)
            : "r"(m[0]), "r"(__funnelshift_l(m[0], m[0], 16)));
        return r & 0x7FFF0000u;
    } else {
#pragma unroll
        for (int s = W / 2; s >= 1; s /= 2)
#pragma unroll
            for (int j = 0; j < s; ++j)
                asm("max.NaN.xorsign.abs.f32 %0, %1, %2;" : "=r"(m[j]) : "r"(m[j]), "r"(m[j + s]));
        return m[0] & 0x7FFFFFFFu;
    }
}

// Element i of the block as fp32 (exact).
template <typename T, int N>
__device__ __forceinline__ float elem(const Blk<T, N> &k, int i)
{
    if constexpr (sizeof(T) == 2)
        return __uint_as_float((i & 1) ? (k.w[i >> 1] & 0xFFFF0000u) : (k.w[i >> 1] << 16));
    else
        return __uint_as_float(k.w[i]);
}

template <typename T, int N>
__device__ __forceinline__ void elems8(const Blk<T, N> &k, int first, float (&x)[8])
{
#pragma unroll
    for (int i = 0; i < 8; ++i)
        x[i] = elem(k, first + i);
}

// Grid-stride loop over n units with U units in flight per thread: `load(u,
// i)` for all U units first, then `work(u, i)`, so that U loads are
// outstanding together.  The main loop runs unguarded over whole groups of
// U; the remaining units go one at a time.  Indices are 32-bit (the host
// splits larger problems into chunks below 2^30 units), so every address is
// one wide multiply-add.
template <int U, typename Load, typename Work>
__device__ __forceinline__ void stream_units(int n, Load &&load, Work &&work)
{
    const int stride = (int)(gridDim.x * blockDim.x);
    int i = (int)(blockIdx.x * blockDim.x + threadIdx.x);
    for (; i + (U - 1) * stride < n; i += U * stride) {
#pragma unroll
        for (int u = 0; u < U; ++u)
            load(u, i + u * stride);
#pragma unroll
        for (int u = 0; u < U; ++u)
            work(u, i + u * stride);
    }
    for (; i < n; i += stride) {
        load(0, i);
        work(0, i);
    }
}

// As stream_units, but the main loop's condition is taken for the warp's
// last lane, so that all 32 lanes run it together (its body may use warp
// collectives): `whole(i, stride)` takes units i + u * stride, u < U; the
// units left over go one at a time to `one(i)`.
template <int U, typename Whole, typename One>
__device__ __forceinline__ void stream_units_warp(int n, Whole &&whole, One &&one)
{
    const int stride = (int)(gridDim.x * blockDim.x);
    const int to_last_lane = 31 - (int)(threadIdx.x & 31u);
    int i = (int)(blockIdx.x * blockDim.x + threadIdx.x);
    for (; i + to_last_lane + (U - 1) * stride < n; i += U * stride)
        whole(i, stride);
    for (; i < n; i += stride)
        one(i);
}

// Largest unit count one launch of a stream_units kernel takes.
constexpr int64_t kMaxUnitsPerLaunch = (int64_t)1 << 30;

__device__ __forceinline__ void pdl_begin()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Tensor amax in one launch.  Each CTA writes the max |x| bit pattern of its
// share to ws[blockIdx.x]; the last CTA to finish (counted with a wrapping
// atomicInc on ws[kMaxPartials], which returns to 0 after every launch)
// folds the partials and writes A as fp32 to *amax (NaN / Inf flags
// FP4_ERR_NONFINITE).  32-byte loads, four in flight per thread.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
    amax_kernel(const T *__restrict__ x, int64_t n, uint32_t *ws, float *amax, int32_t *status)
{
    pdl_begin();
    constexpr int kPerVec = 32 / (int)sizeof(T);
    constexpr int kUnroll = 4;
    const int64_t nvec = n / kPerVec;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t m = 0;
    for (; i + (kUnroll - 1) * stride < nvec; i += kUnroll * stride) {
        Blk<T, kPerVec> v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            load_blk(x, i + u * stride, v[u]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            m = max(m, absmax_bits(v[u]));
    }
    for (; i < nvec; i += stride) {
        Blk<T, kPerVec> v;
        load_blk(x, i, v);
        m = max(m, absmax_bits(v));
    }
    if (blockIdx.x == 0) { // elements past the last whole 32-byte vector
        for (int64_t j = nvec * kPerVec + threadIdx.x; j < n; j += blockDim.x) {
            uint32_t b;
            if constexpr (sizeof(T) == 2)
                b = ((uint32_t)__ldcg(x + j) & 0x7FFFu) << 16;
            else
                b = __float_as_uint(__ldcg(x + j)) & 0x7FFFFFFFu;
            m = max(m, b);
        }
    }
    m = cta_max_u32(m);
    __shared__ bool s_last;
    if (threadIdx.x == 0) {
        ws[blockIdx.x] = m;
        __threadfence();
        s_last = atomicInc(&ws[kMaxPartials], gridDim.x - 1) == gridDim.x - 1;
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        uint32_t a = 0;
        for (int k = threadIdx.x; k < (int)gridDim.x; k += blockDim.x)
            a = max(a, __ldcg(ws + k));
        a = cta_max_u32(a);
        if (threadIdx.x == 0) {
            *amax = __uint_as_float(a);
            if (a >= kNonFiniteBits)
                raise_status(status, kStatusNonFinite);
        }
    }
}

// The NVFP4 global scale from the amax bit pattern: g = fl32(A / 2688),
// A = 0 -> 1.  Returns 0 and sets err for a non-finite A or a g below the
// smallest normal fp32.
__device__ __forceinline__ float nv_global_scale(uint32_t amax_bits, int32_t &err)
{
    err = 0;
    if (amax_bits >= kNonFiniteBits) {
        err = kStatusNonFinite;
        return 0.0f;
    }
    if (amax_bits == 0u)
        return 1.0f;
    float g = __fdiv_rn(__uint_as_float(amax_bits), 2688.0f);
    if (!(g >= 0x1p-126f)) {
        err = kStatusRange;
        return 0.0f;
    }
    return g;
}

// Prologue shared by the NVFP4 quantiser and the scale search: read the
// tensor amax, derive g, publish g / the error from thread 0 of CTA 0.
// Returns false when the kernel must stop (data error).
__device__ __forceinline__ bool nv_prologue(const float *amax, float *global_scale,
                                            int32_t *status, float &g)
{
    int32_t err;
    g = nv_global_scale(__float_as_uint(__ldcg(amax)) & 0x7FFFFFFFu, err);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (err)
            raise_status(status, err);
        else
            *global_scale = g;
    }
    return err == 0;
}

// Per-CTA constants of the NVFP4 block-scale rounding.
struct NvScaleConsts {
    float g;
    float inv6g;  // RN32(1 / (6 g))
    double six_g; // 6 g, exact in double
};

__device__ __forceinline__ NvScaleConsts nv_scale_consts(float g)
{
    NvScaleConsts c;
    c.g = g;
    c.six_g = 6.0 * (double)g;
    c.inv6g = (float)(1.0 / c.six_g);
    return c;
}

// Exact NVFP4 codes of a 16-block at positive scale code c (zero scale ->
// zero codes): v = fl32(x / fl32(s_b g)), E2M1.
template <typename T>
__device__ __forceinline__ uint2 nv_block_codes(const Blk<T, 16> &b, uint32_t c, float g)
{
    if (c == 0u)
        return make_uint2(0u, 0u);
    const NvRecip q = nv_recip(__fmul_rn(e4m3_pos_to_f32(c), g));
    float h[8];
    uint2 pk;
    elems8(b, 0, h);
    pk.x = nv_encode8(h, q);
    elems8(b, 8, h);
    pk.y = nv_encode8(h, q);
    return pk;
}

// ---------------------------------------------------------------------------
// NVFP4 quantise + pack.  One thread per 16-element block: one 32-byte load
// (bf16) or two (fp32), one 8-byte packed store, one scale byte.
// ---------------------------------------------------------------------------
// NVFP4 codes and scale byte of one loaded 16-block under the global scale
// g (constants sc): written to *packed / *scale.
template <typename T>
__device__ __forceinline__ uint2 nv_block_quantize(const Blk<T, 16> &blk, const NvScaleConsts &sc,
                                                   uint32_t &code)
{
    const float amax_b = __uint_as_float(absmax_bits(blk));
    code = nv_scale_code_mg(amax_b, sc.inv6g, sc.g, 6.0f, sc.six_g);
    return nv_block_codes(blk, code, sc.g);
}

template <typename T>
__device__ __forceinline__ void nv_quantize_block(const Blk<T, 16> &blk, const NvScaleConsts &sc,
                                                  uint2 *packed, uint8_t *scale)
{
    uint32_t code;
    *packed = nv_block_quantize(blk, sc, code);
    *scale = (uint8_t)code;
}

// ---------------------------------------------------------------------------
// Warp-shared exact path (bf16 input).  A half-block whose bracket does not
// settle its codes (nv_bracket8) needs its eight IEEE quotients x / d.  Done
// by its own thread, the eight divisions run while the warp's other lanes
// wait, and on tie-rich data (bf16 weights, where an element is often the
// tensor amax times a power of two and a block scale of significand 1.5 or
// 1.75 puts x / d on an E2M1 midpoint) about half the warps meet such a
// half-block at every step.  Here the U blocks of every lane are first
// bracketed; flagged half-blocks go to a per-warp queue in shared memory
// (their eight elements and d); then the whole warp works the queue off with
// one element per lane (eight lanes per half-block, four half-blocks per
// pass, the nibbles gathered by three shuffles), and each owner reads its
// code word back.  The codes are those of the per-thread path bit for bit:
// the same quotients, the same conversion.  All 32 lanes of the warp must
// call it together.
// ---------------------------------------------------------------------------
template <int U> struct NvExactQueue {
    static constexpr int kCap = 32 * 2 * U; // every half-block of the warp
    uint4 x[kCap];     // the eight bf16 elements
    uint32_t d[kCap];  // bits of d = fl32(s_b g); after the pass, the code word
};

template <int U>
__device__ __forceinline__ void nv_quantize_warp(const Blk<uint16_t, 16> (&blk)[U],
                                                 const NvScaleConsts &sc, NvExactQueue<U> &q,
                                                 uint2 (&pk)[U], uint32_t (&code)[U])
{
    const int lane = (int)(threadIdx.x & 31u);
    const uint32_t below = (1u << lane) - 1u;
    int count = 0;
    uint32_t cw[U][2];
    int slot[U][2];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const float amax_b = __uint_as_float(absmax_bits(blk[u]));
        code[u] = nv_scale_code_mg(amax_b, sc.inv6g, sc.g, 6.0f, sc.six_g);
        const NvRecip r = nv_recip(__fmul_rn(e4m3_pos_to_f32(code[u]), sc.g));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float x[8];
            elems8(blk[u], 8 * h, x);
            bool exact;
            cw[u][h] = nv_bracket8(x, r, exact);
            exact = exact && code[u] != 0u; // a zero scale gives zero codes
            slot[u][h] = -1;
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, exact);
            if (m) {
                if (exact) {
                    const int s = count + __popc(m & below);
                    q.x[s] = make_uint4(blk[u].w[4 * h], blk[u].w[4 * h + 1], blk[u].w[4 * h + 2],
                                        blk[u].w[4 * h + 3]);
                    q.d[s] = __float_as_uint(r.d);
                    slot[u][h] = s;
                }
                count += __popc(m);
            }
        }
    }
    if (count) {
        __syncwarp();
        const int i = lane & 7;
        for (int q0 = 0; q0 < count; q0 += 4) {
            const int s = q0 + (lane >> 3);
            uint32_t nib = 0;
            if (s < count) {
                const uint32_t w = reinterpret_cast<const uint32_t *>(&q.x[s])[i >> 1];
                const float xv = __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
                nib = e2m1_nibble(__fdiv_rn(xv, __uint_as_float(q.d[s]))) << (4 * i);
            }
            nib |= __shfl_xor_sync(0xFFFFFFFFu, nib, 1);
            nib |= __shfl_xor_sync(0xFFFFFFFFu, nib, 2);
            nib |= __shfl_xor_sync(0xFFFFFFFFu, nib, 4);
            if (i == 0 && s < count)
                q.d[s] = nib;
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                if (slot[u][h] >= 0)
                    cw[u][h] = q.d[slot[u][h]];
        __syncwarp();
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
        pk[u] = code[u] ? make_uint2(cw[u][0], cw[u][1]) : make_uint2(0u, 0u);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
    nvfp4_quantize_kernel(const T *__restrict__ x, int n_blocks, const float *amax,
                          uint2 *__restrict__ packed, uint8_t *__restrict__ scales,
                          float *global_scale, int32_t *status)
{
    pdl_begin();
    float g;
    if (!nv_prologue(amax, global_scale, status, g))
        return;
    const NvScaleConsts sc = nv_scale_consts(g);
    if constexpr (sizeof(T) == 2) {
        constexpr int U = 3; // 16-blocks per thread per step (fastest of 2-4 on bf16 weights)
        __shared__ NvExactQueue<U> queues[kThreads / 32];
        NvExactQueue<U> &q = queues[threadIdx.x >> 5];
        stream_units_warp<U>(
            n_blocks,
            [&](int b0, int stride) {
                Blk<T, 16> blk[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    load_blk(x, b0 + u * stride, blk[u]);
                uint2 pk[U];
                uint32_t code[U];
                nv_quantize_warp(blk, sc, q, pk, code);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    packed[b0 + u * stride] = pk[u];
                    scales[b0 + u * stride] = (uint8_t)code[u];
                }
            },
            [&](int b) {
                Blk<T, 16> blk;
                load_blk(x, b, blk);
                nv_quantize_block(blk, sc, packed + b, scales + b);
            });
    } else {
        constexpr int U = 4;
        Blk<T, 16> blk[U];
        stream_units<U>(
            n_blocks, [&](int u, int b) { load_blk(x, b, blk[u]); },
            [&](int u, int b) { nv_quantize_block(blk[u], sc, packed + b, scales + b); });
    }
}

// ---------------------------------------------------------------------------
// MXFP4 quantise + pack.  One thread per 32-element block: two 32-byte loads
// (bf16) or four (fp32), one 16-byte packed store, one scale byte.  kCeil
// selects the ceil scale rule instead of the OCP rounding-down one.  The
// scaling x 2^-e is exact, so it runs as packed pair multiplies.  A block
// with a NaN or Inf sets *bad.
// ---------------------------------------------------------------------------
template <bool kCeil, typename T>
__device__ __forceinline__ void mx_quantize_block(const Blk<T, 32> &blk, uint4 *packed,
                                                  uint8_t *scale, bool &bad)
{
    const uint32_t ab = absmax_bits(blk);
    bad |= ab >= kNonFiniteBits;
    const uint32_t byte = kCeil ? e8m0_byte_ceil(ab) : e8m0_byte_floor(ab);
    const float inv = e8m0_inverse(byte);
    const uint64_t inv2 = pack2(inv, inv);
    uint32_t pk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            unpack2(mul2(pack2(elem(blk, 8 * j + 2 * i), elem(blk, 8 * j + 2 * i + 1)), inv2),
                    v[2 * i], v[2 * i + 1]);
        pk[j] = e2m1x8(v);
    }
    *packed = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    *scale = (uint8_t)byte;
}

template <typename T, bool kCeil = false>
__global__ void __launch_bounds__(kThreads)
    mxfp4_quantize_kernel(const T *__restrict__ x, int n_blocks, uint4 *__restrict__ packed,
                          uint8_t *__restrict__ scales, int32_t *status)
{
    pdl_begin();
    bool bad = false;
    Blk<T, 32> blk[2];
    stream_units<2>(
        n_blocks, [&](int u, int b) { load_blk(x, b, blk[u]); },
        [&](int u, int b) { mx_quantize_block<kCeil>(blk[u], packed + b, scales + b, bad); });
    if (bad)
        raise_status(status, kStatusNonFinite);
}

// ---------------------------------------------------------------------------
// Dequantise.  One thread per 16 codes (8 packed bytes) -> 16 outputs (one
// 32-byte bf16 store or two fp32 ones), two units in flight per thread, at
// most kDequantCtasPerSm CTAs per SM: the kernel writes 3.6 bytes for every
// byte it reads, and fewer threads in flight measured faster on the
// 8192 x 14336 activation (NVFP4 55.2 against 58.9 us with four units per
// thread at full occupancy, MXFP4 54.3 against 57.4).
// NVFP4: p * s_b is exact in any format with 6 significant bits and the
// range 2^-10 .. 2688, so it is formed by the mixed-precision
// `fma.rn.f32.f16` (f16 code value x f16 scale + -0, the -0 keeping the
// sign of a zero product), then multiplied by g as fp32 pairs.  MXFP4:
// p * 2^e, exact, as fp32 pairs.  y points at the unit's 16 outputs.
// ---------------------------------------------------------------------------
template <bool kNv>
__device__ __forceinline__ void dequant_floats(uint2 pk, uint32_t sbyte, uint64_t g2, float (&y16)[16])
{
    if constexpr (kNv) {
        const uint16_t sh = e4m3_to_f16(sbyte);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t ph[4];
            e2m1x8_to_f16x2(h ? pk.y : pk.x, ph);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float a, b;
                f16x2_mul_f16_to_f32(ph[j], sh, a, b);
                unpack2(mul2(pack2(a, b), g2), y16[8 * h + 2 * j], y16[8 * h + 2 * j + 1]);
            }
        }
    } else if (sbyte - 103u <= 39u) {
        // 2^e with -24 <= e <= 15 is exact in f16: p * 2^e (exact) by the
        // mixed-precision fma, one instruction per element
        const uint16_t sh = e8m0_to_f16(sbyte);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t ph[4];
            e2m1x8_to_f16x2(h ? pk.y : pk.x, ph);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                f16x2_mul_f16_to_f32(ph[j], sh, y16[8 * h + 2 * j], y16[8 * h + 2 * j + 1]);
        }
    } else {
        const float s = e8m0_to_f32(sbyte);
        const uint64_t s2 = pack2(s, s);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float p[8];
            e2m1x8_decode(h ? pk.y : pk.x, p);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                unpack2(mul2(pack2(p[2 * j], p[2 * j + 1]), s2), y16[8 * h + 2 * j],
                        y16[8 * h + 2 * j + 1]);
        }
    }
}

// fp32 -> output element: bf16 bits (round to nearest even) or fp32.
template <typename TOut> __device__ __forceinline__ TOut to_out(float v)
{
    if constexpr (sizeof(TOut) == 2) {
        uint16_t h;
        asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(v));
        return h;
    } else {
        return v;
    }
}

template <bool kNv, typename TOut>
__device__ __forceinline__ void dequant_unit(uint2 pk, uint32_t sbyte, uint64_t g2, TOut *y)
{
    float y16[16];
    dequant_floats<kNv>(pk, sbyte, g2, y16);
    uint32_t o[8];
    if constexpr (sizeof(TOut) == 2) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[j]) : "f"(y16[2 * j + 1]), "f"(y16[2 * j]));
        stg_v8(y, o);
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                o[j] = __float_as_uint(y16[8 * h + j]);
            stg_v8(y + 8 * h, o);
        }
    }
}

constexpr int kDequantUnits = 2;
constexpr int kDequantCtasPerSm = 4;

template <bool kNv, typename TOut>
__global__ void __launch_bounds__(kThreads)
    dequantize_kernel(const uint2 *__restrict__ packed, const uint8_t *__restrict__ scales,
                      const float *__restrict__ global_scale, int n_units, TOut *__restrict__ y)
{
    pdl_begin();
    const float g = kNv ? __ldcg(global_scale) : 1.0f;
    const uint64_t g2 = pack2(g, g);
    uint2 pk[kDequantUnits];
    uint32_t sbyte[kDequantUnits];
    stream_units<kDequantUnits>(
        n_units,
        [&](int u, int i) {
            pk[u] = __ldcg(packed + i);
            sbyte[u] = __ldcg(scales + (kNv ? i : (i >> 1)));
        },
        [&](int u, int i) { dequant_unit<kNv>(pk[u], sbyte[u], g2, y + (int64_t)i * 16); });
}

// ---------------------------------------------------------------------------
// Scale search.  One thread owns one 16-element block, kept in registers.
//
// Candidate set: c_k = E4M3(m_k A_b / (6g)), m_k = (147 + k)/210.  The raw
// candidates grow by a factor of at most 148/147 from one k to the next
// while every E4M3 rounding interval spans a factor above 1 + 1/16, so the
// 64 candidates hit exactly the codes c_0 .. c_63, all of them: two
// roundings per block (c_63 is the max-based NVFP4 scale).
//
// Order and pruning: codes run from c_63 down.  For a scale whose largest
// reconstruction T7 = fl32(fl32(6 s_b) g) is below A_b, the block maximum
// alone contributes (A_b - T7)^2 to the loss, a lower bound that only grows
// as the scale shrinks; once it exceeds the best loss so far no smaller
// candidate can win or tie, and the search of the block stops (about 2.3 of
// 5 candidates evaluated on Laplace data).
//
// Screening: the block is scaled by k = 2^(127 - f) (f the exponent field
// of A_b, so A_b k is in [1, 2); scaling changes no comparison).  With d_k =
// fl32(s_b g) k, v_i = RN(x_i k r) (r within two ulps of 1/d_k) and p_i the
// E2M1 grid value of v_i, the screening loss is S = d_k^2 sum_i (v_i - p_i)^2.
// Against the exact scaled loss L = sum_i (x_i k - x_hat_i k)^2 it differs by
// at most B(S, d_k) = 1e-6 S + 6e-6 sqrt(S) + 7e-5 d_k^2 + 1e-11: per element
// the two differences agree within 2^-23 (1.5 |x k| + |x_hat k|) <= 7.2e-7;
// an element within a few ulps of an E2M1 midpoint may round to the other
// neighbour, whose squared error differs by at most 4.3e-6 d_k^2; the fp32
// sum adds 1e-6 S.  A comparison with |S_a - S_b| <= B_a + B_b, and every
// comparison when g < 2^-116 (reconstructions could be subnormal), is redone
// on the exact double loss of the definition -- exact codes, x_hat as
// dequantised, sum_i ((double)x_i - (double)x_hat_i)^2 in element order --
// so the winner is the winner of the exact-in-double search, and on equal
// loss the larger scale (the one met first) stays.
// ---------------------------------------------------------------------------
// Eight consecutive elements (half a block) reloaded from memory as fp32.
template <typename T>
__device__ __forceinline__ void load_half(const T *x, int blk, int h, float (&v)[8])
{
    const char *p = reinterpret_cast<const char *>(x) + ((int64_t)blk * 16 + 8 * h) * (int64_t)sizeof(T);
    uint32_t w[8];
    if constexpr (sizeof(T) == 2) {
        asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "l"(p));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    } else {
        ldg_v8(p, w);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = __uint_as_float(w[j]);
    }
}

// Exact codes of one half-block at scale code c (zero scale -> zero codes).
template <typename T>
__device__ __forceinline__ uint32_t exact_half_codes(const T *x, int blk, int h, uint32_t c,
                                                     float g, float (&v)[8])
{
    load_half(x, blk, h, v);
    if (c == 0u)
        return 0u;
    return nv_encode8(v, nv_recip(__fmul_rn(e4m3_pos_to_f32(c), g)));
}

// The definition's loss of scale code c over one block, in double, in
// element order: exact codes, x_hat = fl32(fl32(p s_b) g), sum of
// ((double)x - (double)x_hat)^2.  Reloads the block (an L2 hit); one half
// at a time to stay light on registers (inlined: it is small, and ptxas
// 12.9 crashed on an out-of-line version called from two kernels).
template <typename T>
__device__ __forceinline__ double exact_loss_of(const T *x, int blk, uint32_t c, float g)
{
    const float sb = e4m3_pos_to_f32(c);
    double acc = 0.0;
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
        float v[8], p[8];
        e2m1x8_decode(exact_half_codes(x, blk, h, c, g, v), p);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double dd = __dsub_rn((double)v[i], (double)nv_dequant(p[i], sb, g));
            acc = __dadd_rn(acc, __dmul_rn(dd, dd));
        }
    }
    return acc;
}

// Exact codes of a whole block at scale code c (used when g is so small that
// the scaled encode could see subnormal reconstructions).
template <typename T>
__device__ __forceinline__ uint2 exact_codes_of(const T *x, int blk, uint32_t c, float g)
{
    float v[8];
    uint2 pk;
    pk.x = exact_half_codes(x, blk, 0, c, g, v);
    pk.y = exact_half_codes(x, blk, 1, c, g, v);
    return pk;
}

// Screening loss of candidate code c and its error bound.
struct Screen {
    float s, bound;
};

__device__ __forceinline__ Screen screen(const float (&xk)[16], uint32_t c, float g, float k)
{
    Screen r;
    if (c == 0u) { // zero scale: x_hat = 0, the sum of squares in fp32
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            acc = fmaf(xk[i], xk[i], acc);
        r.s = acc;
        r.bound = fmaf(acc, 1e-6f, 1e-11f);
        return r;
    }
    const float dk = __fmul_rn(__fmul_rn(e4m3_pos_to_f32(c), g), k);
    const float r0 = rcp_approx(dk);
    const float rc = fmaf(r0, fmaf(-dk, r0, 1.0f), r0);
    // four interleaved fp32 sums (two packed pairs, two short dependency
    // chains); summation error < 7u S
    const uint64_t rc2 = pack2(rc, rc);
    uint64_t acc2[2] = {pack2(0.0f, 0.0f), pack2(0.0f, 0.0f)};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float v[8], e[8];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            unpack2(mul2(pack2(xk[8 * h + 2 * j], xk[8 * h + 2 * j + 1]), rc2), v[2 * j], v[2 * j + 1]);
        e2m1x8_error(v, e);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint64_t e2 = pack2(e[2 * j], e[2 * j + 1]);
            acc2[j & 1] = fma2(e2, e2, acc2[j & 1]);
        }
    }
    float a0, a1, a2, a3;
    unpack2(acc2[0], a0, a1);
    unpack2(acc2[1], a2, a3);
    const float acc = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
    const float d2 = __fmul_rn(dk, dk);
    r.s = __fmul_rn(acc, d2);
    // sqrt.approx is within 2^-21 of sqrt(S): the 6.001e-6 covers it
    r.bound = fmaf(r.s, 1e-6f, fmaf(sqrt_approx(r.s), 6.001e-6f, fmaf(d2, 7e-5f, 1e-11f)));
    return r;
}

// One block's search.  Only the scaled block x k stays in registers: the
// codes of x/d and of (x k)/(d k) are the same (the two quotients are the same
// real number, and an x k that underflowed is tiny, code 0 with x's sign,
// like x/d), so the final encode runs on x k; the exact comparisons and the
// optional loss output reload the block.
template <typename T> struct BlockSearch {
    const T *x;
    int blk;
    float xk[16];
    float g, k, ak, gk;
    uint32_t c_lo, best_c, next_c;
    float best, best_bound;
    bool exact_always;

    // Loads the block; returns max |x| over it.
    __device__ __forceinline__ float setup(const T *x_, int blk_, float g_, bool exact_always_)
    {
        x = x_;
        blk = blk_;
        g = g_;
        exact_always = exact_always_;
        Blk<T, 16> b;
        load_blk(x, blk, b);
        const uint32_t ab = absmax_bits(b);
        k = __uint_as_float((254u - min(ab >> 23, 253u)) << 23);
        gk = __fmul_rn(g, k);
        ak = __fmul_rn(__uint_as_float(ab), k);
        const uint64_t k2 = pack2(k, k);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            unpack2(mul2(pack2(elem(b, 2 * i), elem(b, 2 * i + 1)), k2), xk[2 * i], xk[2 * i + 1]);
        return __uint_as_float(ab);
    }

    // Screen candidate c against the best so far; returns false when the
    // lower bound ends the search.
    __device__ __forceinline__ bool step(uint32_t c)
    {
        const float t7 = __fmul_rn(__fmul_rn(6.0f, e4m3_pos_to_f32(c)), gk);
        if (ak > t7) {
            const float e = __fsub_rn(ak, t7);
            if (__fmul_rn(e, e) > __fmul_rn(__fadd_rn(best, best_bound), 1.0000003f))
                return false;
        }
        const Screen sc = screen(xk, c, g, k);
        bool take;
        if (!exact_always && fabsf(__fsub_rn(sc.s, best)) > __fadd_rn(sc.bound, best_bound))
            take = sc.s < best;
        else
            take = exact_loss_of(x, blk, c, g) < exact_loss_of(x, blk, best_c, g);
        if (take) {
            best_c = c;
            best = sc.s;
            best_bound = sc.bound;
        }
        return true;
    }

    // Continue from next_c down to c_lo for at most max_steps candidates;
    // true when the search is complete.
    __device__ __forceinline__ bool run(int max_steps)
    {
#pragma unroll 1
        for (int n = 0; n < max_steps; ++n) {
            if (next_c <= c_lo)
                return true;
            const uint32_t c = next_c - 1;
            if (!step(c)) {
                next_c = c_lo;
                return true;
            }
            next_c = c;
        }
        return next_c <= c_lo;
    }

    __device__ __forceinline__ void finish(uint2 *packed, uint8_t *scales, float *block_loss)
    {
        uint2 pk = make_uint2(0u, 0u);
        if (exact_always) {
            pk = exact_codes_of(x, blk, best_c, g);
        } else if (best_c != 0u) {
            const NvRecip q = nv_recip(__fmul_rn(__fmul_rn(e4m3_pos_to_f32(best_c), g), k));
            float h[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                h[i] = xk[i];
            pk.x = nv_encode8(h, q);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                h[i] = xk[8 + i];
            pk.y = nv_encode8(h, q);
        }
        packed[blk] = pk;
        scales[blk] = (uint8_t)best_c;
        if (block_loss)
            block_loss[blk] = (float)exact_loss_of(x, blk, best_c, g);
    }
};

// The candidate grid m_k = (p + k) / q, k = 0..n-1 (the fixed search: 64,
// 147, 210) is passed as num_lo = p, num_hi = p + n - 1 and q; with p >= 16
// consecutive raw candidates differ by a factor of at most 17/16, so they
// hit every code from c_lo (k = 0) to c_hi (k = n - 1), as above.  num and
// q are at most 2^20: num A_b and 6 q g are exact in double.  kFixed: the
// fixed grid, compiled in (the arguments are ignored).
constexpr int kSearchP = 147, kSearchQ = 210, kSearchN = 64;

template <typename T, bool kFixed>
__global__ void __launch_bounds__(kThreads, 4)
    scale_search_kernel(const T *__restrict__ x, int n_blocks, const float *amax,
                        uint2 *__restrict__ packed, uint8_t *__restrict__ scales,
                        float *global_scale, float *__restrict__ block_loss, int32_t *status,
                        int num_lo_arg, int num_hi_arg, int q_arg)
{
    pdl_begin();
    float g;
    if (!nv_prologue(amax, global_scale, status, g))
        return;
    const int num_lo = kFixed ? kSearchP : num_lo_arg;
    const int num_hi = kFixed ? kSearchP + kSearchN - 1 : num_hi_arg;
    const int q = kFixed ? kSearchQ : q_arg;
    const NvScaleConsts sc = nv_scale_consts(g);
    const double den = 6.0 * (double)q * (double)g;      // exact: at most 23 + 24 significant bits
    const float inv_lo = (float)((double)num_lo / den);  // RN32 of m_0 / (6g), within an ulp
    const float inv_hi = (float)((double)num_hi / den);
    const bool hi_is_max = kFixed || num_hi == q; // the largest candidate is the max-based scale
    const bool exact_always = !(g >= 0x1p-116f);
    const int stride = (int)(gridDim.x * blockDim.x);
    for (int blk = (int)(blockIdx.x * blockDim.x + threadIdx.x); blk < n_blocks; blk += stride) {
        BlockSearch<T> bs;
        const float amax_b = bs.setup(x, blk, g, exact_always);
        const uint32_t c_hi = hi_is_max ? nv_scale_code_mg(amax_b, sc.inv6g, sc.g, 6.0f, sc.six_g)
                                        : nv_scale_code(amax_b, inv_hi, (double)num_hi, den);
        bs.c_lo = nv_scale_code(amax_b, inv_lo, (double)num_lo, den);
        bs.best_c = c_hi;
        bs.next_c = c_hi;
        const Screen s0 = screen(bs.xk, c_hi, g, bs.k);
        bs.best = s0.s;
        bs.best_bound = s0.bound;
        bs.run(128);
        bs.finish(packed, scales, block_loss);
    }
}

// ---------------------------------------------------------------------------
// NVFP4 "four over six" ("FP4、FP8 与 INT8/INT4" section 4: mapping the block
// maximum to 4 instead of 6 can put the other values on better grid points;
// neither wins on every block).  Per block the E4M3 codes nearest to
// A_b/(6g) (the max-based scale) and A_b/(4g) are compared on the loss of the
// emitted artefact, screened and, when close, settled exactly as in the
// search; the max-to-4 scale is taken only when strictly better.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
    nvfp4_four_over_six_kernel(const T *__restrict__ x, int n_blocks, const float *amax,
                               uint2 *__restrict__ packed, uint8_t *__restrict__ scales,
                               float *global_scale, float *__restrict__ block_loss,
                               int32_t *status)
{
    pdl_begin();
    float g;
    if (!nv_prologue(amax, global_scale, status, g))
        return;
    const NvScaleConsts sc = nv_scale_consts(g);
    const double four_g = 4.0 * (double)g;    // exact
    const float inv4g = (float)(1.0 / four_g); // RN32(1 / (4g))
    const bool exact_always = !(g >= 0x1p-116f);
    const int stride = (int)(gridDim.x * blockDim.x);
    for (int blk = (int)(blockIdx.x * blockDim.x + threadIdx.x); blk < n_blocks; blk += stride) {
        BlockSearch<T> bs;
        const float amax_b = bs.setup(x, blk, g, exact_always);
        const uint32_t c6 = nv_scale_code_mg(amax_b, sc.inv6g, sc.g, 6.0f, sc.six_g);
        const uint32_t c4 = nv_scale_code_mg(amax_b, inv4g, sc.g, 4.0f, four_g);
        bs.best_c = c6;
        const Screen s0 = screen(bs.xk, c6, g, bs.k);
        bs.best = s0.s;
        bs.best_bound = s0.bound;
        if (c4 != c6)
            bs.step(c4);
        bs.finish(packed, scales, block_loss);
    }
}

// ---------------------------------------------------------------------------
// Test-only element kernels (internal linkage: this header is included by
// more than one translation unit).
// ---------------------------------------------------------------------------
static __global__ void e2m1_round_kernel(const float *__restrict__ v, uint8_t *__restrict__ codes,
                                  int64_t n)
{
    pdl_begin();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u * 8 < n; u += stride) {
        float a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            a[i] = (u * 8 + i < n) ? v[u * 8 + i] : 0.0f;
        const uint32_t pk = e2m1x8(a);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (u * 8 + i < n)
                codes[u * 8 + i] = (uint8_t)((pk >> (4 * i)) & 15u);
    }
}

// decode(encode(v)) with the codes passed from one helper to the other in
// registers, as the kernels do.
static __global__ void e2m1_roundtrip_kernel(const float *__restrict__ v, float *__restrict__ out,
                                      int64_t n)
{
    pdl_begin();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u * 8 < n; u += stride) {
        float a[8], p[8], q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            a[i] = (u * 8 + i < n) ? v[u * 8 + i] : 0.0f;
        e2m1x8_decode(e2m1x8(a), p);
        e2m1x8_qdq(a, q);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (u * 8 + i < n) {
                out[2 * (u * 8 + i)] = p[i];
                out[2 * (u * 8 + i) + 1] = q[i];
            }
    }
}

static __global__ void nv_encode_quotient_kernel(const float *__restrict__ x, const float *__restrict__ d,
                                          uint8_t *__restrict__ codes, int64_t n)
{
    pdl_begin();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        float a[8] = {x[i], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        codes[i] = (uint8_t)(nv_encode8(a, nv_recip(d[i])) & 15u);
    }
}

} // namespace fp4
