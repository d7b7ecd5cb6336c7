// fp4_grouped.cuh -- kernels that quantise or dequantise many matrices in
// one launch, each matrix with its own scales ("NVFP4 与 MXFP4 格式"
// section 3: the global scale g is a per-tensor quantity, so a whole-model
// weight set needs one tensor amax and one g per matrix).
//
// The matrices of one launch are described by a table passed by value as a
// kernel parameter (__grid_constant__, at most kGroupMax entries, about
// 11 KB): per entry its pointers and first[e], the first unit of the entry
// in the launch's concatenated unit space (first[n] = total, below 2^30).
// The MXFP4 and dequantisation kernels give each CTA one contiguous range of
// units (stream_units_blocked), so a thread meets only one or two matrices;
// the NVFP4 quantiser keeps the grid-stride order, which measured faster for
// it.  Units are the same as in the single-tensor kernels (a 16-block for NVFP4,
// a 32-block for MXFP4, 16 codes for dequantisation, 64 KB of input for the
// amax), so every thread runs the single-tensor per-block code.  A thread
// walks its units in increasing order and finds each unit's entry with a
// forward-only cursor; the per-entry constants (g, 1/(6g)) are recomputed
// only when the entry changes.  A matrix larger than one launch allows is
// split by the host into several entries over sub-ranges that share its
// amax word and g.
#pragma once

#include <cstdint>

#include "fp4_kernels.cuh"

namespace fp4 {

constexpr int kGroupMax = 256;
constexpr int kAmaxChunkVecs = kThreads * 8; // 32-byte vectors per amax unit (64 KB)

// Entry of unit i, searching forward from entry e (i < first[n]).
__device__ __forceinline__ int entry_from(const int *first, int i, int e)
{
    while (i >= first[e + 1])
        ++e;
    return e;
}

// ---------------------------------------------------------------------------
// Per-entry tensor amax.  A unit is a chunk of kAmaxChunkVecs vectors of one
// entry (the last chunk of an entry may be short); each CTA takes whole
// chunks, reduces them across the CTA and folds the result into the
// entry's amax word with one atomicMax (max |x| bit patterns order like the
// values; NaN / Inf patterns sort above every finite value) and raises
// FP4_ERR_NONFINITE for a NaN or Inf.  The amax words must be zero before
// the launch.
// ---------------------------------------------------------------------------
struct AmaxGroup {
    int n;
    int first[kGroupMax + 1];   // first chunk of each entry
    const void *x[kGroupMax];
    int64_t nvec[kGroupMax];    // 32-byte vectors in the entry
    uint32_t *amax[kGroupMax];  // the entry's amax word (bits of max |x|)
};

template <typename T>
__global__ void __launch_bounds__(kThreads)
    amax_grouped_kernel(const __grid_constant__ AmaxGroup grp, int32_t *status)
{
    pdl_begin();
    constexpr int kPerVec = 32 / (int)sizeof(T);
    constexpr int kPer = kAmaxChunkVecs / kThreads;
    const int total = grp.first[grp.n];
    int e = 0;
    for (int c = blockIdx.x; c < total; c += gridDim.x) {
        e = entry_from(grp.first, c, e);
        const T *x = static_cast<const T *>(grp.x[e]);
        const int64_t v0 = (int64_t)(c - grp.first[e]) * kAmaxChunkVecs + threadIdx.x;
        const int64_t nv = grp.nvec[e];
        Blk<T, kPerVec> v[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u)
            if (v0 + u * kThreads < nv)
                load_blk(x, v0 + u * kThreads, v[u]);
        uint32_t m = 0;
#pragma unroll
        for (int u = 0; u < kPer; ++u)
            if (v0 + u * kThreads < nv)
                m = max(m, absmax_bits(v[u]));
        m = cta_max_u32(m);
        if (threadIdx.x == 0) {
            atomicMax(grp.amax[e], m);
            if (m >= kNonFiniteBits)
                raise_status(status, kStatusNonFinite);
        }
    }
}

// ---------------------------------------------------------------------------
// NVFP4 quantise of every entry with its own g = fl32(A_e / 2688).  Thread t
// of the grid first publishes entry t's g (or raises the entry's data
// error); then the blocks are quantised, an entry with an error skipped.
// ---------------------------------------------------------------------------
struct NvGroup {
    int n;
    int first[kGroupMax + 1];        // first 16-block of each entry
    const void *x[kGroupMax];
    uint2 *packed[kGroupMax];
    uint8_t *scales[kGroupMax];
    const uint32_t *amax[kGroupMax]; // bits of the entry's matrix amax
    float *global_scale[kGroupMax];
};

template <typename T>
__global__ void __launch_bounds__(kThreads)
    nvfp4_quantize_grouped_kernel(const __grid_constant__ NvGroup grp, int32_t *status)
{
    pdl_begin();
    const int t = (int)(blockIdx.x * blockDim.x + threadIdx.x);
    if (t < grp.n) {
        int32_t err;
        const float g = nv_global_scale(__ldcg(grp.amax[t]), err);
        if (err)
            raise_status(status, err);
        else
            *grp.global_scale[t] = g;
    }
    int e = 0, cur = -1;
    int ent[2];
    bool ok = false;
    NvScaleConsts sc = nv_scale_consts(1.0f);
    Blk<T, 16> blk[2];
    stream_units<2>(
        grp.first[grp.n],
        [&](int u, int i) {
            e = entry_from(grp.first, i, e);
            ent[u] = e;
            load_blk(static_cast<const T *>(grp.x[e]), i - grp.first[e], blk[u]);
        },
        [&](int u, int i) {
            const int en = ent[u];
            if (en != cur) {
                cur = en;
                int32_t err;
                const float g = nv_global_scale(__ldcg(grp.amax[en]), err);
                ok = err == 0;
                if (ok)
                    sc = nv_scale_consts(g);
            }
            if (ok) {
                const int b = i - grp.first[en];
                nv_quantize_block(blk[u], sc, grp.packed[en] + b, grp.scales[en] + b);
            }
        });
}

// ---------------------------------------------------------------------------
// MXFP4 quantise of every entry (no tensor-level scale).
// ---------------------------------------------------------------------------
struct MxGroup {
    int n;
    int first[kGroupMax + 1]; // first 32-block of each entry
    const void *x[kGroupMax];
    uint4 *packed[kGroupMax];
    uint8_t *scales[kGroupMax];
};

template <typename T, bool kCeil>
__global__ void __launch_bounds__(kThreads)
    mxfp4_quantize_grouped_kernel(const __grid_constant__ MxGroup grp, int32_t *status)
{
    pdl_begin();
    bool bad = false;
    int e = 0;
    int ent[2];
    Blk<T, 32> blk[2];
    stream_units_blocked<2>(
        grp.first[grp.n],
        [&](int u, int i) {
            e = entry_from(grp.first, i, e);
            ent[u] = e;
            load_blk(static_cast<const T *>(grp.x[e]), i - grp.first[e], blk[u]);
        },
        [&](int u, int i) {
            const int en = ent[u];
            const int b = i - grp.first[en];
            mx_quantize_block<kCeil>(blk[u], grp.packed[en] + b, grp.scales[en] + b, bad);
        });
    if (bad)
        raise_status(status, kStatusNonFinite);
}

// ---------------------------------------------------------------------------
// Dequantise every entry (16 codes per unit).  MXFP4 entries start on an
// even unit of their matrix (the host splits only at even units), so the
// scale of unit b is scales[b >> 1].
// ---------------------------------------------------------------------------
struct DqGroup {
    int n;
    int first[kGroupMax + 1]; // first unit of each entry
    const uint2 *packed[kGroupMax];
    const uint8_t *scales[kGroupMax];
    const float *global_scale[kGroupMax]; // NVFP4 only
    void *y[kGroupMax];
};

template <bool kNv, typename TOut>
__global__ void __launch_bounds__(kThreads)
    dequantize_grouped_kernel(const __grid_constant__ DqGroup grp)
{
    pdl_begin();
    int e = 0, cur = -1;
    int ent[4];
    uint2 pk[4];
    uint32_t sbyte[4];
    uint64_t g2 = pack2(1.0f, 1.0f);
    stream_units_blocked<4>(
        grp.first[grp.n],
        [&](int u, int i) {
            e = entry_from(grp.first, i, e);
            ent[u] = e;
            const int b = i - grp.first[e];
            pk[u] = __ldcg(grp.packed[e] + b);
            sbyte[u] = __ldcg(grp.scales[e] + (kNv ? b : (b >> 1)));
        },
        [&](int u, int i) {
            const int en = ent[u];
            if (kNv && en != cur) {
                cur = en;
                const float g = __ldcg(grp.global_scale[en]);
                g2 = pack2(g, g);
            }
            const int b = i - grp.first[en];
            dequant_unit<kNv>(pk[u], sbyte[u], g2, static_cast<TOut *>(grp.y[en]) + (int64_t)b * 16);
        });
}

} // namespace fp4
