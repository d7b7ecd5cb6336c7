// fp4_grouped.cuh -- kernels that quantise or dequantise many matrices in
// one launch, each matrix with its own scales ("NVFP4 与 MXFP4 格式"
// section 3: the global scale g is a per-tensor quantity, so a whole-model
// weight set needs one tensor amax and one g per matrix).
//
// The matrices of one launch are described by a table passed by value as a
// kernel parameter (__grid_constant__, at most kGroupMax entries, about
// 11 KB): per entry its pointers and first[e], the first unit of the entry
// in the launch's concatenated unit space (first[n] = total, below 2^30).
// The quantisers and dequantisers walk the table tile by tile
// (grouped_tiles: a tile is kThreads * U consecutive units of one entry, so
// the entry lookup, the entry's pointers and its constants are per tile and
// uniform across the CTA, and nothing is looked up per unit).  Units are the
// same as in the single-tensor kernels (a 16-block for NVFP4, a 32-block for
// MXFP4, 16 codes for dequantisation, 64 KB of input for the amax), so every
// thread runs the single-tensor per-block code; per-entry constants (g,
// 1/(6g)) are recomputed only when the entry changes.  A matrix larger than
// one launch allows is split by the host into several entries over
// sub-ranges that share its amax word and g.
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
// Tile-major walk of a grouped table.  The units of every entry are cut
// into tiles of kThreads * U consecutive units (the last tile of an entry
// may be short); tile_first[e] is entry e's first tile in the launch's
// concatenated tile space.  CTA c takes tiles c, c + gridDim.x, ...: every
// tile lies in one entry, so the entry lookup, the entry's pointers and its
// constants are per tile and uniform across the CTA, and the per-unit work
// is the single-tensor kernels' own.  `enter(e)` is called when the entry
// changes and returns false to skip the entry; `load(u, e, b)` and
// `work(u, e, b)` take unit b of entry e.
// ---------------------------------------------------------------------------
template <int U, typename Table, typename Enter, typename Load, typename Work>
__device__ __forceinline__ void grouped_tiles(const Table &grp, Enter &&enter, Load &&load, Work &&work)
{
    constexpr int kTile = kThreads * U;
    const int tiles = grp.tile_first[grp.n];
    int e = 0, cur = -1;
    bool ok = false;
    for (int t = (int)blockIdx.x; t < tiles; t += (int)gridDim.x) {
        e = entry_from(grp.tile_first, t, e);
        if (e != cur) {
            cur = e;
            ok = enter(e);
        }
        if (!ok)
            continue;
        const int nb = grp.first[e + 1] - grp.first[e];
        const int b0 = (t - grp.tile_first[e]) * kTile + (int)threadIdx.x;
        if (b0 + (U - 1) * kThreads < nb) {
#pragma unroll
            for (int u = 0; u < U; ++u)
                load(u, e, b0 + u * kThreads);
#pragma unroll
            for (int u = 0; u < U; ++u)
                work(u, e, b0 + u * kThreads);
        } else {
            for (int b = b0; b < nb; b += kThreads) {
                load(0, e, b);
                work(0, e, b);
            }
        }
    }
}

// As grouped_tiles, with the choice between a tile's two paths uniform
// across the CTA: a tile all of whose kThreads * U units exist goes to
// `whole(e, b0)` (this thread's units b0 + u * kThreads, u < U; all lanes of
// every warp together, so the body may use warp collectives), the units of a
// short tile one at a time to `one(e, b)`.
template <int U, typename Table, typename Enter, typename Whole, typename One>
__device__ __forceinline__ void grouped_tiles_cta(const Table &grp, Enter &&enter, Whole &&whole, One &&one)
{
    constexpr int kTile = kThreads * U;
    const int tiles = grp.tile_first[grp.n];
    int e = 0, cur = -1;
    bool ok = false;
    for (int t = (int)blockIdx.x; t < tiles; t += (int)gridDim.x) {
        e = entry_from(grp.tile_first, t, e);
        if (e != cur) {
            cur = e;
            ok = enter(e);
        }
        if (!ok)
            continue;
        const int nb = grp.first[e + 1] - grp.first[e];
        const int first = (t - grp.tile_first[e]) * kTile;
        if (first + kTile <= nb) {
            whole(e, first + (int)threadIdx.x);
        } else {
            for (int b = first + (int)threadIdx.x; b < nb; b += kThreads)
                one(e, b);
        }
    }
}

// Tiles of `units` units at U units per thread (host and device).
__host__ __device__ constexpr int grouped_tile_count(int64_t units, int U)
{
    return (int)((units + (int64_t)kThreads * U - 1) / ((int64_t)kThreads * U));
}

// ---------------------------------------------------------------------------
// NVFP4 quantise of every entry with its own g = fl32(A_e / 2688).  Thread t
// of the grid first publishes entry t's g (or raises the entry's data
// error); then the blocks are quantised tile by tile, an entry with an
// error skipped.
// ---------------------------------------------------------------------------
// 16-blocks per thread per tile, and the register budget: three blocks in
// flight at four CTAs per SM measured fastest on the 7B weight set (3.90 ms
// against 4.33 with four blocks at two CTAs, 3.93 with two blocks).
constexpr int kNvGroupedU = 3;
constexpr int kNvGroupedCtasPerSm = 4;

struct NvGroup {
    int n;
    int first[kGroupMax + 1];        // first 16-block of each entry
    int tile_first[kGroupMax + 1];   // first tile of each entry
    const void *x[kGroupMax];
    uint2 *packed[kGroupMax];
    uint8_t *scales[kGroupMax];
    const uint32_t *amax[kGroupMax]; // bits of the entry's matrix amax
    float *global_scale[kGroupMax];
};

template <typename T>
__global__ void __launch_bounds__(kThreads, kNvGroupedCtasPerSm)
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
    NvScaleConsts sc = nv_scale_consts(1.0f);
    const T *x = nullptr;
    uint2 *packed = nullptr;
    uint8_t *scales = nullptr;
    constexpr int U = kNvGroupedU;
    auto enter = [&](int e) {
        int32_t err;
        const float g = nv_global_scale(__ldcg(grp.amax[e]), err);
        if (err)
            return false;
        sc = nv_scale_consts(g);
        x = static_cast<const T *>(grp.x[e]);
        packed = grp.packed[e];
        scales = grp.scales[e];
        return true;
    };
    auto one = [&](int, int b) {
        Blk<T, 16> blk;
        load_blk(x, b, blk);
        nv_quantize_block(blk, sc, packed + b, scales + b);
    };
    if constexpr (sizeof(T) == 2) {
        __shared__ NvExactQueue<U> queues[kThreads / 32];
        NvExactQueue<U> &q = queues[threadIdx.x >> 5];
        grouped_tiles_cta<U>(
            grp, enter,
            [&](int, int b0) {
                Blk<T, 16> blk[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    load_blk(x, b0 + u * kThreads, blk[u]);
                uint2 pk[U];
                uint32_t code[U];
                nv_quantize_warp(blk, sc, q, pk, code);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    packed[b0 + u * kThreads] = pk[u];
                    scales[b0 + u * kThreads] = (uint8_t)code[u];
                }
            },
            one);
    } else {
        grouped_tiles_cta<U>(
            grp, enter,
            [&](int e, int b0) {
                Blk<T, 16> blk[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    load_blk(x, b0 + u * kThreads, blk[u]);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    nv_quantize_block(blk[u], sc, packed + b0 + u * kThreads, scales + b0 + u * kThreads);
            },
            one);
    }
}

// ---------------------------------------------------------------------------
// MXFP4 quantise of every entry (no tensor-level scale), tile by tile.
// ---------------------------------------------------------------------------
constexpr int kMxGroupedU = 2; // 32-blocks per thread per tile

struct MxGroup {
    int n;
    int first[kGroupMax + 1];      // first 32-block of each entry
    int tile_first[kGroupMax + 1]; // first tile of each entry
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
    const T *x = nullptr;
    uint4 *packed = nullptr;
    uint8_t *scales = nullptr;
    Blk<T, 32> blk[kMxGroupedU];
    grouped_tiles<kMxGroupedU>(
        grp,
        [&](int e) {
            x = static_cast<const T *>(grp.x[e]);
            packed = grp.packed[e];
            scales = grp.scales[e];
            return true;
        },
        [&](int u, int, int b) { load_blk(x, b, blk[u]); },
        [&](int u, int, int b) { mx_quantize_block<kCeil>(blk[u], packed + b, scales + b, bad); });
    if (bad)
        raise_status(status, kStatusNonFinite);
}

// ---------------------------------------------------------------------------
// Dequantise every entry (16 codes per unit), tile by tile (grouped_tiles,
// kDequantUnits units per thread per tile, at most kDequantCtasPerSm CTAs
// per SM as the single-tensor dequantiser).  MXFP4 entries start on an even
// unit of their matrix (the host splits only at even units), so the scale
// of unit b is scales[b >> 1].
// ---------------------------------------------------------------------------
struct DqGroup {
    int n;
    int first[kGroupMax + 1];      // first unit of each entry
    int tile_first[kGroupMax + 1]; // first tile of each entry
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
    const uint2 *packed = nullptr;
    const uint8_t *scales = nullptr;
    TOut *y = nullptr;
    uint2 pk[kDequantUnits];
    uint32_t sbyte[kDequantUnits];
    uint64_t g2 = pack2(1.0f, 1.0f);
    grouped_tiles<kDequantUnits>(
        grp,
        [&](int e) {
            if (kNv) {
                const float g = __ldcg(grp.global_scale[e]);
                g2 = pack2(g, g);
            }
            packed = grp.packed[e];
            scales = grp.scales[e];
            y = static_cast<TOut *>(grp.y[e]);
            return true;
        },
        [&](int u, int, int b) {
            pk[u] = __ldcg(packed + b);
            sbyte[u] = __ldcg(scales + (kNv ? b : (b >> 1)));
        },
        [&](int u, int, int b) { dequant_unit<kNv>(pk[u], sbyte[u], g2, y + (int64_t)b * 16); });
}

} // namespace fp4
