// fp4_layouts.cuh -- the other block layouts of "NVFP4 与 MXFP4 格式":
//
//   ragged rows (section 8: padding each row to whole blocks, R*ceil(K/G)
//     blocks; section 7: the padded layout is decoded as padded and then cut
//     back to the logical shape).  Rows of K elements, K not a multiple of
//     the block size G, are quantised as if padded with +0 to
//     Kp = ceil(K/G)*G; the outputs are the plain layout of the padded
//     [R, Kp] matrix.  Dequantisation writes only the K logical columns.
//   column-wise grouping (section 6: grouping along the other axis changes
//     which elements share a block, Q(W)^T != Q(W^T)).  The blocks of
//     Q(W^T) run down the columns of W [R, C]; the output is the plain
//     row-padded layout of the [C, R] transpose, produced from W directly.
//
// The column-wise quantiser stages 64-row x 512-byte tiles of W in shared
// memory with 2-D TMA loads (cp.async.bulk.tensor, no multicast), two
// stages deep: each stage has a "full" mbarrier (the TMA bytes landed) and
// an "empty" one (every warp released the tile), and thread 0 refills a
// stage as soon as it is empty, so no CTA-wide barrier sits in the loop.
// Each thread then quantises whole 16- or 32-element blocks down one (fp32)
// or two (bf16) tile columns.  Rows past R read as zeros (TMA out-of-bounds
// fill), which is the +0 padding.  Every mbarrier wait is bounded: a thread
// that runs out records FP4_ERR_TIMEOUT and leaves the loop, the waits that
// depended on it run out in turn, and thread 0 waits (bounded again) for
// every copy it started before the CTA ends.
#pragma once

#include <cstdint>

#include <cuda.h>

#include "fp4_kernels.cuh"

namespace fp4 {

constexpr int32_t kStatusTimeout = 8;

// ---------------------------------------------------------------------------
// Ragged rows.  Block b of the row-padded [R, Kp] matrix is row b / nbp,
// block b % nbp of that row; it covers the elements [f, f + cnt) of the flat
// input, f = (b / nbp) K + (b % nbp) G, cnt = min(G, K - (b % nbp) G), and
// reads +0 past them.  The quantisers read every block from its window of
// aligned 32-byte vectors in registers (PadWin below).  Consecutive units
// cover consecutive flat elements, so the dequantiser's tile of kPadTile
// units is one contiguous span of y: it assembles the span in shared memory
// and writes its interior back with 256-bit stores.  In shared memory each
// 32-byte vector takes 36 bytes (one pad word per eight): a unit that
// starts 32 bytes after its neighbour's then starts in another bank, so the
// word accesses of a warp are conflict-free.
// ---------------------------------------------------------------------------
constexpr int kPadTile = 256; // 16-code units per tile of the dequantiser

// Word w of the staged span lives at word w + w / 8.
__device__ __forceinline__ int pad_word(int w) { return w + (w >> 3); }

template <typename T> constexpr int pad_smem_bytes(int G)
{
    // span of kPadTile units of G elements, one vector of slack at each end,
    // and room for the last unit's writes past its real elements
    return (kPadTile * G * (int)sizeof(T) / 32 + 4) * 36;
}

// First element of the span of [f0, ...) that starts a 32-byte vector at
// the absolute address (p: the array, element-aligned; the result may lie a
// few elements before f0 when p itself is not 32-byte aligned).
template <typename T> __device__ __forceinline__ int64_t span_base(const T *p, int64_t f0)
{
    constexpr int kPerVec = 32 / (int)sizeof(T);
    const int64_t mis = (int64_t)((reinterpret_cast<uintptr_t>(p) / sizeof(T)) % kPerVec);
    return f0 - (f0 + mis) % kPerVec;
}

// Division of a 31-bit unsigned n by a launch-invariant d >= 1 (the round-up
// method of Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1,
// q = (mulhi(m, n) + n) >> l; mulhi(m, n) <= n < 2^31, so the sum does not
// overflow.  The host builds it (fast_div_for).
struct FastDiv {
    uint32_t d, m, l;
    __device__ __forceinline__ int div(int n) const
    {
        return (int)((__umulhi(m, (uint32_t)n) + (uint32_t)n) >> l);
    }
};

inline FastDiv fast_div_for(uint32_t d)
{
    uint32_t l = 0;
    while (l < 32 && (1ull << l) < d)
        ++l;
    const uint64_t m = ((1ull << 32) * ((1ull << l) - d)) / d + 1;
    return FastDiv{d, (uint32_t)m, l};
}

// First flat element of block b and its element count.
__device__ __forceinline__ int64_t pad_block_start(int b, const FastDiv &nbp, int64_t K, int G, int &cnt)
{
    const int r = nbp.div(b);
    const int j = b - r * (int)nbp.d;
    const int64_t c0 = (int64_t)j * G;
    cnt = (int)min((int64_t)G, K - c0);
    return (int64_t)r * K + c0;
}

// A ragged block read straight from global memory.  Every block of a row
// starts at the same offset within a 32-byte vector (row r starts at
// element r K, and blocks are G elements = a whole number of vectors apart),
// so a block lies in the kVecs aligned vectors from the one that holds its
// first element: one more vector than the block fills.  The window is loaded
// with 256-bit loads (the vector a block shares with its neighbour is read
// twice, the second time from L2) and the block is cut out of it with
// funnel shifts.  The word shift is the same for all the blocks of a row, so
// a warp inside one row takes one branch of the switch below.  A vector that
// starts at or past the end of the launch's rows is not read (zeros); the
// vector that holds the last element is read whole (an aligned 32-byte
// vector never crosses a page), and elements past the block's count are
// masked to +0.
template <typename T, int G> struct PadWin {
    static constexpr int kVecs = G * (int)sizeof(T) / 32 + 1;
    uint32_t w[kVecs * 8];
    int shift; // byte offset of the block's first element in the window
    int cnt;   // real elements of the block (the rest is padding)
};

template <typename T, int G>
__device__ __forceinline__ void pad_win_load(const T *x, const char *x_end, int b, const FastDiv &nbp, int64_t K,
                                             PadWin<T, G> &pw)
{
    const int64_t f = pad_block_start(b, nbp, K, G, pw.cnt);
    const uintptr_t pa = reinterpret_cast<uintptr_t>(x + f);
    const char *ab = reinterpret_cast<const char *>(pa & ~(uintptr_t)31);
    pw.shift = (int)(pa & 31u);
#pragma unroll
    for (int m = 0; m < PadWin<T, G>::kVecs; ++m) {
        if (ab + 32 * m < x_end) {
            ldg_v8(ab + 32 * m, &pw.w[8 * m]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                pw.w[8 * m + i] = 0u;
        }
    }
}

// Words [S, S + W] of the window funnel-shifted right by sh bits.
template <int S, int W, int N>
__device__ __forceinline__ void pad_win_cut(const uint32_t (&w)[N], uint32_t sh, uint32_t *out)
{
    static_assert(S + W < N, "window too short");
#pragma unroll
    for (int i = 0; i < W; ++i)
        out[i] = __funnelshift_r(w[S + i], w[S + i + 1], sh);
}

template <typename T, int G>
__device__ __forceinline__ void pad_win_block(const PadWin<T, G> &pw, Blk<T, G> &k)
{
    constexpr int W = G * (int)sizeof(T) / 4;
    const uint32_t sh = (uint32_t)(pw.shift & 3) * 8u;
    switch (pw.shift >> 2) {
    case 0: pad_win_cut<0, W>(pw.w, sh, k.w); break;
    case 1: pad_win_cut<1, W>(pw.w, sh, k.w); break;
    case 2: pad_win_cut<2, W>(pw.w, sh, k.w); break;
    case 3: pad_win_cut<3, W>(pw.w, sh, k.w); break;
    case 4: pad_win_cut<4, W>(pw.w, sh, k.w); break;
    case 5: pad_win_cut<5, W>(pw.w, sh, k.w); break;
    case 6: pad_win_cut<6, W>(pw.w, sh, k.w); break;
    default: pad_win_cut<7, W>(pw.w, sh, k.w); break;
    }
    if (pw.cnt < G) {
#pragma unroll
        for (int i = 0; i < W; ++i) {
            if constexpr (sizeof(T) == 2) {
                if (2 * i >= pw.cnt)
                    k.w[i] = 0u;
                else if (2 * i + 1 >= pw.cnt)
                    k.w[i] &= 0xFFFFu;
            } else if (i >= pw.cnt) {
                k.w[i] = 0u;
            }
        }
    }
}

// Units per thread of the padded quantisers (the window of an MXFP4 block
// is twice as long).
template <int G> constexpr int pad_units() { return G == 16 ? 2 : 1; }

template <typename T>
__global__ void __launch_bounds__(kThreads)
    nvfp4_quantize_padded_kernel(const T *__restrict__ x, int64_t K, FastDiv nbp, int n_blocks,
                                 const float *amax, uint2 *__restrict__ packed,
                                 uint8_t *__restrict__ scales, float *global_scale, int32_t *status)
{
    pdl_begin();
    float g;
    if (!nv_prologue(amax, global_scale, status, g))
        return;
    const NvScaleConsts sc = nv_scale_consts(g);
    const char *x_end = reinterpret_cast<const char *>(x + (int64_t)nbp.div(n_blocks) * K);
    constexpr int U = pad_units<16>();
    PadWin<T, 16> pw[U];
    stream_units<U>(
        n_blocks, [&](int u, int b) { pad_win_load(x, x_end, b, nbp, K, pw[u]); },
        [&](int u, int b) {
            Blk<T, 16> blk;
            pad_win_block(pw[u], blk);
            nv_quantize_block(blk, sc, packed + b, scales + b);
        });
}

template <typename T, bool kCeil>
__global__ void __launch_bounds__(kThreads)
    mxfp4_quantize_padded_kernel(const T *__restrict__ x, int64_t K, FastDiv nbp, int n_blocks,
                                 uint4 *__restrict__ packed, uint8_t *__restrict__ scales,
                                 int32_t *status)
{
    pdl_begin();
    bool bad = false;
    const char *x_end = reinterpret_cast<const char *>(x + (int64_t)nbp.div(n_blocks) * K);
    constexpr int U = pad_units<32>();
    PadWin<T, 32> pw[U];
    stream_units<U>(
        n_blocks, [&](int u, int b) { pad_win_load(x, x_end, b, nbp, K, pw[u]); },
        [&](int u, int b) {
            Blk<T, 32> blk;
            pad_win_block(pw[u], blk);
            mx_quantize_block<kCeil>(blk, packed + b, scales + b, bad);
        });
    if (bad)
        raise_status(status, kStatusNonFinite);
}

// Dequantise a row-padded layout into the logical [R, K] output.  Unit i is
// 16 codes of the padded matrix (row i / nup, columns (i % nup) * 16 ..);
// each thread writes its unit's logical outputs (columns below K) into the
// staged span, then the CTA stores the span: whole 32-byte vectors with
// 256-bit stores (the span starts on a 32-byte boundary of y), the two edge
// vectors, shared with the neighbouring tiles, element by element.
template <bool kNv, typename TOut>
__global__ void __launch_bounds__(kPadTile)
    dequantize_padded_kernel(const uint2 *__restrict__ packed, const uint8_t *__restrict__ scales,
                             const float *__restrict__ global_scale, int64_t K, FastDiv nup,
                             int n_units, TOut *__restrict__ y)
{
    constexpr int kPerVec = 32 / (int)sizeof(TOut);
    extern __shared__ __align__(16) uint32_t sw[];
    uint16_t *sh = reinterpret_cast<uint16_t *>(sw);
    pdl_begin();
    const float g = kNv ? __ldcg(global_scale) : 1.0f;
    const uint64_t g2 = pack2(g, g);
    for (int i0 = (int)blockIdx.x * kPadTile; i0 < n_units; i0 += (int)gridDim.x * kPadTile) {
        const int nu = min(kPadTile, n_units - i0);
        int cnt0, cnt1;
        const int64_t f0 = pad_block_start(i0, nup, K, 16, cnt0);
        const int64_t f1 = pad_block_start(i0 + nu - 1, nup, K, 16, cnt1) + cnt1;
        const int64_t base = span_base(y, f0);
        const int lo = (int)(f0 - base), hi = (int)(f1 - base); // the span, relative to base
        if ((int)threadIdx.x < nu) {
            const int i = i0 + (int)threadIdx.x;
            int cnt;
            const int q = (int)(pad_block_start(i, nup, K, 16, cnt) - base);
            float y16[16];
            dequant_floats<kNv>(__ldcg(packed + i), __ldcg(scales + (kNv ? i : (i >> 1))), g2, y16);
            if constexpr (sizeof(TOut) == 2) {
                uint32_t pr[8]; // bf16 pairs (y[2k], y[2k+1]), low half first
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(pr[k]) : "f"(y16[2 * k + 1]), "f"(y16[2 * k]));
                const int w0 = q >> 1;
                if (cnt == 16 && !(q & 1)) {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        sw[pad_word(w0 + k)] = pr[k];
                } else if (cnt == 16) {
                    // odd start: y[0] is the high half of word w0, y[15] the
                    // low half of word w0 + 8 (the other halves belong to the
                    // neighbouring units); words in between hold (y[2k-1], y[2k])
                    sh[2 * pad_word(w0) + 1] = (uint16_t)pr[0];
#pragma unroll
                    for (int k = 1; k < 8; ++k)
                        sw[pad_word(w0 + k)] = __byte_perm(pr[k - 1], pr[k], 0x5432);
                    sh[2 * pad_word(w0 + 8)] = (uint16_t)(pr[7] >> 16);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (j >= cnt)
                            break;
                        const int e = q + j;
                        sh[2 * pad_word(e >> 1) + (e & 1)] = (uint16_t)(pr[j >> 1] >> (16 * (j & 1)));
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (j >= cnt)
                        break;
                    sw[pad_word(q + j)] = __float_as_uint(y16[j]);
                }
            }
        }
        __syncthreads();
        const int nvec = (hi + kPerVec - 1) / kPerVec;
        for (int v = (int)threadIdx.x; v < nvec; v += (int)blockDim.x) {
            const int e = v * kPerVec;
            if (e >= lo && e + kPerVec <= hi) {
                uint32_t w[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    w[k] = sw[v * 9 + k];
                stg_v8(y + base + e, w);
            } else {
                for (int k = max(lo - e, 0); k < min(kPerVec, hi - e); ++k) {
                    const int ei = e + k;
                    if constexpr (sizeof(TOut) == 2)
                        y[base + ei] = sh[2 * pad_word(ei >> 1) + (ei & 1)];
                    else
                        y[base + ei] = __uint_as_float(sw[pad_word(ei)]);
                }
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Column-wise quantisation.  Tiles of kColTileRows rows x 512 bytes of W
// (256 bf16 or 128 fp32 columns).  A tile row is 128 four-byte words; the
// CTA has 128 threads per block row of the tile (64 / G block rows: 512
// threads for NVFP4, 256 for MXFP4), and thread (j, w) quantises the
// block(s) of block row j in word column w: one fp32 column, or the two bf16
// columns that share the word.  NVFP4 stores its 8-byte blocks straight into
// the output rows; MXFP4 (bound by its stores, not its instructions) stages a
// tile's blocks in shared memory and stores each output row's 32 bytes from
// one thread.
// ---------------------------------------------------------------------------
constexpr int kColWords = 128;
constexpr int kColTileRows = 64;
constexpr int kColTileBytes = kColTileRows * 512;
constexpr int kColStages = 2;
// Staging of one tile's results: packed codes (32 bytes per tile column:
// 4 NVFP4 or 2 MXFP4 blocks) and scale bytes, for up to 256 columns.
constexpr int kColStagePacked = 256 * 32;
constexpr int kColStageBytes = kColStagePacked + 256 * 4;
template <bool kNv> constexpr int col_threads() { return kColWords * (kColTileRows / (kNv ? 16 : 32)); }
constexpr uint32_t kWaitTries = 1u << 22;

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// Bounded wait for phase `parity` of the barrier; false when the tries run out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    for (uint32_t t = 0; t < kWaitTries; ++t) {
        uint32_t done;
        asm volatile("{\n\t"
                     ".reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t"
                     "}"
                     : "=r"(done)
                     : "r"(smem_addr(bar)), "r"(parity)
                     : "memory");
        if (done)
            return true;
    }
    return false;
}

// 2-D TMA tile load of box (x = column, y = row) into shared memory,
// completing on `bar`.  x is a multiple of 512 bytes' worth of elements.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
                 : "memory");
}

// Tile t of the column-wise pass: column tile t % n_tc, row tile t / n_tc
// (consecutive CTAs sweep across the columns of one row band together).
struct ColTile {
    int r0, c0;
};

__device__ __forceinline__ ColTile col_tile(int t, int n_tc, int tile_cols)
{
    const int tr = t / n_tc;
    return {tr * kColTileRows, (t - tr * n_tc) * tile_cols};
}

// Quantises the G-element blocks of the tile rows [j*G, j*G + G) in this
// thread's columns and stores them straight into the output rows (= columns
// of W): the NVFP4 pass, which is bound by its instruction issue, not by
// these partial-sector stores.
template <typename T, bool kNv, bool kCeil, int G>
__device__ __forceinline__ void column_blocks_direct(const uint8_t *tile, int j, int w, int c_first, int C,
                                              int blk, const NvScaleConsts &sc, uint8_t *packed,
                                              uint8_t *scales, int64_t prow, int nbo, bool &bad)
{
    constexpr int kPerThread = 4 / (int)sizeof(T); // columns per word: 2 (bf16) or 1 (fp32)
    const uint32_t *tw = reinterpret_cast<const uint32_t *>(tile) + j * G * kColWords + w;
    uint32_t rowv[G]; // row i of this thread's word column
#pragma unroll
    for (int i = 0; i < G; ++i)
        rowv[i] = tw[i * kColWords];
#pragma unroll
    for (int p = 0; p < kPerThread; ++p) {
        const int c = c_first + p;
        if (c >= C)
            continue;
        Blk<T, G> b;
        if constexpr (sizeof(T) == 2) {
            // bf16: a word holds columns 2t (low half) and 2t+1 (high half);
            // gather one column's halves of rows 2i, 2i+1 into word i.
#pragma unroll
            for (int i = 0; i < G / 2; ++i)
                b.w[i] = __byte_perm(rowv[2 * i], rowv[2 * i + 1], p ? 0x7632 : 0x5410);
        } else {
#pragma unroll
            for (int i = 0; i < G; ++i)
                b.w[i] = rowv[i];
        }
        uint8_t *orow = packed + (int64_t)c * prow;
        if constexpr (kNv)
            nv_quantize_block(b, sc, reinterpret_cast<uint2 *>(orow) + blk, scales + (int64_t)c * nbo + blk);
        else
            mx_quantize_block<kCeil>(b, reinterpret_cast<uint4 *>(orow) + blk,
                                     scales + (int64_t)c * nbo + blk, bad);
    }
}

// Quantises the G-element blocks of the tile rows [j*G, j*G + G) in this
// thread's columns into the staging tile: packed codes of block row j and
// tile column c at stage_p + (j * kCols + c) * G/2, its scale byte at
// stage_s[j * kCols + c] (block-row-major: a warp's writes are consecutive).
template <typename T, bool kNv, bool kCeil, int G>
__device__ __forceinline__ void column_blocks(const uint8_t *tile, int j, int w, const NvScaleConsts &sc,
                                              uint8_t *stage_p, uint8_t *stage_s, bool &bad)
{
    constexpr int kPerThread = 4 / (int)sizeof(T); // columns per word: 2 (bf16) or 1 (fp32)
    constexpr int kCols = kColWords * kPerThread;
    const uint32_t *tw = reinterpret_cast<const uint32_t *>(tile) + j * G * kColWords + w;
    uint32_t rowv[G]; // row i of this thread's word column
#pragma unroll
    for (int i = 0; i < G; ++i)
        rowv[i] = tw[i * kColWords];
#pragma unroll
    for (int p = 0; p < kPerThread; ++p) {
        const int c = w * kPerThread + p; // tile column
        Blk<T, G> b;
        if constexpr (sizeof(T) == 2) {
            // bf16: a word holds columns 2t (low half) and 2t+1 (high half);
            // gather one column's halves of rows 2i, 2i+1 into word i.
#pragma unroll
            for (int i = 0; i < G / 2; ++i)
                b.w[i] = __byte_perm(rowv[2 * i], rowv[2 * i + 1], p ? 0x7632 : 0x5410);
        } else {
#pragma unroll
            for (int i = 0; i < G; ++i)
                b.w[i] = rowv[i];
        }
        uint8_t *dp = stage_p + (j * kCols + c) * (G / 2);
        uint8_t *ds = stage_s + j * kCols + c;
        if constexpr (kNv)
            nv_quantize_block(b, sc, reinterpret_cast<uint2 *>(dp), ds);
        else
            mx_quantize_block<kCeil>(b, reinterpret_cast<uint4 *>(dp), ds, bad);
    }
}

// Stores tile column c's staged blocks: kBR blocks of G/2 bytes (32 bytes)
// contiguous in output row c, and their kBR scale bytes; only the n_valid
// first ones when the column is cut by the padded length.  wide: the row's
// 32 bytes start on a 32-byte boundary.
template <int G, int kCols>
__device__ __forceinline__ void column_store(const uint8_t *stage_p, const uint8_t *stage_s, int c,
                                             uint8_t *orow, uint8_t *srow, int n_valid, bool wide)
{
    constexpr int kBR = kColTileRows / G; // block rows per tile: 4 (NVFP4) or 2 (MXFP4)
    constexpr int kBytes = G / 2;         // packed bytes per block: 8 or 16
    uint32_t wds[8];
#pragma unroll
    for (int j = 0; j < kBR; ++j) {
        const uint32_t *src = reinterpret_cast<const uint32_t *>(stage_p + (j * kCols + c) * kBytes);
#pragma unroll
        for (int i = 0; i < kBytes / 4; ++i)
            wds[j * (kBytes / 4) + i] = src[i];
    }
    if (n_valid == kBR && wide) {
        stg_v8(orow, wds);
    } else {
#pragma unroll
        for (int j = 0; j < kBR; ++j)
            if (j < n_valid) {
#pragma unroll
                for (int i = 0; i < kBytes / 8; ++i)
                    *reinterpret_cast<uint2 *>(orow + j * kBytes + 8 * i) =
                        make_uint2(wds[j * (kBytes / 4) + 2 * i], wds[j * (kBytes / 4) + 2 * i + 1]);
            }
    }
#pragma unroll
    for (int j = 0; j < kBR; ++j)
        if (j < n_valid)
            srow[j] = stage_s[j * kCols + c];
}

template <typename T, bool kNv, bool kCeil>
__global__ void __launch_bounds__(col_threads<kNv>())
    quantize_columns_kernel(const __grid_constant__ CUtensorMap map, int R, int C, int n_tiles,
                            const float *amax, uint8_t *__restrict__ packed,
                            uint8_t *__restrict__ scales, float *global_scale, int32_t *status)
{
    constexpr int G = kNv ? 16 : 32;
    constexpr int kCols = 512 / (int)sizeof(T);          // tile columns
    constexpr int kPerWord = 4 / (int)sizeof(T);         // columns per 4-byte word
    constexpr int kWarps = col_threads<kNv>() / 32;
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ __align__(8) uint64_t full[kColStages];  // tile landed (TMA bytes)
    __shared__ __align__(8) uint64_t empty[kColStages]; // every warp is done with the tile

    pdl_begin();
    float g = 1.0f;
    if constexpr (kNv) {
        if (!nv_prologue(amax, global_scale, status, g))
            return;
    }
    const NvScaleConsts sc = nv_scale_consts(g);
    const int n_tc = (C + kCols - 1) / kCols;
    const int Rp = (R + G - 1) / G * G;                  // padded column length
    const int64_t prow = Rp / 2;                         // packed bytes per output row
    const int nbo = Rp / G;                              // blocks (scale bytes) per output row
    const int first_tile = blockIdx.x;
    const int stride = gridDim.x;
    const int w = (int)threadIdx.x % kColWords;          // word column of the tile
    const int jb = (int)threadIdx.x / kColWords;         // block row of the tile
    const bool producer = threadIdx.x == 0;

    if (producer) {
        for (int s = 0; s < kColStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    int issued = 0; // tiles of this CTA whose copy thread 0 has started
    if (producer) {
        for (int s = 0; s < kColStages; ++s) {
            const int t = first_tile + s * stride;
            if (t < n_tiles) {
                const ColTile ct = col_tile(t, n_tc, kCols);
                mbar_expect_tx(&full[s], kColTileBytes);
                tma_load_2d(smem + s * kColTileBytes, &map, ct.c0, ct.r0, &full[s]);
                ++issued;
            }
        }
    }
    bool bad = false, timed_out = false;
    int k = 0;
    if constexpr (kNv) {
        // Each warp waits for its tiles on full[s], releases them on empty[s];
        // thread 0 refills a stage once every warp has released it.  All waits
        // are bounded; a thread that gives up leaves the loop, and every wait
        // that depended on it then runs out in turn.
        for (int t = first_tile; t < n_tiles; t += stride, ++k) {
            const int s = k % kColStages;
            const uint32_t phase = (uint32_t)(k / kColStages) & 1u;
            if (!mbar_wait(&full[s], phase)) {
                timed_out = true;
                break;
            }
            const ColTile ct = col_tile(t, n_tc, kCols);
            const int blk_row = ct.r0 + jb * G;
            if (blk_row < R)
                column_blocks_direct<T, kNv, kCeil, G>(smem + s * kColTileBytes, jb, w, ct.c0 + w * kPerWord,
                                                       C, blk_row / G, sc, packed, scales, prow, nbo, bad);
            __syncwarp();
            if ((threadIdx.x & 31) == 0)
                mbar_arrive(&empty[s]);
            if (producer) {
                const int tn = t + kColStages * stride;
                if (tn < n_tiles) {
                    if (!mbar_wait(&empty[s], phase)) {
                        timed_out = true;
                        break;
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    const ColTile cn = col_tile(tn, n_tc, kCols);
                    mbar_expect_tx(&full[s], kColTileBytes);
                    tma_load_2d(smem + s * kColTileBytes, &map, cn.c0, cn.r0, &full[s]);
                    ++issued;
                }
            }
        }
    } else {
        // MXFP4, bound by its stores: per tile every thread waits (bounded)
        // for the tile on full[s], and the CTA votes: if any wait ran out,
        // all threads leave the loop together (the barriers below must be
        // reached by all or none).  The threads quantise their blocks into
        // the staging tile, release the TMA stage (each warp on empty[s]),
        // and after a barrier thread c < kCols stores tile column c's
        // blocks: 32 contiguous bytes of one output row instead of 16 bytes
        // from each of two warps.  Thread 0 refills the stage once every warp
        // has released it; a refill wait that runs out goes into the next
        // vote.
        uint8_t *stage_p = smem + kColStages * kColTileBytes;
        uint8_t *stage_s = stage_p + kColStagePacked;
        const bool wide = (reinterpret_cast<uintptr_t>(packed) % 32u) == 0 && prow % 32 == 0;
        for (int t = first_tile; t < n_tiles; t += stride, ++k) {
            const int s = k % kColStages;
            const uint32_t phase = (uint32_t)(k / kColStages) & 1u;
            const bool ok = !timed_out && mbar_wait(&full[s], phase);
            if (__syncthreads_or(!ok)) {
                timed_out = true;
                break;
            }
            const ColTile ct = col_tile(t, n_tc, kCols);
            if (ct.r0 + jb * G < R)
                column_blocks<T, kNv, kCeil, G>(smem + s * kColTileBytes, jb, w, sc, stage_p, stage_s, bad);
            __syncwarp();
            if ((threadIdx.x & 31) == 0)
                mbar_arrive(&empty[s]);
            __syncthreads(); // staging tile complete
            const int c = (int)threadIdx.x;
            const int blk0 = ct.r0 / G;
            if (c < kCols && ct.c0 + c < C) {
                const int n_valid = nbo - blk0 < kColTileRows / G ? nbo - blk0 : kColTileRows / G;
                const int64_t oc = ct.c0 + c;
                column_store<G, kCols>(stage_p, stage_s, c, packed + oc * prow + (int64_t)blk0 * (G / 2),
                                       scales + oc * nbo + blk0, n_valid, wide);
            }
            if (producer) {
                const int tn = t + kColStages * stride;
                if (tn < n_tiles) {
                    if (!mbar_wait(&empty[s], phase)) {
                        timed_out = true; // the next vote ends the loop for everyone
                    } else {
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        const ColTile cn = col_tile(tn, n_tc, kCols);
                        mbar_expect_tx(&full[s], kColTileBytes);
                        tma_load_2d(smem + s * kColTileBytes, &map, cn.c0, cn.r0, &full[s]);
                        ++issued;
                    }
                }
            }
        }
    }
    if (timed_out)
        raise_status(status, kStatusTimeout);
    if (producer) {
        // Before the CTA can end, every copy thread 0 started must have
        // landed: wait (bounded) for those not consumed above.
        for (int j = k; j < issued; ++j)
            (void)mbar_wait(&full[j % kColStages], (uint32_t)(j / kColStages) & 1u);
    }
    if (bad)
        raise_status(status, kStatusNonFinite);
}

} // namespace fp4
