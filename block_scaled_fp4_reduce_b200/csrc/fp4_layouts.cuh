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
// The column-wise quantisers read W straight from global memory: a CTA
// takes a tile of 256 rows x a 128-byte strip, every lane of a warp one
// 4-byte word column of 32 rows (one coalesced 128-byte row segment per warp
// load), quantises the blocks of its columns in registers and stages them in
// shared memory, from where the CTA stores whole output rows with wide
// stores.  Rows past R read as +0, which is the padding.  No kernel here
// waits on another thread beyond __syncthreads.
#pragma once

#include <cstdint>

#include "fp4_kernels.cuh"

namespace fp4 {

// ---------------------------------------------------------------------------
// Ragged rows.  Block b of the row-padded [R, Kp] matrix is row b / nbp,
// block b % nbp of that row; it covers the elements [f, f + cnt) of the flat
// input, f = (b / nbp) K + (b % nbp) G, cnt = min(G, K - (b % nbp) G), and
// reads +0 past them.  The quantisers read every block from its window of
// aligned 32-byte vectors in registers (PadWin below); the dequantiser
// writes whole aligned vectors of y assembled across a warp with shuffles
// (dequantize_padded_kernel).
// ---------------------------------------------------------------------------
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

// First flat element of block b, its element count and its row.
__device__ __forceinline__ int64_t pad_block_start(int b, const FastDiv &nbp, int64_t K, int G, int &cnt, int &r)
{
    r = nbp.div(b);
    const int j = b - r * (int)nbp.d;
    const int64_t c0 = (int64_t)j * G;
    cnt = (int)min((int64_t)G, K - c0);
    return (int64_t)r * K + c0;
}

__device__ __forceinline__ int64_t pad_block_start(int b, const FastDiv &nbp, int64_t K, int G, int &cnt)
{
    int r;
    return pad_block_start(b, nbp, K, G, cnt, r);
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
    if constexpr (sizeof(T) == 2) {
        // whole warp steps take the warp-shared exact path
        __shared__ NvExactQueue<U> queues[kThreads / 32];
        NvExactQueue<U> &q = queues[threadIdx.x >> 5];
        stream_units_warp<U>(
            n_blocks,
            [&](int b0, int stride) {
                PadWin<T, 16> pw[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    pad_win_load(x, x_end, b0 + u * stride, nbp, K, pw[u]);
                Blk<T, 16> blk[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    pad_win_block(pw[u], blk[u]);
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
                PadWin<T, 16> pw;
                pad_win_load(x, x_end, b, nbp, K, pw);
                Blk<T, 16> blk;
                pad_win_block(pw, blk);
                nv_quantize_block(blk, sc, packed + b, scales + b);
            });
    } else {
        PadWin<T, 16> pw[U];
        stream_units<U>(
            n_blocks, [&](int u, int b) { pad_win_load(x, x_end, b, nbp, K, pw[u]); },
            [&](int u, int b) {
                Blk<T, 16> blk;
                pad_win_block(pw[u], blk);
                nv_quantize_block(blk, sc, packed + b, scales + b);
            });
    }
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
// 16 codes of the padded matrix (row i / nup, columns (i % nup) * 16 ..).
// The outputs of consecutive units are contiguous in y, and every unit of a
// row starts at the same offset s within a 32-byte vector (units are 16
// elements apart), so the aligned vector(s) that start s bytes before unit u
// hold the tail of unit u - 1 and the head of unit u.  A warp takes a chunk
// of 31 units, u = 31 c .. 31 c + 30, and its 32 lanes decode units 31 c - 1
// .. 31 c + 30: lane L >= 1 moves the tail of lane L - 1's unit over with a
// shuffle, joins it to its own head and writes the whole vector(s) with
// 256-bit stores; lane 0 only supplies its unit's tail.  So every vector
// inside a run of such chunks is written once, whole, by one lane (no
// partial edge stores: every store is an L2 write request, and the partial
// stores at both edges of 32-unit chunks cost 3.03 M requests against 1.84 M
// for the row dequantiser on 8192 x 14335).  A chunk whose 32 decoded units
// are not all whole (16 logical elements) in one row -- a row boundary, a
// partial unit, the first chunk of a launch, the end of the launch -- writes
// every decoded unit's logical elements one by one; the bytes it shares with
// a neighbouring chunk's vectors are then written twice with the same values.
template <int K4, int W>
__device__ __forceinline__ void pad_join(const uint32_t (&q)[2 * W], uint32_t sh, uint32_t *out)
{
    // out[j] = the words of q from word W - K4 on, shifted right by sh bits
#pragma unroll
    for (int j = 0; j < W; ++j)
        out[j] = __funnelshift_r(q[W - K4 + j], q[W - K4 + j + 1], sh);
}

template <typename TOut> __device__ __forceinline__ void pad_store_elem(TOut *y, int64_t e, uint32_t word, int half)
{
    if constexpr (sizeof(TOut) == 2)
        y[e] = (uint16_t)(word >> (16 * half));
    else
        y[e] = __uint_as_float(word);
}

constexpr int kPadDqChunks = 4; // chunks per warp whose loads go out together
constexpr int kPadDqStep = 31;  // units a chunk stores (its 32 lanes decode one unit more)

template <bool kNv, typename TOut>
__global__ void __launch_bounds__(kThreads)
    dequantize_padded_kernel(const uint2 *__restrict__ packed, const uint8_t *__restrict__ scales,
                             const float *__restrict__ global_scale, int64_t K, FastDiv nup,
                             int n_units, TOut *__restrict__ y)
{
    constexpr int kE = (int)sizeof(TOut);
    constexpr int kW = 16 * kE / 4; // output words of a unit: 8 (bf16) or 16 (fp32)
    pdl_begin();
    const float g = kNv ? __ldcg(global_scale) : 1.0f;
    const uint64_t g2 = pack2(g, g);
    const int lane = (int)(threadIdx.x & 31u);
    constexpr int U = kPadDqChunks;
    const int n_warps = (int)(gridDim.x * (blockDim.x >> 5));
    const int n_chunks = (n_units + kPadDqStep - 1) / kPadDqStep;
    uint2 pkv[U];
    uint32_t sbv[U];
    int slot = 0;
    for (int c = (int)(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)); c < n_chunks;
         c += n_warps, slot = (slot + 1) % U) {
        // the codes and scale bytes of the next U chunks, loaded together
        if (slot == 0) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int cu = c + u * n_warps;
                const int iu = cu * kPadDqStep - 1 + lane;
                if (cu < n_chunks && iu >= 0 && iu < n_units) {
                    pkv[u] = __ldcg(packed + iu);
                    sbv[u] = __ldcg(scales + (kNv ? iu : (iu >> 1)));
                }
            }
        }
        const int i = c * kPadDqStep - 1 + lane; // lane 0: the unit before the chunk
        const bool valid = i >= 0 && i < n_units;
        int cnt = 0;
        int row = -1;
        int64_t f = 0;
        uint32_t o[kW];
        if (valid) {
            f = pad_block_start(i, nup, K, 16, cnt, row);
            uint2 pk = pkv[0];
            uint32_t sbyte = sbv[0];
#pragma unroll
            for (int u = 1; u < U; ++u)
                if (slot == u) {
                    pk = pkv[u];
                    sbyte = sbv[u];
                }
            float y16[16];
            dequant_floats<kNv>(pk, sbyte, g2, y16);
            if constexpr (kE == 2) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[k]) : "f"(y16[2 * k + 1]), "f"(y16[2 * k]));
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    o[k] = __float_as_uint(y16[k]);
            }
        }
        const int row0 = __shfl_sync(0xFFFFFFFFu, row, 0);
        if (__all_sync(0xFFFFFFFFu, valid && cnt == 16 && row == row0)) {
            const uintptr_t start = reinterpret_cast<uintptr_t>(y + f);
            const int sb = (int)(start & 31u); // the same in every lane
            uint8_t *vec = reinterpret_cast<uint8_t *>(start - (uintptr_t)sb);
            if (sb == 0) {
                if (lane > 0) {
#pragma unroll
                    for (int v = 0; v < kW / 8; ++v)
                        stg_v8(vec + 32 * v, o + 8 * v);
                }
                continue;
            }
            uint32_t q[2 * kW];
#pragma unroll
            for (int k = 0; k < kW; ++k) {
                q[k] = __shfl_up_sync(0xFFFFFFFFu, o[k], 1);
                q[kW + k] = o[k];
            }
            uint32_t out[kW]; // the aligned vector(s) holding the tail of unit L-1 and the head of unit L
            const uint32_t sh = (uint32_t)((32 - sb) & 3) * 8u;
            switch ((sb + 3) >> 2) { // words of unit L-1 in the first vector
            case 1: pad_join<1, kW>(q, sh, out); break;
            case 2: pad_join<2, kW>(q, sh, out); break;
            case 3: pad_join<3, kW>(q, sh, out); break;
            case 4: pad_join<4, kW>(q, sh, out); break;
            case 5: pad_join<5, kW>(q, sh, out); break;
            case 6: pad_join<6, kW>(q, sh, out); break;
            case 7: pad_join<7, kW>(q, sh, out); break;
            default: pad_join<8, kW>(q, sh, out); break;
            }
            if (lane > 0) {
#pragma unroll
                for (int v = 0; v < kW / 8; ++v)
                    stg_v8(vec + 32 * v, out + 8 * v);
            }
        } else if (valid) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
                if (e < cnt)
                    pad_store_elem(y, f + e, o[e * kE / 4], kE == 2 ? (e & 1) : 0);
        }
    }
}

// ---------------------------------------------------------------------------
// Column-wise NVFP4, straight from global memory, results staged in shared
// memory.  A CTA takes a tile of 256 rows x one 128-byte strip of W (64
// bf16 or 32 fp32 columns); warp k quantises rows [32k, 32k + 32) of it:
// each lane loads its 4-byte word of 16 rows at a time (one coalesced
// 128-byte row segment per warp load), assembles the 16-row block of each
// of its columns in registers and quantises it.  The blocks go to a staging
// tile in shared memory, one 128-byte row per output row (column of W), and
// after a barrier the CTA stores every output row's 128 bytes of codes and
// 16 scale bytes with 32-byte and 4-byte stores.  Every global store is an
// L2 write request: storing each lane's blocks straight into its two output
// rows took four requests per 32 rows and column, against 2 / 64 here, and
// the stores, not the loads or the arithmetic, bounded that kernel.  Staging
// is double-buffered, so one barrier per tile suffices: a warp that reaches
// the next-but-one tile has passed the barrier that every warp reaches only
// after storing this tile.  Rows past R read as +0 (the padding); blocks past
// the padded column length are not stored.
// ---------------------------------------------------------------------------
constexpr int kNvColRows = 256;               // rows of W per tile: 8 warps x 32 rows
constexpr int kNvColBlocks = kNvColRows / 16; // blocks per output row per tile
constexpr int kNvColCtasPerSm = 4;
static_assert(kNvColRows == 32 * (kThreads / 32), "one warp per 32 rows of a tile");
static_assert(kNvColBlocks * 8 == 128, "a tile's output row is 128 bytes of codes");

// Store layout flags of the column-wise NVFP4 outputs (host computed).
constexpr int kColPacked32 = 1; // every output row's packed bytes start 32-byte aligned
constexpr int kColPacked16 = 2; // ... 16-byte aligned
constexpr int kColScales4 = 4;  // every output row's scale bytes start 4-byte aligned

// Staging-tile position (8-byte chunk) of block j of tile column cl: chunk j
// of the column's 128-byte row, XOR-swizzled so that the 16 lanes of a
// half-warp storing one block each of 16 different columns hit all 32 banks
// once, and the 8 rows x 4 quarter rows read by a warp in the store phase
// hit every bank exactly twice (the minimum for 256 bytes).
template <int kPerWord> __device__ __forceinline__ int col_swizzle(int cl)
{
    return kPerWord == 2 ? (((cl >> 1) ^ ((cl & 1) << 3)) & 15) : (cl & 15);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, kNvColCtasPerSm)
    nvfp4_quantize_columns_kernel(const uint32_t *__restrict__ xw, int R, int Cw, int C,
                                  const float *amax, uint8_t *__restrict__ packed,
                                  uint8_t *__restrict__ scales, float *global_scale, int32_t *status,
                                  int layout)
{
    constexpr int kPerWord = 4 / (int)sizeof(T); // columns per word
    constexpr int kTileCols = 32 * kPerWord;     // columns of W (output rows) per tile
    constexpr int kScaleRow = 20;                // staged scale bytes per output row (16 + 4 of padding)
    __shared__ __align__(16) uint8_t st_packed[2][kTileCols * 128];
    __shared__ __align__(16) uint8_t st_scales[2][kTileCols * kScaleRow];
    __shared__ NvExactQueue<kPerWord> queues[sizeof(T) == 2 ? kThreads / 32 : 1];
    pdl_begin();
    float g;
    if (!nv_prologue(amax, global_scale, status, g))
        return;
    const NvScaleConsts sc = nv_scale_consts(g);
    const int lane = (int)(threadIdx.x & 31u), warp = (int)(threadIdx.x >> 5);
    const int n_strips = (Cw + 31) / 32;
    const int n_tiles = ((R + kNvColRows - 1) / kNvColRows) * n_strips;
    const int nbo = (R + 15) / 16;         // blocks (scale bytes) per output row
    const int64_t prow = (int64_t)nbo * 8; // packed bytes per output row
    int s = 0;
    for (int tile = (int)blockIdx.x; tile < n_tiles; tile += (int)gridDim.x, s ^= 1) {
        const int band = tile / n_strips;
        const int strip = tile - band * n_strips;
        const int w = strip * 32 + lane;                     // word column of W
        const int r0 = band * kNvColRows + warp * 32;      // this warp's first row
        if (w < Cw && r0 < R) {
            // all 32 lanes here (the strip is whole): the warp-shared exact path
            const bool whole_warp = strip * 32 + 32 <= Cw;
            uint32_t sb2[kPerWord]; // the two scale bytes of each column
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int rh = r0 + 16 * h;
                uint32_t v[16];
                const uint32_t *src = xw + (int64_t)rh * Cw + w;
                if (rh + 16 <= R) {
#pragma unroll
                    for (int i = 0; i < 16; ++i, src += Cw)
                        v[i] = __ldcg(src);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i, src += Cw)
                        v[i] = rh + i < R ? __ldcg(src) : 0u;
                }
                Blk<T, 16> b[kPerWord];
#pragma unroll
                for (int p = 0; p < kPerWord; ++p) {
                    if constexpr (sizeof(T) == 2) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            b[p].w[i] = __byte_perm(v[2 * i], v[2 * i + 1], p ? 0x7632 : 0x5410);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            b[p].w[i] = v[i];
                    }
                }
                uint2 q[kPerWord];
                uint32_t sbyte[kPerWord];
                if constexpr (sizeof(T) == 2) {
                    if (whole_warp) {
                        nv_quantize_warp(b, sc, queues[warp], q, sbyte);
                    } else {
#pragma unroll
                        for (int p = 0; p < kPerWord; ++p)
                            q[p] = nv_block_quantize(b[p], sc, sbyte[p]);
                    }
                } else {
#pragma unroll
                    for (int p = 0; p < kPerWord; ++p)
                        q[p] = nv_block_quantize(b[p], sc, sbyte[p]);
                }
#pragma unroll
                for (int p = 0; p < kPerWord; ++p) {
                    const int cl = lane * kPerWord + p;
                    const int chunk = (2 * warp + h) ^ col_swizzle<kPerWord>(cl);
                    *reinterpret_cast<uint2 *>(&st_packed[s][cl * 128 + 8 * chunk]) = q[p];
                    sb2[p] = h ? sb2[p] | (sbyte[p] << 8) : sbyte[p];
                }
            }
#pragma unroll
            for (int p = 0; p < kPerWord; ++p) {
                const int cl = lane * kPerWord + p;
                *reinterpret_cast<uint16_t *>(&st_scales[s][cl * kScaleRow + 2 * warp]) = (uint16_t)sb2[p];
            }
        }
        __syncthreads();
        // store phase: four threads per output row, a quarter row each
        const int b0 = band * kNvColBlocks;     // first block of the tile in an output row
        const int nbt = min(kNvColBlocks, nbo - b0); // blocks of the tile inside the padded length
        for (int t = (int)threadIdx.x; t < kTileCols * 4; t += kThreads) {
            const int cl = t >> 2, qr = t & 3;
            const int c = strip * kTileCols + cl;
            if (c >= C || 4 * qr >= nbt)
                continue;
            const int f = col_swizzle<kPerWord>(cl);
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint2 q = *reinterpret_cast<const uint2 *>(&st_packed[s][cl * 128 + 8 * ((4 * qr + i) ^ f)]);
                o[2 * i] = q.x;
                o[2 * i + 1] = q.y;
            }
            const int nq = min(4, nbt - 4 * qr); // blocks of this quarter row inside the padded length
            uint8_t *orow = packed + (int64_t)c * prow + (int64_t)(b0 + 4 * qr) * 8;
            if (nq == 4 && (layout & kColPacked32)) {
                stg_v8(orow, o);
            } else if (layout & kColPacked16) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    if (2 * k + 2 <= nq)
                        reinterpret_cast<uint4 *>(orow)[k] = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
                    else if (2 * k < nq)
                        reinterpret_cast<uint2 *>(orow)[2 * k] = make_uint2(o[4 * k], o[4 * k + 1]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (k < nq)
                        reinterpret_cast<uint2 *>(orow)[k] = make_uint2(o[2 * k], o[2 * k + 1]);
            }
            const uint32_t sw = *reinterpret_cast<const uint32_t *>(&st_scales[s][cl * kScaleRow + 4 * qr]);
            uint8_t *srow = scales + (int64_t)c * nbo + b0 + 4 * qr;
            if (nq == 4 && (layout & kColScales4)) {
                *reinterpret_cast<uint32_t *>(srow) = sw;
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (k < nq)
                        srow[k] = (uint8_t)(sw >> (8 * k));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Column-wise MXFP4, the same way: a CTA takes a tile of 256 rows x one
// 128-byte strip of W, warp k rows [32k, 32k + 32) -- one 32-row block per
// column -- each lane its 4-byte word of all 32 rows (32 coalesced row
// segments per warp in flight).  The blocks are staged in shared memory, 16
// bytes each, 8 per output row, 16-byte chunks XOR-swizzled (chunk k of
// column c at k ^ ((c >> 1) & 7) ^ (c & 1)) so that the eight lanes of a
// quarter-warp writing one block each, and the eight threads of a quarter-warp
// reading two rows' quarters in the store phase, hit eight different chunks;
// after one barrier per tile the CTA stores each output row's 128 bytes with
// 32-byte stores and its 8 scale bytes with 4-byte stores.  Rows past R read
// as +0; blocks past the padded column length are not stored.
// ---------------------------------------------------------------------------
constexpr int kMxColRows = 256;                 // rows of W per tile: 8 warps x 32 rows
constexpr int kMxColBlocks = kMxColRows / 32;   // blocks per output row per tile
constexpr int kMxColCtasPerSm = 3;
static_assert(kMxColRows == 32 * (kThreads / 32), "one warp per 32 rows of a tile");

template <int kPerWord> __device__ __forceinline__ int mx_col_swizzle(int cl)
{
    return kPerWord == 2 ? (((cl >> 1) & 7) ^ (cl & 1)) : (cl & 7);
}

template <typename T, bool kCeil>
__global__ void __launch_bounds__(kThreads, kMxColCtasPerSm)
    mxfp4_quantize_columns_kernel(const uint32_t *__restrict__ xw, int R, int Cw, int C,
                                         uint8_t *__restrict__ packed, uint8_t *__restrict__ scales,
                                         int32_t *status, int layout)
{
    constexpr int kPerWord = 4 / (int)sizeof(T); // columns per word
    constexpr int kTileCols = 32 * kPerWord;     // columns of W (output rows) per tile
    __shared__ __align__(16) uint8_t st_packed[2][kTileCols * 128];
    __shared__ __align__(16) uint8_t st_scales[2][kTileCols * 8];
    pdl_begin();
    const int lane = (int)(threadIdx.x & 31u), warp = (int)(threadIdx.x >> 5);
    const int n_strips = (Cw + 31) / 32;
    const int n_tiles = ((R + kMxColRows - 1) / kMxColRows) * n_strips;
    const int nbo = (R + 31) / 32;          // blocks (scale bytes) per output row
    const int64_t prow = (int64_t)nbo * 16; // packed bytes per output row
    bool bad = false;
    int s = 0;
    for (int tile = (int)blockIdx.x; tile < n_tiles; tile += (int)gridDim.x, s ^= 1) {
        const int band = tile / n_strips;
        const int strip = tile - band * n_strips;
        const int w = strip * 32 + lane;                 // word column of W
        const int r0 = band * kMxColRows + warp * 32;    // this warp's first row
        if (w < Cw && r0 < R) {
            uint32_t v[32];
            const uint32_t *src = xw + (int64_t)r0 * Cw + w;
            if (r0 + 32 <= R) {
#pragma unroll
                for (int i = 0; i < 32; ++i, src += Cw)
                    v[i] = __ldcg(src);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i, src += Cw)
                    v[i] = r0 + i < R ? __ldcg(src) : 0u;
            }
#pragma unroll
            for (int p = 0; p < kPerWord; ++p) {
                Blk<T, 32> b;
                if constexpr (sizeof(T) == 2) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        b.w[i] = __byte_perm(v[2 * i], v[2 * i + 1], p ? 0x7632 : 0x5410);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        b.w[i] = v[i];
                }
                uint4 q;
                uint8_t sbyte;
                mx_quantize_block<kCeil>(b, &q, &sbyte, bad);
                const int cl = lane * kPerWord + p;
                const int chunk = warp ^ mx_col_swizzle<kPerWord>(cl);
                *reinterpret_cast<uint4 *>(&st_packed[s][cl * 128 + 16 * chunk]) = q;
                st_scales[s][cl * 8 + warp] = sbyte;
            }
        }
        __syncthreads();
        // store phase: four threads per output row, a quarter row (two blocks) each
        const int b0 = band * kMxColBlocks;             // first block of the tile in an output row
        const int nbt = min(kMxColBlocks, nbo - b0);    // blocks of the tile inside the padded length
        for (int t = (int)threadIdx.x; t < kTileCols * 4; t += kThreads) {
            const int cl = t >> 2, qr = t & 3;
            const int c = strip * kTileCols + cl;
            const int nq = min(2, nbt - 2 * qr); // blocks of this quarter row inside the padded length
            if (c >= C || nq <= 0)
                continue;
            const int f = mx_col_swizzle<kPerWord>(cl);
            const uint4 q0 = *reinterpret_cast<const uint4 *>(&st_packed[s][cl * 128 + 16 * ((2 * qr) ^ f)]);
            const uint4 q1 = *reinterpret_cast<const uint4 *>(&st_packed[s][cl * 128 + 16 * ((2 * qr + 1) ^ f)]);
            uint8_t *orow = packed + (int64_t)c * prow + (int64_t)(b0 + 2 * qr) * 16;
            if (nq == 2 && (layout & kColPacked32)) {
                const uint32_t o[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                stg_v8(orow, o);
            } else {
                reinterpret_cast<uint4 *>(orow)[0] = q0;
                if (nq == 2)
                    reinterpret_cast<uint4 *>(orow)[1] = q1;
            }
            if (qr < 2) { // scale bytes 4 qr .. 4 qr + 3 of the row
                const int ns = min(4, nbt - 4 * qr);
                if (ns > 0) {
                    const uint32_t sw = *reinterpret_cast<const uint32_t *>(&st_scales[s][cl * 8 + 4 * qr]);
                    uint8_t *srow = scales + (int64_t)c * nbo + b0 + 4 * qr;
                    if (ns == 4 && (layout & kColScales4)) {
                        *reinterpret_cast<uint32_t *>(srow) = sw;
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            if (j < ns)
                                srow[j] = (uint8_t)(sw >> (8 * j));
                    }
                }
            }
        }
    }
    if (bad)
        raise_status(status, kStatusNonFinite);
}

} // namespace fp4
