// fp4_gemm.cuh -- the consumer of the quantised operands on the tensor cores.
//
// "NVFP4 与 MXFP4 格式" section 6: for Y = X W with X [M, K] and W [K, N]
// both blocked along K, an output element is g_X g_W sum over blocks of
// s_X s_W (sum of the block's payload products): the block scales can only
// be taken out of one block's dot product.  The sm100 block-scaled MMA
// (tcgen05.mma kind::mxf4nvf4, block16) computes exactly that sum with the
// E2M1 payloads and the E4M3 block scales as operands and an fp32
// accumulator in tensor memory; the global scales multiply the result.
//
//   scales_to_mma_kernel  block scales [rows, K/16] (plain, as the quantisers
//                         write them) -> the tiled layout the MMA reads:
//                         128-row x 4-block tiles of 512 bytes, row r = r0 +
//                         32 r1 and block j of a tile at byte 16 r0 + 4 r1 + j,
//                         tiles row-tile-major with the block tiles
//                         contiguous; padding 0 (the sm100 block-scaled
//                         layout; it is not on the pages)
//   nvfp4_gemm_kernel     D [M, N] fp32 = g_a g_b A B^T for NVFP4 A [M, K]
//                         and B [N, K] (both K-major, i.e. blocked along K),
//                         one CTA per 128 x 128 tile of D
//   nvfp4_gemm_pair_kernel the same on persistent clusters of two CTAs,
//                         256 x 256 tiles, cta_group::2 (described with it
//                         below)
//
// One-CTA GEMM structure: one CTA per 128 x (128 kGemmHalves) tile of D (one
// accumulator of 128 columns per half, sharing the A tile), 128 threads.
// Warp 0 is the producer (its lane 0 issues): per K step of 256 elements it
// loads the A tile and the B tile(s) (128 rows x 128 bytes each, 2-D TMA
// with 128-byte swizzle) and the four 512-byte scale tiles of each (1-D
// bulk copies) into one of three shared-memory stages, completing on the
// stage's "full" mbarrier.  Warp 1 is the MMA issuer (lane 0 issues): it
// copies the scale tiles to tensor memory (tcgen05.cp 32x128b.warpx4),
// issues four K=64 MMAs per B tile and commits them to the stage's "empty"
// mbarrier, which frees the stage for the producer.  Both warps wait with
// all their lanes (warp-uniform), so no lane of theirs sits in another wait
// while lane 0 works.  After the last K step a commit to the "done"
// mbarrier releases all four warps into the epilogue: tcgen05.ld of their
// 32 accumulator lanes, times g_a g_b, fp32 stores.  Tensor memory: the
// accumulators and the scale columns of every stage (kGemmTmemCols; shared
// memory lets as many CTAs share an SM as the 512 columns serve, so
// allocation never waits).  All mbarrier waits are bounded: on running out
// the warp records FP4_ERR_TIMEOUT, the waits that depend on it run out in
// turn, the producer waits (bounded) for its copies, and the tensor memory
// is freed before the CTA ends.
#pragma once

#include <cstdint>

#include <cuda.h>

#include "fp4_async.cuh"
#include "fp4_kernels.cuh"

namespace fp4 {

// ---------------------------------------------------------------------------
// TMA tile loads (the mbarrier helpers and the bounded wait are in
// fp4_async.cuh).
// ---------------------------------------------------------------------------
// 2-D TMA tile load of box (x = column, y = row) into shared memory,
// completing on `bar`.  x (the innermost coordinate) times the element size
// is a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
                 : "memory");
}

// ---------------------------------------------------------------------------
// Scale layout for the MMA, as a tiled transpose.  CTA (band, chunk) takes
// the 128 rows of one band and kSfKc consecutive 4-block tiles (64 scale
// bytes per row): it loads the 128 x 64-byte strip with row-contiguous
// loads into shared memory (rows padded to 17 words, so that the column
// reads below are free of bank conflicts), then writes the strip's output
// tiles, which are contiguous in the MMA layout: 16 bytes per thread, word
// 4 r0 + r1 of tile t = the four block scales of row 32 r1 + r0 in tile t.
// Rows past `rows` and blocks past `nb` are 0.
// ---------------------------------------------------------------------------
constexpr int kSfKc = 16;                 // 4-block tiles per CTA
constexpr int kSfRowWords = kSfKc + 1;    // padded shared-memory row (words)

__global__ void __launch_bounds__(256)
    scales_to_mma_kernel(const uint8_t *__restrict__ s, int rows, int nb, int kt, uint32_t *__restrict__ out)
{
    __shared__ uint32_t strip[128 * kSfRowWords];
    pdl_begin();
    const int band = (int)blockIdx.x, kc0 = (int)blockIdx.y * kSfKc;
    const int n_kt = kt - kc0 < kSfKc ? kt - kc0 : kSfKc;
    const int t = (int)threadIdx.x;
    {
        // thread t: row t / 2 of the band, words 8 (t % 2) .. + 7 of its strip
        const int r = t >> 1, h = t & 1;
        const int row = band * 128 + r;
        const int b0 = kc0 * 4 + h * 32; // first block of this thread's 32
        const uint8_t *src = s + (int64_t)row * nb;
        const bool words = (nb & 3) == 0 && (reinterpret_cast<uintptr_t>(s) & 3u) == 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int b = b0 + 4 * i;
            uint32_t v = 0;
            if (row < rows) {
                if (words && b + 3 < nb) {
                    v = __ldcg(reinterpret_cast<const uint32_t *>(src + b));
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (b + j < nb)
                            v |= (uint32_t)__ldcg(src + b + j) << (8 * j);
                }
            }
            strip[r * kSfRowWords + h * 8 + i] = v;
        }
    }
    __syncthreads();
    uint32_t *dst = out + ((int64_t)band * kt + kc0) * 128;
    const bool vec = (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
    for (int i = t; i < n_kt * 32; i += 256) {
        const int tt = i >> 5, q = i & 31; // tile, 16-byte chunk (= r0)
        const uint4 v = make_uint4(strip[q * kSfRowWords + tt], strip[(32 + q) * kSfRowWords + tt],
                                   strip[(64 + q) * kSfRowWords + tt], strip[(96 + q) * kSfRowWords + tt]);
        uint32_t *o = dst + tt * 128 + 4 * q;
        if (vec) {
            *reinterpret_cast<uint4 *>(o) = v;
        } else {
            o[0] = v.x;
            o[1] = v.y;
            o[2] = v.z;
            o[3] = v.w;
        }
    }
}

// ---------------------------------------------------------------------------
// tcgen05 primitives (sm_100a).
// ---------------------------------------------------------------------------
constexpr int kGemmTile = 128;            // M of a CTA tile, N of one accumulator
// Accumulators per CTA (N tile = 128 x kGemmHalves).  Two share the A tile
// but need 167 KB of shared memory, one CTA per SM; one (108 KB) lets two
// CTAs share an SM, so that one's prologue and epilogue overlap the other's
// MMAs, and measured faster (8192^3: 0.93 ms against 1.08 ms).
constexpr int kGemmHalves = 1;
constexpr int kGemmKStep = 256;           // elements of K per stage (128 bytes)
constexpr int kGemmStages = 3;
constexpr int kGemmOpBytes = kGemmTile * 128;          // one operand tile: 16 KB
constexpr int kGemmSfBytes = 4 * 512;                  // scale tiles of one 128-row operand per K step
constexpr int kGemmStageBytes = (1 + kGemmHalves) * (kGemmOpBytes + kGemmSfBytes); // 54 KB
constexpr int kGemmSmem = kGemmStages * kGemmStageBytes + 1024;     // + alignment slack
constexpr uint32_t kGemmSfCols = 16 * (1 + kGemmHalves); // scale columns per stage
// Accumulators, then the scale columns of every stage, rounded up to a power
// of two: 256 for one half (two CTAs per SM use all 512 columns, so an
// allocation never waits), 512 for two (one CTA per SM).
constexpr uint32_t kGemmTmemCols = kGemmHalves == 1 ? 256u : 512u;
static_assert(kGemmTile * kGemmHalves + kGemmStages * kGemmSfCols <= kGemmTmemCols, "tensor memory");

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4 block16: A and B
// E2M1 (format 1 in this kind), K-major, UE4M3 scales (format 0), M = 128
// (bits 24..28 = M / 16), N = 128 (bits 17..22 = N / 8), dense, K = 64.
constexpr uint32_t kGemmIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kGemmTile / 8) << 17) |
                                ((uint32_t)(kGemmTile / 16) << 24);

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: rows of 128
// bytes, 8-row groups 1024 bytes apart (SBO 64 x 16 B), LBO 1, descriptor
// version 1, layout type 2.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}

// Shared-memory descriptor of a 512-byte scale tile for tcgen05.cp (32 rows
// of 16 bytes, K-major without swizzle: 8-row core matrices of 128 bytes,
// SBO 8 x 16 B), version 1, layout type 0.
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t addr)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | (8ull << 32) | (1ull << 46);
}

__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_copy_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_mma_nvfp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile("{\n\t"
                 ".reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
                 "}" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
                 : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

// 32 consecutive accumulator columns of this warp's 32 lanes.
__device__ __forceinline__ void tc_load_32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
                   "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
                   "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    // the registers are operands of the wait, so no use moves above it
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                   "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                   "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// The GEMM.  Grid (ceil(N / (128 kGemmHalves)), M / 128): CTA (bn, bm)
// computes rows bm*128 .. +127 and the 128-column halves of columns
// bn * 128 kGemmHalves .. of D (a half only when it exists: N is a multiple
// of 128) with one accumulator each, sharing the A tile.  map_a / map_b: 2-D uint8 tensor
// maps of the packed operands ([rows, K/2] bytes, box 128 bytes x 128 rows,
// 128-byte swizzle); sfa / sfb: the scale tiles of the whole operands in
// the MMA layout (K/64 tiles per 128-row band).
// Stage layout: A | B halves | SFA | SFB halves.  Tensor memory: columns
// [0, 128 kGemmHalves) the accumulators, then kGemmSfCols scale columns per
// stage (A 16, 16 per B half; 4 per MMA).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const uint8_t *__restrict__ sfa, const uint8_t *__restrict__ sfb,
                      const float *g_a, const float *g_b, int M, int N, int K, float *__restrict__ d,
                      int32_t *status)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kGemmStages], empty[kGemmStages], done;
    __shared__ uint32_t tmem_slot;
    __shared__ int consumed_steps; // K steps the MMA issuer waited for
    // 1024-byte aligned stages (128-byte swizzle atoms)
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

    pdl_begin();
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
    const int bn = (int)blockIdx.x, bm = (int)blockIdx.y;
    const int halves = kGemmHalves == 2 && (bn * kGemmHalves + 1) * kGemmTile < N ? 2 : 1;
    const int kt_steps = K / kGemmKStep;
    const int sf_tiles_per_band = K / 64; // 4-block scale tiles per 128-row band
    const uint32_t stage_tx = (uint32_t)(1 + halves) * (kGemmOpBytes + kGemmSfBytes);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done, 1);
        mbar_init_fence();
        consumed_steps = 0;
    }
    __syncwarp();
    if (warp == 0)
        tmem_alloc(&tmem_slot, kGemmTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;       // lane 0, first allocated column
    const uint32_t tmem_sf = tmem + kGemmTile * kGemmHalves; // scale columns of stage 0

    // Warps 0 and 1 run their loops with all 32 lanes (waits warp-uniform,
    // by __all_sync), and lane 0 issues: no lane of these warps sits in an
    // unrelated wait while its lane 0 works.
    bool timed_out = false;
    int issued = 0;
    if (warp == 0) {
        // producer
        for (int k = 0; k < kt_steps; ++k) {
            const int s = k % kGemmStages;
            if (k >= kGemmStages &&
                !__all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], (uint32_t)((k / kGemmStages) - 1) & 1u))) {
                timed_out = true;
                break;
            }
            if (lane == 0) {
                uint8_t *st = smem + s * kGemmStageBytes;
                uint8_t *sf = st + (1 + kGemmHalves) * kGemmOpBytes;
                mbar_expect_tx(&full[s], stage_tx);
                tma_load_2d(st, &map_a, k * 128, bm * kGemmTile, &full[s]);
                bulk_load(sf, sfa + ((int64_t)bm * sf_tiles_per_band + 4 * k) * 512, kGemmSfBytes, &full[s]);
                for (int h = 0; h < halves; ++h) {
                    const int band = bn * kGemmHalves + h; // 128-row band of B
                    tma_load_2d(st + (1 + h) * kGemmOpBytes, &map_b, k * 128, band * kGemmTile, &full[s]);
                    bulk_load(sf + (1 + h) * kGemmSfBytes,
                              sfb + ((int64_t)band * sf_tiles_per_band + 4 * k) * 512, kGemmSfBytes, &full[s]);
                }
            }
            __syncwarp();
            ++issued;
        }
    } else if (warp == 1) {
        // MMA issuer
        for (int k = 0; k < kt_steps; ++k) {
            const int s = k % kGemmStages;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (uint32_t)(k / kGemmStages) & 1u))) {
                timed_out = true;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint8_t *st = smem + s * kGemmStageBytes;
                const uint32_t a_addr = smem_addr(st);
                const uint32_t sf_addr = smem_addr(st + (1 + kGemmHalves) * kGemmOpBytes);
                const uint32_t sf_cols = tmem_sf + (uint32_t)s * kGemmSfCols;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    tc_copy_sf(sf_cols + 4 * i, smem_desc_sf(sf_addr + 512 * i));
                for (int h = 0; h < halves; ++h)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        tc_copy_sf(sf_cols + 16 * (1 + h) + 4 * i,
                                   smem_desc_sf(sf_addr + (1 + h) * kGemmSfBytes + 512 * i));
                for (int h = 0; h < halves; ++h) {
                    const uint32_t b_addr = smem_addr(st + (1 + h) * kGemmOpBytes);
#pragma unroll
                    for (int i = 0; i < 4; ++i) // four MMAs of K = 64 (32 bytes of each 128-byte row)
                        tc_mma_nvfp4(tmem + (uint32_t)h * kGemmTile, smem_desc_sw128(a_addr + 32 * i),
                                     smem_desc_sw128(b_addr + 32 * i), kGemmIdesc, sf_cols + 4 * i,
                                     sf_cols + 16 * (1 + h) + 4 * i, (k | i) != 0);
                }
                tc_commit(&empty[s]); // frees the stage once these MMAs have read it
                consumed_steps = k + 1;
            }
            __syncwarp();
        }
        if (lane == 0)
            tc_commit(&done);
        __syncwarp();
    }
    // Everyone: wait for the accumulators (bounded), then the epilogue.
    const bool ok = mbar_wait(&done, 0);
    if (!ok || timed_out)
        raise_status(status, kStatusTimeout);
    __syncthreads();
    if (warp == 0) {
        // Copies started that the issuer never waited for (only after a
        // timeout; at most one per stage) must land before the CTA ends.
        for (int j = consumed_steps; j < issued; ++j)
            (void)mbar_wait(&full[j % kGemmStages], (uint32_t)(j / kGemmStages) & 1u);
    }
    __syncwarp();
    if (ok) {
        tc_fence_after();
        const float gg = __fmul_rn(__ldcg(g_a), __ldcg(g_b));
        const int row = bm * kGemmTile + warp * 32 + lane;
        for (int h = 0; h < halves; ++h) {
            float *drow = d + (int64_t)row * N + (int64_t)(bn * kGemmHalves + h) * kGemmTile;
#pragma unroll 1
            for (int c = 0; c < kGemmTile / 32; ++c) {
                float v[32];
                tc_load_32(tmem + (uint32_t)h * kGemmTile + ((uint32_t)(warp * 32) << 16) + (uint32_t)(c * 32), v);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float4 o = make_float4(__fmul_rn(v[4 * q], gg), __fmul_rn(v[4 * q + 1], gg),
                                           __fmul_rn(v[4 * q + 2], gg), __fmul_rn(v[4 * q + 3], gg));
                    *reinterpret_cast<float4 *>(drow + c * 32 + 4 * q) = o;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, kGemmTmemCols);
}

// ---------------------------------------------------------------------------
// The GEMM on CTA pairs: tcgen05 cta_group::2, persistent.
//
// A 128 x 128 tile per SM reads 32 KB of operands from shared memory per
// 8.4 MFLOP.  Two SMs of a cluster pair computing one 256 x 256 tile of D
// with one MMA stream (M = 256, N = 256) read the same bytes per SM for
// twice the flops: each SM holds 128 rows of A and 128 rows of B, the
// pair's tensor cores read both halves.
//
// Roles (320 threads per CTA): warp 0 of both CTAs loads (2-D TMA, 128-byte
// swizzle) this CTA's 128 rows of A and of B and the scale tiles (its own
// 128 rows of A's, all 256 rows of B's) into a four-stage ring; every copy
// completes on the leader CTA's "full" barrier, so the leader sees the
// stage of both CTAs arrive.  Warp 1 of the leader issues: scale tiles to
// tensor memory (tcgen05.cp, which reaches the same columns of both CTAs),
// four K = 64 MMAs per stage, and a commit that arrives on the "empty"
// barrier of the stage in both CTAs.  A scale copy costs the tensor pipe
// about the same per instruction whatever its width, so the scales go over
// in six 128-lane x 256-bit copies per stage (A's for two K steps, or B's
// two bands for one, each) rather than twelve 32-lane x 128-bit ones with
// four-way replication: the stage holds every 512-byte scale tile four
// times (one per 32-lane quarter of tensor memory), placed by TMA loads
// from maps whose replica dimension has stride 0.  The copy writes exactly
// the columns the 32x128b.warpx4 copies wrote.  After a tile's last stage a commit
// arrives on "acc_full" in both CTAs.  Warps 2..9 of both CTAs drain the
// accumulator: each reads its 32 lanes (warp % 4) and one 128-column half
// into registers, releases the accumulator (an arrival on the leader's
// "acc_empty", 16 per tile), and only then scales and stores: each lane
// writes its row's 128 columns (512 contiguous bytes, whole 128-byte lines)
// straight from registers with 32- or 16-byte stores, so the next tile's
// MMAs run while the stores drain, and no shared memory goes to staging
// (it holds a fourth stage instead).  The grid is persistent: cluster p takes
// tiles p, p + P, ... (M-tile fastest).  Tensor memory (512 columns,
// allocated by the pair): the accumulator in columns 0..255, then a ring of
// four scale column sets (16 for A, 32 for B).  All waits are bounded; on
// running out a warp records FP4_ERR_TIMEOUT and leaves its loop, the waits
// that depend on it run out in turn, the leader waits (bounded) for copies
// nobody consumed and for its MMAs, and both CTAs free the tensor memory
// together.
// ---------------------------------------------------------------------------
constexpr int kPairTileM = 256;
constexpr int kPairTileN = 256;
constexpr int kPairStages = 4;
constexpr int kPairSfaBytes = 4 * 4 * 512; // this CTA's 128 rows of A: four scale tiles, each four times
constexpr int kPairSfbBytes = 8 * 4 * 512; // both 128-row bands of the B tile: eight tiles, each four times
constexpr int kPairStageBytes = 2 * kGemmOpBytes + kPairSfaBytes + kPairSfbBytes; // 56 KB
constexpr int kPairEpiWarps = 8;
constexpr int kPairThreads = 320;
constexpr int kPairSmem = kPairStages * kPairStageBytes + 1024; // + alignment to 1024 bytes
constexpr uint32_t kPairSfCols = 16 + 32; // A: 4 columns per MMA; B (256 rows): 8
constexpr uint32_t kPairSfRing = 4;
constexpr uint32_t kPairTmemCols = 512;
static_assert(kPairTileN + kPairSfRing * kPairSfCols <= kPairTmemCols, "tensor memory");
static_assert(kPairStageBytes % 1024 == 0, "stages stay 1024-byte aligned");
static_assert(kPairSmem <= 232448 - 256, "shared memory (with the static barriers)");
// M = 256 (bits 24..28 = M / 16), N = 256 (bits 17..22 = N / 8), E2M1 x E2M1,
// UE4M3 scales, K-major, dense.
constexpr uint32_t kPairIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kPairTileN / 8) << 17) |
                                ((uint32_t)(kPairTileM / 16) << 24);

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank)
{
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_addr(p)), "r"(rank));
    return a;
}

// Every thread of both CTAs (release / acquire).
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}

__device__ __forceinline__ int ld_cluster_s32(uint32_t cl_addr)
{
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(cl_addr) : "memory");
    return v;
}

// 2-D TMA load into this CTA's shared memory, completing on a barrier of
// either CTA of the pair (bar_cl: a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, int x, int y, uint32_t bar_cl)
{
    asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cl)
                 : "memory");
}

// 4-D TMA tile load (pair form, completing on the leader's barrier).
__device__ __forceinline__ void tma_load_4d_pair(void *dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                                 uint32_t bar_cl)
{
    asm volatile("cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar_cl)
                 : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t *slot, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

// Scale tile of each CTA's shared memory into the same columns of each
// CTA's tensor memory.
__device__ __forceinline__ void tc_copy_sf_pair(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a 128-row x 32-byte scale block for the wide
// copy: two 2 KB halves (the first and second 16 bytes of every row), each
// 128 rows x 16 bytes in 8-row core matrices 128 bytes apart; the halves
// are 2 KB apart.
__device__ __forceinline__ uint64_t smem_desc_sf_wide(uint32_t addr)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(2048 >> 4) << 16) | (8ull << 32) | (1ull << 46);
}

// 128 lanes x 256 bits into tensor memory: eight columns of every lane.
__device__ __forceinline__ void tc_copy_sf_wide_pair(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_mma_nvfp4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                  uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile("{\n\t"
                 ".reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
                 "}" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
                 : "memory");
}

// Arrive on the barrier at this offset in both CTAs once the issued
// tcgen05 operations are done.
__device__ __forceinline__ void tc_commit_both(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     smem_addr(bar)),
                 "h"((uint16_t)0x3)
                 : "memory");
}

// Arrive on this CTA's barrier only.
__device__ __forceinline__ void tc_commit_own(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// map_a / map_b: the packed operands as in nvfp4_gemm_kernel.  map_sfa /
// map_sfb: the MMA scale layouts as 4-D uint32 maps (the 128 words of a
// 512-byte tile, four replicas at stride 0, then K steps and bands: for A
// K steps inner, for B bands inner), box 128 x 4 x 2 x 1: two tiles (two K
// steps of A's band, or B's two bands at one K step), each four times.  d:
// D fp32 row-major (16-byte aligned; 32-byte stores when it is 32-byte
// aligned).  M and N multiples of 256, K of 256; grid = 2 x pairs, cluster 2.
__global__ void __launch_bounds__(kPairThreads, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                           const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                           float *__restrict__ d, const float *g_a, const float *g_b, int M, int N, int K,
                           int32_t *status)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kPairStages], empty[kPairStages], acc_full, acc_empty, mma_done;
    __shared__ uint32_t tmem_slot;
    __shared__ int issued_steps, consumed_steps;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

    pdl_begin();
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = (int)blockIdx.x >> 1, n_pairs = (int)gridDim.x >> 1;
    const int tiles_m = M / kPairTileM;
    const int n_tiles = tiles_m * (N / kPairTileN);
    const int kt_steps = K / kGemmKStep;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, 2 * kPairEpiWarps);
        mbar_init(&mma_done, 1);
        mbar_init_fence();
        issued_steps = 0;
        consumed_steps = 0;
    }
    __syncwarp();
    if (warp == 0)
        tmem_alloc_pair(&tmem_slot, kPairTmemCols);
    tc_fence_before();
    cluster_sync(); // both CTAs' barriers initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    bool timed_out = false;
    if (warp == 0) {
        // producer, both CTAs
        int it = 0;
        for (int t = pair; t < n_tiles && !timed_out; t += n_pairs) {
            const int tm = t % tiles_m, tn = t / tiles_m;
            for (int k = 0; k < kt_steps; ++k, ++it) {
                const int s = it % kPairStages;
                if (it >= kPairStages &&
                    !__all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], (uint32_t)((it / kPairStages) - 1) & 1u))) {
                    timed_out = true;
                    break;
                }
                if (lane == 0) {
                    uint8_t *st = smem + s * kPairStageBytes;
                    uint8_t *sf = st + 2 * kGemmOpBytes;
                    const uint32_t bar = cluster_addr(&full[s], 0);
                    if (leader)
                        mbar_expect_tx(&full[s], 2u * kPairStageBytes); // both CTAs' copies
                    tma_load_2d_pair(st, &map_a, k * 128, tm * kPairTileM + (int)rank * kGemmTile, bar);
                    tma_load_2d_pair(st + kGemmOpBytes, &map_b, k * 128, tn * kPairTileN + (int)rank * kGemmTile, bar);
                    // every scale tile four times (one copy per 32-lane quarter of
                    // tensor memory), from maps whose replica dimension has stride
                    // 0: A's tiles 2j, 2j + 1 as [tile 2j x4][tile 2j+1 x4] at
                    // 4096 j, B's tile i of both bands as [band 0 x4][band 1 x4]
                    // at 4096 i
#pragma unroll
                    for (int j = 0; j < 2; ++j)
                        tma_load_4d_pair(sf + 4096 * j, &map_sfa, 0, 0, 4 * k + 2 * j, tm * 2 + (int)rank, bar);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        tma_load_4d_pair(sf + kPairSfaBytes + 4096 * i, &map_sfb, 0, 0, tn * 2, 4 * k + i, bar);
                    issued_steps = it + 1;
                }
                __syncwarp();
            }
        }
        // The last release of every stage (a commit arriving on this CTA's
        // empty barrier) lands before the CTA can end.
        for (int j = it - kPairStages > 0 ? it - kPairStages : 0; j < it; ++j)
            (void)mbar_wait(&empty[j % kPairStages], (uint32_t)(j / kPairStages) & 1u);
    } else if (warp == 1) {
        if (leader) {
            // MMA issuer
            int it = 0, j = 0;
            for (int t = pair; t < n_tiles; t += n_pairs, ++j) {
                if (j > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(&acc_empty, (uint32_t)(j - 1) & 1u))) {
                    timed_out = true;
                    break;
                }
                tc_fence_after();
                for (int k = 0; k < kt_steps; ++k, ++it) {
                    const int s = it % kPairStages;
                    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (uint32_t)(it / kPairStages) & 1u))) {
                        timed_out = true;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a_addr = smem_addr(smem + s * kPairStageBytes);
                        const uint32_t b_addr = a_addr + kGemmOpBytes;
                        const uint32_t sfa_addr = a_addr + 2 * kGemmOpBytes;
                        const uint32_t sfb_addr = sfa_addr + kPairSfaBytes;
                        const uint32_t sfa_t = tmem + kPairTileN + (uint32_t)(it % kPairSfRing) * kPairSfCols;
                        const uint32_t sfb_t = sfa_t + 16;
                        // A's scales for MMAs 2j and 2j + 1 in columns 8j..8j+3 and
                        // 8j+4..8j+7; B's for MMA i: rows 0..127 in columns
                        // 8i..8i+3, rows 128..255 in 8i+4..8i+7 -- one wide copy
                        // each (the copies cost per instruction, not per byte)
#pragma unroll
                        for (int j = 0; j < 2; ++j)
                            tc_copy_sf_wide_pair(sfa_t + 8 * j, smem_desc_sf_wide(sfa_addr + 4096 * j));
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            tc_copy_sf_wide_pair(sfb_t + 8 * i, smem_desc_sf_wide(sfb_addr + 4096 * i));
#pragma unroll
                        for (int i = 0; i < 4; ++i) // four MMAs of K = 64 (32 bytes of each 128-byte row)
                            tc_mma_nvfp4_pair(tmem, smem_desc_sw128(a_addr + 32 * i), smem_desc_sw128(b_addr + 32 * i),
                                              kPairIdesc, sfa_t + 4 * i, sfb_t + 8 * i, (k | i) != 0);
                        tc_commit_both(&empty[s]); // frees the stage in both CTAs
                        consumed_steps = it + 1;
                    }
                    __syncwarp();
                }
                if (timed_out)
                    break;
                if (lane == 0)
                    tc_commit_both(&acc_full);
                __syncwarp();
            }
            // the epilogues have read the last accumulator
            if (!timed_out && j > 0 &&
                !__all_sync(0xFFFFFFFFu, mbar_wait(&acc_empty, (uint32_t)(j - 1) & 1u)))
                timed_out = true;
            // every MMA issued has finished before tensor memory is freed
            if (lane == 0)
                tc_commit_own(&mma_done);
            __syncwarp();
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&mma_done, 0)))
                timed_out = true;
        }
    } else {
        // epilogue, both CTAs: lanes of warp % 4, columns 128 h .. 128 h + 127;
        // lane l stores row 32 q + l of this CTA's half of the tile
        const int q = warp & 3, h = (warp - 2) >> 2;
        const float gg = __fmul_rn(__ldcg(g_a), __ldcg(g_b));
        const uint32_t release = cluster_addr(&acc_empty, 0);
        const bool wide = (reinterpret_cast<uintptr_t>(d) & 31u) == 0; // 32-byte stores
        int j = 0;
        for (int t = pair; t < n_tiles; t += n_pairs, ++j) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&acc_full, (uint32_t)j & 1u))) {
                timed_out = true;
                break;
            }
            tc_fence_after();
            float v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tc_load_32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * 128 + c * 32), v[c]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(release); // the accumulator may be overwritten now
            const int tm = t % tiles_m, tn = t / tiles_m;
            const int row = tm * kPairTileM + (int)rank * kGemmTile + q * 32 + lane;
            float *drow = d + (int64_t)row * N + tn * kPairTileN + h * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t o[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        o[i] = __float_as_uint(__fmul_rn(v[c][8 * u + i], gg));
                    float *p = drow + c * 32 + 8 * u;
                    if (wide) {
                        stg_v8(p, o);
                    } else {
                        *reinterpret_cast<uint4 *>(p) = make_uint4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<uint4 *>(p + 4) = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
            }
        }
    }
    if (timed_out)
        raise_status(status, kStatusTimeout);

    tc_fence_before();
    cluster_sync(); // every role of both CTAs is done
    if (leader && warp == 0) {
        // After a timeout only: copies of either CTA that the MMA warp never
        // waited for complete on the leader's full barriers; wait (bounded).
        const int peer_issued = ld_cluster_s32(cluster_addr(&issued_steps, 1));
        const int last = issued_steps > peer_issued ? issued_steps : peer_issued;
        for (int j = consumed_steps; j < last; ++j)
            (void)mbar_wait(&full[j % kPairStages], (uint32_t)(j / kPairStages) & 1u);
    }
    cluster_sync(); // the peer stays until the leader's drain is done
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kPairTmemCols);
    }
}

} // namespace fp4
