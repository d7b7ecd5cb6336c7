// fp4_gemm.cu -- entry points of include/fp4.h for the consumer of the
// quantised operands: the tiled scale layout of the tensor-core MMA and the
// block-scaled NVFP4 matrix product.  Argument checks, TMA tensor maps, the
// launches.
#include <climits>
#include <cstdint>
#include <cstring>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fp4.h"
#include "fp4_gemm.cuh"
#include "fp4_launch.cuh"

namespace {

using namespace fp4_launch;

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// 2-D tensor map of a packed NVFP4 operand [rows, K/2] bytes: box 128 bytes
// x 128 rows, 128-byte swizzle (the MMA's K-major shared-memory layout).
fp4_status operand_map(const uint8_t *p, int64_t rows, int64_t K, CUtensorMap *map)
{
    EncodeTiled enc = encode_tiled();
    if (!enc)
        return FP4_ERR_CUDA;
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    const cuuint32_t box[2] = {128u, (cuuint32_t)fp4::kGemmTile};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(p), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FP4_OK : FP4_ERR_CUDA;
}

// 4-D tensor maps of an MMA scale layout (rows / 128 bands of K / 64 tiles of
// 512 bytes) that place every tile four times: dimension 0 the 128 words of
// a tile, dimension 1 four replicas (stride 0), then the tile within its
// band and the band (box 128 x 4 x 2 x 1, in the order the wide copy reads:
// two tiles of one band for A, one tile of two bands for B).
fp4_status scale_map_rep(const uint8_t *sf, int64_t rows, int64_t K, bool band_inner, CUtensorMap *map)
{
    EncodeTiled enc = encode_tiled();
    if (!enc)
        return FP4_ERR_CUDA;
    const cuuint64_t tiles = (cuuint64_t)(K / 64), bands = (cuuint64_t)(rows / 128);
    const cuuint64_t band_stride = tiles * 512u;
    const cuuint64_t dims[4] = {128u, 4u, band_inner ? bands : tiles, band_inner ? tiles : bands};
    const cuuint64_t strides[3] = {0u, band_inner ? band_stride : 512u, band_inner ? 512u : band_stride};
    const cuuint32_t box[4] = {128u, 4u, 2u, 1u};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint8_t *>(sf), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FP4_OK : FP4_ERR_CUDA;
}

bool set_smem_attr(const void *kernel, int bytes, bool (&done)[kMaxDevices], int dev)
{
    if (done[dev])
        return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    done[dev] = true;
    return true;
}

// Clusters of two CTAs of the pair kernel that fit on the device at once.
int pair_clusters(int dev)
{
    static int cached[kMaxDevices] = {0};
    if (cached[dev] > 0)
        return cached[dev];
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(fp4::kPairThreads);
    cfg.dynamicSmemBytes = fp4::kPairSmem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fp4::nvfp4_gemm_pair_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    cached[dev] = n;
    return n;
}

fp4_status launch_pair(const uint8_t *packed_a, const uint8_t *sfa, const float *g_a, const uint8_t *packed_b,
                       const uint8_t *sfb, const float *g_b, int64_t M, int64_t N, int64_t K, float *d,
                       int32_t *status, cudaStream_t stream, int dev)
{
    static bool attr_set[kMaxDevices] = {false};
    if (!set_smem_attr((const void *)fp4::nvfp4_gemm_pair_kernel, fp4::kPairSmem, attr_set, dev))
        return FP4_ERR_CUDA;
    const int clusters = pair_clusters(dev);
    if (clusters <= 0)
        return FP4_ERR_CUDA;
    CUtensorMap map_a, map_b, map_sfa, map_sfb;
    std::memset(&map_a, 0, sizeof(map_a));
    std::memset(&map_b, 0, sizeof(map_b));
    std::memset(&map_sfa, 0, sizeof(map_sfa));
    std::memset(&map_sfb, 0, sizeof(map_sfb));
    fp4_status st;
    if ((st = operand_map(packed_a, M, K, &map_a)) != FP4_OK || (st = operand_map(packed_b, N, K, &map_b)) != FP4_OK ||
        (st = scale_map_rep(sfa, M, K, false, &map_sfa)) != FP4_OK ||
        (st = scale_map_rep(sfb, N, K, true, &map_sfb)) != FP4_OK)
        return st;
    const int64_t tiles = (M / fp4::kPairTileM) * (N / fp4::kPairTileN);
    const int64_t pairs = tiles < clusters ? tiles : clusters;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(fp4::kPairThreads);
    cfg.dynamicSmemBytes = fp4::kPairSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, fp4::nvfp4_gemm_pair_kernel, map_a, map_b, map_sfa, map_sfb, d, g_a, g_b,
                           (int)M, (int)N, (int)K, status) != cudaSuccess) {
        (void)cudaGetLastError();
        return FP4_ERR_CUDA;
    }
    return FP4_OK;
}

} // namespace

extern "C" {

size_t fp4_mma_scales_bytes(int64_t rows, int64_t blocks)
{
    if (rows < 0 || blocks < 0)
        return 0;
    return (size_t)(cdiv(rows, 128) * 128 * cdiv(blocks, 4) * 4);
}

fp4_status fp4_scales_to_mma_layout(const uint8_t *scales, int64_t rows, int64_t blocks, uint8_t *out,
                                    cudaStream_t stream)
{
    if (rows < 0 || blocks < 0)
        return FP4_ERR_INVALID_ARG;
    const int64_t words = (int64_t)fp4_mma_scales_bytes(rows, blocks) / 4;
    if (words == 0)
        return FP4_OK;
    if (!out || (rows * blocks > 0 && !scales))
        return FP4_ERR_INVALID_ARG;
    const int64_t bands = cdiv(rows, 128), kt = cdiv(blocks, 4), chunks = cdiv(kt, fp4::kSfKc);
    if (words > INT_MAX || rows > INT_MAX || blocks > INT_MAX || chunks > 65535)
        return FP4_ERR_SHAPE;
    if (!aligned(out, 4))
        return FP4_ERR_ALIGN;
    return launch_cfg(fp4::scales_to_mma_kernel, dim3((unsigned)bands, (unsigned)chunks), 256, 0, stream, scales,
                      (int)rows, (int)blocks, (int)kt, reinterpret_cast<uint32_t *>(out));
}

fp4_status fp4_nvfp4_gemm(const uint8_t *packed_a, const uint8_t *scales_a_mma, const float *global_scale_a,
                          const uint8_t *packed_b, const uint8_t *scales_b_mma, const float *global_scale_b,
                          int64_t M, int64_t N, int64_t K, float *d, int32_t *status, cudaStream_t stream)
{
    return fp4_nvfp4_gemm_ex(packed_a, scales_a_mma, global_scale_a, packed_b, scales_b_mma, global_scale_b, M, N, K,
                             d, FP4_GEMM_AUTO, status, stream);
}

fp4_status fp4_nvfp4_gemm_ex(const uint8_t *packed_a, const uint8_t *scales_a_mma, const float *global_scale_a,
                             const uint8_t *packed_b, const uint8_t *scales_b_mma, const float *global_scale_b,
                             int64_t M, int64_t N, int64_t K, float *d, fp4_gemm_kernel kernel, int32_t *status,
                             cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || !status ||
        (kernel != FP4_GEMM_AUTO && kernel != FP4_GEMM_CTA && kernel != FP4_GEMM_CTA_PAIR))
        return FP4_ERR_INVALID_ARG;
    if (M % fp4::kGemmTile || N % fp4::kGemmTile || K % fp4::kGemmKStep || M > INT_MAX || N > INT_MAX ||
        K > INT_MAX)
        return FP4_ERR_SHAPE;
    // the pair kernel indexes its tiles and scale-tile rows with 32-bit ints
    const bool pair_shape = M % fp4::kPairTileM == 0 && N % fp4::kPairTileN == 0 && (M / 128) * (K / 64) <= INT_MAX &&
                            (N / 128) * (K / 64) <= INT_MAX &&
                            (M / fp4::kPairTileM) * (N / fp4::kPairTileN) <= INT_MAX;
    if (kernel == FP4_GEMM_CTA_PAIR && !pair_shape)
        return FP4_ERR_SHAPE;
    if (M == 0 || N == 0)
        return FP4_OK;
    if (!packed_a || !packed_b || !scales_a_mma || !scales_b_mma || !global_scale_a || !global_scale_b || !d)
        return FP4_ERR_INVALID_ARG;
    if (!aligned(packed_a, 16) || !aligned(packed_b, 16) || !aligned(scales_a_mma, 16) ||
        !aligned(scales_b_mma, 16) || !aligned(d, 16) || !aligned(global_scale_a, 4) ||
        !aligned(global_scale_b, 4))
        return FP4_ERR_ALIGN;
    if (K == 0) { // an empty sum: D = 0
        if (cudaMemsetAsync(d, 0, (size_t)(M * N) * sizeof(float), stream) != cudaSuccess) {
            (void)cudaGetLastError();
            return FP4_ERR_CUDA;
        }
        return FP4_OK;
    }
    int dev = 0;
    const int sms = sm_count(dev);
    if (sms <= 0 || dev >= kMaxDevices)
        return FP4_ERR_CUDA;
    // The pair kernel once its 256 x 256 tiles give every SM pair work
    // (measured on B200 with its wide scale copies: 8192 x 4096 x 14336 3.66
    // against 3.18 PFLOP/s for the one-CTA kernel, 8192^3 3.60 against 2.86,
    // 4096 x 4096 x 14336 3.24 against 2.77).
    if (kernel == FP4_GEMM_CTA_PAIR ||
        (kernel == FP4_GEMM_AUTO && pair_shape && (M / fp4::kPairTileM) * (N / fp4::kPairTileN) >= sms / 2))
        return launch_pair(packed_a, scales_a_mma, global_scale_a, packed_b, scales_b_mma, global_scale_b, M, N, K, d,
                           status, stream, dev);
    static bool attr_set[kMaxDevices] = {false};
    if (!set_smem_attr((const void *)fp4::nvfp4_gemm_kernel, fp4::kGemmSmem, attr_set, dev))
        return FP4_ERR_CUDA;
    CUtensorMap map_a, map_b;
    std::memset(&map_a, 0, sizeof(map_a));
    std::memset(&map_b, 0, sizeof(map_b));
    fp4_status st = operand_map(packed_a, M, K, &map_a);
    if (st != FP4_OK)
        return st;
    if ((st = operand_map(packed_b, N, K, &map_b)) != FP4_OK)
        return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(N / fp4::kGemmTile), (unsigned)(M / fp4::kGemmTile));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = fp4::kGemmSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fp4::nvfp4_gemm_kernel, map_a, map_b, scales_a_mma, scales_b_mma, global_scale_a,
                           global_scale_b, (int)M, (int)N, (int)K, d, status) != cudaSuccess) {
        (void)cudaGetLastError();
        return FP4_ERR_CUDA;
    }
    return FP4_OK;
}

} // extern "C"
