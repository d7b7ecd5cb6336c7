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
    if (words > INT_MAX || rows > INT_MAX || blocks > INT_MAX)
        return FP4_ERR_SHAPE;
    if (!aligned(out, 4))
        return FP4_ERR_ALIGN;
    const int grid = grid_for(fp4::scales_to_mma_kernel, words, kThreads);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    return launch(fp4::scales_to_mma_kernel, grid, stream, scales, (int)rows, (int)blocks,
                  (int)cdiv(blocks, 4), (int)words, reinterpret_cast<uint32_t *>(out));
}

fp4_status fp4_nvfp4_gemm(const uint8_t *packed_a, const uint8_t *scales_a_mma, const float *global_scale_a,
                          const uint8_t *packed_b, const uint8_t *scales_b_mma, const float *global_scale_b,
                          int64_t M, int64_t N, int64_t K, float *d, int32_t *status, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || !status)
        return FP4_ERR_INVALID_ARG;
    if (M % fp4::kGemmTile || N % fp4::kGemmTile || K % fp4::kGemmKStep || M > INT_MAX || N > INT_MAX ||
        K > INT_MAX)
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
    static bool attr_set[kMaxDevices] = {false};
    int dev = 0;
    if (sm_count(dev) <= 0 || dev >= kMaxDevices)
        return FP4_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(fp4::nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 fp4::kGemmSmem) != cudaSuccess) {
            (void)cudaGetLastError();
            return FP4_ERR_CUDA;
        }
        attr_set[dev] = true;
    }
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
