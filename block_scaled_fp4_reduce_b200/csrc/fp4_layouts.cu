// fp4_layouts.cu -- entry points of include/fp4.h for ragged rows (padded
// to whole blocks) and column-wise grouping: argument checks, store-layout
// flags and the launches.
#include <climits>
#include <cstdint>

#include <cuda_runtime.h>

#include "fp4.h"
#include "fp4_launch.cuh"
#include "fp4_layouts.cuh"

namespace {

using namespace fp4_launch;

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

fp4_status check_rows_cols(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0)
        return FP4_ERR_INVALID_ARG;
    if (cols > 0 && rows > INT64_MAX / cols / 4)
        return FP4_ERR_SHAPE;
    return FP4_OK;
}

// ---------------------------------------------------------------- padded --

template <typename T>
fp4_status nv_padded(const T *x, int64_t rows, int64_t cols, const float *amax, uint8_t *packed,
                     uint8_t *scales, float *global_scale, int32_t *status, cudaStream_t stream)
{
    const int64_t nbp = ceil_div(cols, 16);
    return for_row_chunks(rows, nbp, [&](int64_t r0, int64_t nr) {
        const int n = (int)(nr * nbp);
        const int grid = grid_for(fp4::nvfp4_quantize_padded_kernel<T>, n, (int64_t)kThreads * fp4::pad_units<16>());
        if (grid <= 0)
            return FP4_ERR_CUDA;
        return launch(fp4::nvfp4_quantize_padded_kernel<T>, grid, stream,
                          x + r0 * cols, cols, fp4::fast_div_for((uint32_t)nbp), n, amax,
                          reinterpret_cast<uint2 *>(packed) + r0 * nbp, scales + r0 * nbp, global_scale,
                          status);
    });
}

template <typename T, bool kCeil>
fp4_status mx_padded(const T *x, int64_t rows, int64_t cols, uint8_t *packed, uint8_t *scales,
                     int32_t *status, cudaStream_t stream)
{
    const int64_t nbp = ceil_div(cols, 32);
    return for_row_chunks(rows, nbp, [&](int64_t r0, int64_t nr) {
        const int n = (int)(nr * nbp);
        const int grid = grid_for(fp4::mxfp4_quantize_padded_kernel<T, kCeil>, n,
                                  (int64_t)kThreads * fp4::pad_units<32>());
        if (grid <= 0)
            return FP4_ERR_CUDA;
        return launch(fp4::mxfp4_quantize_padded_kernel<T, kCeil>, grid, stream,
                          x + r0 * cols, cols, fp4::fast_div_for((uint32_t)nbp), n,
                          reinterpret_cast<uint4 *>(packed) + r0 * nbp, scales + r0 * nbp, status);
    });
}

template <bool kNv, typename TOut>
fp4_status dq_padded(const uint8_t *packed, const uint8_t *scales, const float *global_scale,
                     int64_t rows, int64_t cols, TOut *y, cudaStream_t stream)
{
    const int64_t nup = ceil_div(cols, kNv ? 16 : 32) * (kNv ? 1 : 2); // 16-code units per row
    return for_row_chunks(rows, nup, [&](int64_t r0, int64_t nr) {
        const int n = (int)(nr * nup);
        const int grid = grid_for(fp4::dequantize_padded_kernel<kNv, TOut>, n, (int64_t)kThreads * 2);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        return launch(fp4::dequantize_padded_kernel<kNv, TOut>, grid, stream,
                          reinterpret_cast<const uint2 *>(packed) + r0 * nup,
                          scales + (kNv ? r0 * nup : r0 * nup / 2), global_scale, cols,
                          fp4::fast_div_for((uint32_t)nup), n, y + r0 * cols);
    });
}

// ----------------------------------------------------------- column-wise --

template <typename T>
fp4_status nv_columns(const T *x, int64_t rows, int64_t cols, const float *amax, uint8_t *packed,
                      uint8_t *scales, float *global_scale, int32_t *status, cudaStream_t stream)
{
    const int64_t cw = cols * (int64_t)sizeof(T) / 4; // 4-byte words per row (rows are 4-byte aligned)
    const int64_t tiles = ceil_div(rows, fp4::kNvColRows) * ceil_div(cw, 32);
    const int64_t nbo = ceil_div(rows, 16);
    // the widest stores every output row allows: four blocks (32 bytes) and
    // four scale bytes at once
    int layout = 0;
    if ((nbo * 8) % 32 == 0 && aligned(packed, 32))
        layout |= fp4::kColPacked32;
    if ((nbo * 8) % 16 == 0 && aligned(packed, 16))
        layout |= fp4::kColPacked16;
    if (nbo % 4 == 0 && aligned(scales, 4))
        layout |= fp4::kColScales4;
    const int grid = grid_for(fp4::nvfp4_quantize_columns_kernel<T>, tiles, 1);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    return launch(fp4::nvfp4_quantize_columns_kernel<T>, grid, stream, reinterpret_cast<const uint32_t *>(x),
                  (int)rows, (int)cw, (int)cols, amax, packed, scales, global_scale, status, layout);
}

template <typename T, bool kCeil>
fp4_status mx_columns(const T *x, int64_t rows, int64_t cols, uint8_t *packed, uint8_t *scales, int32_t *status,
                      cudaStream_t stream)
{
    const int64_t cw = cols * (int64_t)sizeof(T) / 4; // 4-byte words per row (rows are 4-byte aligned)
    const int64_t tiles = ceil_div(rows, fp4::kMxColRows) * ceil_div(cw, 32);
    const int64_t nbo = ceil_div(rows, 32);
    // the widest stores every output row allows: two blocks (32 bytes) and
    // four scale bytes at once
    int layout = 0;
    if ((nbo * 16) % 32 == 0 && aligned(packed, 32))
        layout |= fp4::kColPacked32;
    if (nbo % 4 == 0 && aligned(scales, 4))
        layout |= fp4::kColScales4;
    auto kernel = fp4::mxfp4_quantize_columns_kernel<T, kCeil>;
    const int grid = grid_for(kernel, tiles, 1);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    return launch(kernel, grid, stream, reinterpret_cast<const uint32_t *>(x), (int)rows, (int)cw, (int)cols,
                  packed, scales, status, layout);
}

// Common checks of the quantisers here; NV also needs a workspace.
fp4_status check_quant(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                       const uint8_t *packed, const uint8_t *scales, const int32_t *status)
{
    if (!status || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    const fp4_status st = check_rows_cols(rows, cols);
    if (st != FP4_OK)
        return st;
    if (rows * cols > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16))
        return FP4_ERR_ALIGN;
    return FP4_OK;
}

fp4_status check_ws(const void *workspace, size_t bytes)
{
    if (!workspace || bytes < kWsWords * sizeof(uint32_t) || !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    return FP4_OK;
}

// The column-wise pass reads W through a TMA tensor map: 32-bit sizes and
// a row pitch that is a multiple of 16 bytes.
fp4_status check_columns(fp4_dtype dtype, int64_t rows, int64_t cols)
{
    if (rows > INT_MAX || cols > INT_MAX)
        return FP4_ERR_SHAPE;
    if ((cols * (dtype == FP4_BF16 ? 2 : 4)) % 4) // the kernels read rows as 4-byte words
        return FP4_ERR_ALIGN;
    return FP4_OK;
}

} // namespace

extern "C" {

fp4_status fp4_nvfp4_quantize_padded_with_amax(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                               const float *amax, uint8_t *packed, uint8_t *scales,
                                               float *global_scale, int32_t *status, cudaStream_t stream)
{
    fp4_status st = check_quant(x, dtype, rows, cols, packed, scales, status);
    if (st != FP4_OK)
        return st;
    if (!global_scale || !amax)
        return FP4_ERR_INVALID_ARG;
    if (!aligned(amax, 4))
        return FP4_ERR_ALIGN;
    if (cols % 16 == 0)
        return fp4_nvfp4_quantize_with_amax(x, dtype, rows, cols, amax, packed, scales, global_scale, status,
                                            stream);
    if (dtype == FP4_BF16)
        return nv_padded(static_cast<const uint16_t *>(x), rows, cols, amax, packed, scales,
                         global_scale, status, stream);
    return nv_padded(static_cast<const float *>(x), rows, cols, amax, packed, scales, global_scale,
                     status, stream);
}

fp4_status fp4_nvfp4_quantize_padded(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                     uint8_t *packed, uint8_t *scales, float *global_scale,
                                     void *workspace, size_t workspace_bytes, int32_t *status,
                                     cudaStream_t stream)
{
    fp4_status st = check_quant(x, dtype, rows, cols, packed, scales, status);
    if (st != FP4_OK)
        return st;
    if (!global_scale)
        return FP4_ERR_INVALID_ARG;
    if ((st = check_ws(workspace, workspace_bytes)) != FP4_OK)
        return st;
    float *amax = reinterpret_cast<float *>(static_cast<uint32_t *>(workspace) + kWsAmax);
    st = fp4_tensor_amax(x, dtype, rows * cols, amax, workspace, workspace_bytes, status, stream);
    if (st != FP4_OK)
        return st;
    return fp4_nvfp4_quantize_padded_with_amax(x, dtype, rows, cols, amax, packed, scales, global_scale, status,
                                               stream);
}

fp4_status fp4_mxfp4_quantize_padded(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                     fp4_mx_rule rule, uint8_t *packed, uint8_t *scales,
                                     int32_t *status, cudaStream_t stream)
{
    fp4_status st = check_quant(x, dtype, rows, cols, packed, scales, status);
    if (st != FP4_OK)
        return st;
    if (rule != FP4_MX_FLOOR && rule != FP4_MX_CEIL)
        return FP4_ERR_INVALID_ARG;
    if (cols % 32 == 0)
        return rule == FP4_MX_CEIL
                   ? fp4_mxfp4_quantize_ceil(x, dtype, rows, cols, packed, scales, status, stream)
                   : fp4_mxfp4_quantize(x, dtype, rows, cols, packed, scales, status, stream);
    const bool bf = dtype == FP4_BF16, ceil = rule == FP4_MX_CEIL;
    if (bf && ceil)
        return mx_padded<uint16_t, true>(static_cast<const uint16_t *>(x), rows, cols, packed, scales, status, stream);
    if (bf)
        return mx_padded<uint16_t, false>(static_cast<const uint16_t *>(x), rows, cols, packed, scales, status, stream);
    if (ceil)
        return mx_padded<float, true>(static_cast<const float *>(x), rows, cols, packed, scales, status, stream);
    return mx_padded<float, false>(static_cast<const float *>(x), rows, cols, packed, scales, status, stream);
}

fp4_status fp4_dequantize_padded(fp4_format fmt, const uint8_t *packed, const uint8_t *scales,
                                 const float *global_scale, int64_t rows, int64_t cols, void *y,
                                 fp4_dtype out_dtype, cudaStream_t stream)
{
    if ((fmt != FP4_NVFP4 && fmt != FP4_MXFP4) || !valid_dtype(out_dtype))
        return FP4_ERR_INVALID_ARG;
    const bool nv = fmt == FP4_NVFP4;
    fp4_status st = check_rows_cols(rows, cols);
    if (st != FP4_OK)
        return st;
    if (rows * cols == 0)
        return FP4_OK;
    if (!packed || !scales || !y || (nv && !global_scale))
        return FP4_ERR_INVALID_ARG;
    const size_t esz = out_dtype == FP4_BF16 ? 2 : 4;
    if (!aligned(packed, 16) || !aligned(y, esz) || (nv && !aligned(global_scale, 4)))
        return FP4_ERR_ALIGN;
    if (cols % (nv ? 16 : 32) == 0 && aligned(y, 32))
        return fp4_dequantize(fmt, packed, scales, global_scale, rows, cols, y, out_dtype, stream);
    if (nv && out_dtype == FP4_BF16)
        return dq_padded<true>(packed, scales, global_scale, rows, cols, static_cast<uint16_t *>(y), stream);
    if (nv)
        return dq_padded<true>(packed, scales, global_scale, rows, cols, static_cast<float *>(y), stream);
    if (out_dtype == FP4_BF16)
        return dq_padded<false>(packed, scales, global_scale, rows, cols, static_cast<uint16_t *>(y), stream);
    return dq_padded<false>(packed, scales, global_scale, rows, cols, static_cast<float *>(y), stream);
}

fp4_status fp4_nvfp4_quantize_columns_with_amax(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                                const float *amax, uint8_t *packed, uint8_t *scales,
                                                float *global_scale, int32_t *status, cudaStream_t stream)
{
    fp4_status st = check_quant(x, dtype, rows, cols, packed, scales, status);
    if (st != FP4_OK)
        return st;
    if (!global_scale || !amax)
        return FP4_ERR_INVALID_ARG;
    if ((st = check_columns(dtype, rows, cols)) != FP4_OK)
        return st;
    if (!aligned(amax, 4))
        return FP4_ERR_ALIGN;
    if (dtype == FP4_BF16)
        return nv_columns(static_cast<const uint16_t *>(x), rows, cols, amax, packed, scales, global_scale,
                          status, stream);
    return nv_columns(static_cast<const float *>(x), rows, cols, amax, packed, scales, global_scale, status,
                      stream);
}

fp4_status fp4_nvfp4_quantize_columns(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                      uint8_t *packed, uint8_t *scales, float *global_scale,
                                      void *workspace, size_t workspace_bytes, int32_t *status,
                                      cudaStream_t stream)
{
    fp4_status st = check_quant(x, dtype, rows, cols, packed, scales, status);
    if (st != FP4_OK)
        return st;
    if (!global_scale)
        return FP4_ERR_INVALID_ARG;
    if ((st = check_columns(dtype, rows, cols)) != FP4_OK)
        return st;
    if ((st = check_ws(workspace, workspace_bytes)) != FP4_OK)
        return st;
    float *amax = reinterpret_cast<float *>(static_cast<uint32_t *>(workspace) + kWsAmax);
    st = fp4_tensor_amax(x, dtype, rows * cols, amax, workspace, workspace_bytes, status, stream);
    if (st != FP4_OK)
        return st;
    return fp4_nvfp4_quantize_columns_with_amax(x, dtype, rows, cols, amax, packed, scales, global_scale, status,
                                                stream);
}

fp4_status fp4_mxfp4_quantize_columns(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                      fp4_mx_rule rule, uint8_t *packed, uint8_t *scales,
                                      int32_t *status, cudaStream_t stream)
{
    fp4_status st = check_quant(x, dtype, rows, cols, packed, scales, status);
    if (st != FP4_OK)
        return st;
    if (rule != FP4_MX_FLOOR && rule != FP4_MX_CEIL)
        return FP4_ERR_INVALID_ARG;
    if ((st = check_columns(dtype, rows, cols)) != FP4_OK)
        return st;
    const bool bf = dtype == FP4_BF16, ceil = rule == FP4_MX_CEIL;
    const uint16_t *xb = static_cast<const uint16_t *>(x);
    const float *xf = static_cast<const float *>(x);
    if (bf && ceil)
        return mx_columns<uint16_t, true>(xb, rows, cols, packed, scales, status, stream);
    if (bf)
        return mx_columns<uint16_t, false>(xb, rows, cols, packed, scales, status, stream);
    if (ceil)
        return mx_columns<float, true>(xf, rows, cols, packed, scales, status, stream);
    return mx_columns<float, false>(xf, rows, cols, packed, scales, status, stream);
}

} // extern "C"
