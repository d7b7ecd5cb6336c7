// fp4_capi.cu -- the extern "C" entry points declared in include/fp4.h.
//
// Argument checking and launch configuration only: every step of the path
// runs in the kernels of fp4_kernels.cuh.  Nothing here allocates, frees or
// synchronises; every launch goes on the caller's stream.
#include <climits>
#include <cstdint>
#include <type_traits>

#include <cuda_runtime.h>

#include "fp4.h"
#include "fp4_kernels.cuh"
#include "fp4_async.cuh"
#include "fp4_launch.cuh"

namespace fp4_launch {
int64_t g_launch_unit_limit = fp4::kMaxUnitsPerLaunch;
}

namespace {

using namespace fp4_launch;
using fp4::kMaxPartials;
using fp4::kThreads;

// rows, cols >= 0, cols % block == 0, rows * cols representable.
fp4_status check_shape(int64_t rows, int64_t cols, int64_t block)
{
    if (rows < 0 || cols < 0)
        return FP4_ERR_INVALID_ARG;
    if (cols % block)
        return FP4_ERR_SHAPE;
    if (cols > 0 && rows > INT64_MAX / cols / 4)
        return FP4_ERR_SHAPE;
    return FP4_OK;
}


} // namespace

namespace {
template <bool kCeil>
fp4_status mxfp4_quantize_rule(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                               uint8_t *packed, uint8_t *scales, int32_t *status,
                               cudaStream_t stream)
{
    if (!status || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    fp4_status st = check_shape(rows, cols, 32);
    if (st != FP4_OK)
        return st;
    const int64_t n = rows * cols;
    if (n == 0)
        return FP4_OK;
    if (!x || !packed || !scales)
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16))
        return FP4_ERR_ALIGN;
    uint4 *pk = reinterpret_cast<uint4 *>(packed);
    auto run = [&](auto *xt) {
        using T = std::remove_const_t<std::remove_pointer_t<decltype(xt)>>;
        return for_chunks(n / 32, [&](int64_t first, int count) {
            const int grid =
                grid_for(fp4::mxfp4_quantize_kernel<T, kCeil>, count, (int64_t)kThreads * 2);
            if (grid <= 0)
                return FP4_ERR_CUDA;
            return launch(fp4::mxfp4_quantize_kernel<T, kCeil>, grid, stream, xt + first * 32,
                          count, pk + first, scales + first, status);
        });
    };
    if (dtype == FP4_BF16)
        return run(static_cast<const uint16_t *>(x));
    return run(static_cast<const float *>(x));
}
} // namespace

namespace {
template <typename K, typename T>
fp4_status launch_block_kernel(K kernel, const T *x, int64_t n, const float *amax,
                               uint8_t *packed, uint8_t *scales, float *global_scale,
                               float *block_loss, int32_t *status, cudaStream_t stream)
{
    uint2 *pk = reinterpret_cast<uint2 *>(packed);
    return for_chunks(n / 16, [&](int64_t first, int count) {
        const int grid = grid_for(kernel, count, kThreads);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        return launch(kernel, grid, stream, x + first * 16, count, amax, pk + first,
                      scales + first, global_scale, block_loss ? block_loss + first : block_loss,
                      status);
    });
}

template <typename T, bool kFixed>
fp4_status launch_search_t(const T *x, int64_t n, const float *amax, uint8_t *packed, uint8_t *scales,
                           float *global_scale, float *block_loss, int32_t *status, cudaStream_t stream,
                           int n_cand, int p, int q)
{
    uint2 *pk = reinterpret_cast<uint2 *>(packed);
    auto kernel = fp4::scale_search_kernel<T, kFixed>;
    return for_chunks(n / 16, [&](int64_t first, int count) {
        const int grid = grid_for(kernel, count, kThreads);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        return launch(kernel, grid, stream, x + first * 16, count, amax, pk + first, scales + first, global_scale,
                      block_loss ? block_loss + first : block_loss, status, p, p + n_cand - 1, q);
    });
}

// n_cand = 0: the fixed grid of 64 candidates (147 + k) / 210.
fp4_status launch_search(const void *x, fp4_dtype dtype, int64_t n, const float *amax,
                         uint8_t *packed, uint8_t *scales, float *global_scale,
                         float *block_loss, int32_t *status, cudaStream_t stream,
                         int n_cand = 0, int p = 0, int q = 0)
{
    const bool bf = dtype == FP4_BF16;
    const uint16_t *xb = static_cast<const uint16_t *>(x);
    const float *xf = static_cast<const float *>(x);
    if (n_cand == 0)
        return bf ? launch_search_t<uint16_t, true>(xb, n, amax, packed, scales, global_scale, block_loss, status,
                                                    stream, 0, 0, 0)
                  : launch_search_t<float, true>(xf, n, amax, packed, scales, global_scale, block_loss, status,
                                                 stream, 0, 0, 0);
    return bf ? launch_search_t<uint16_t, false>(xb, n, amax, packed, scales, global_scale, block_loss, status,
                                                 stream, n_cand, p, q)
              : launch_search_t<float, false>(xf, n, amax, packed, scales, global_scale, block_loss, status,
                                              stream, n_cand, p, q);
}
} // namespace

extern "C" {

const char *fp4_status_string(int status)
{
    switch (status) {
    case FP4_OK: return "ok";
    case FP4_ERR_INVALID_ARG: return "invalid argument";
    case FP4_ERR_SHAPE: return "shape: incomplete block or size overflow";
    case FP4_ERR_ALIGN: return "pointer misaligned (x, y: 32 bytes; packed: 16 bytes)";
    case FP4_ERR_NONFINITE: return "non-finite input";
    case FP4_ERR_RANGE: return "global scale out of range";
    case FP4_ERR_WORKSPACE: return "workspace missing or too small";
    case FP4_ERR_CUDA: return "CUDA launch failure";
    case FP4_ERR_TIMEOUT: return "a bounded device wait ran out";
    default: return "unknown status";
    }
}

int fp4_version(void) { return 100; }

fp4_status fp4_set_launch_unit_limit(int64_t units)
{
    if (units == 0)
        units = fp4::kMaxUnitsPerLaunch;
    if (units < 64 || units > fp4::kMaxUnitsPerLaunch || units % 64)
        return FP4_ERR_INVALID_ARG;
    fp4_launch::g_launch_unit_limit = units;
    return FP4_OK;
}

size_t fp4_workspace_bytes(fp4_format fmt, int64_t rows, int64_t cols)
{
    (void)fmt;
    (void)rows;
    (void)cols;
    return kWsWords * sizeof(uint32_t);
}

fp4_status fp4_tensor_amax(const void *x, fp4_dtype dtype, int64_t n, float *amax,
                           void *workspace, size_t workspace_bytes, int32_t *status,
                           cudaStream_t stream)
{
    if (!amax || !status || !valid_dtype(dtype) || n < 0 || (n > 0 && !x))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32))
        return FP4_ERR_ALIGN;
    if (!workspace || workspace_bytes < fp4_workspace_bytes(FP4_NVFP4, 1, n) ||
        !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    return launch_amax(x, dtype, n, static_cast<uint32_t *>(workspace), amax, status, stream);
}

fp4_status fp4_nvfp4_quantize(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                              uint8_t *packed, uint8_t *scales, float *global_scale,
                              void *workspace, size_t workspace_bytes, int32_t *status,
                              cudaStream_t stream)
{
    if (!global_scale || !status || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    fp4_status st = check_shape(rows, cols, 16);
    if (st != FP4_OK)
        return st;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16))
        return FP4_ERR_ALIGN;
    if (!workspace || workspace_bytes < fp4_workspace_bytes(FP4_NVFP4, rows, cols) ||
        !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    uint32_t *ws = static_cast<uint32_t *>(workspace);
    float *amax = reinterpret_cast<float *>(ws + kWsAmax);
    st = launch_amax(x, dtype, n, ws, amax, status, stream);
    if (st != FP4_OK)
        return st;
    return launch_nv_quantize(x, dtype, n, amax, packed, scales, global_scale, status, stream);
}

fp4_status fp4_nvfp4_quantize_with_amax(const void *x, fp4_dtype dtype, int64_t rows,
                                        int64_t cols, const float *amax, uint8_t *packed,
                                        uint8_t *scales, float *global_scale, int32_t *status,
                                        cudaStream_t stream)
{
    if (!global_scale || !status || !amax || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    fp4_status st = check_shape(rows, cols, 16);
    if (st != FP4_OK)
        return st;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16) || !aligned(amax, 4))
        return FP4_ERR_ALIGN;
    return launch_nv_quantize(x, dtype, n, amax, packed, scales, global_scale, status, stream);
}

fp4_status fp4_mxfp4_quantize(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                              uint8_t *packed, uint8_t *scales, int32_t *status,
                              cudaStream_t stream)
{
    return mxfp4_quantize_rule<false>(x, dtype, rows, cols, packed, scales, status, stream);
}

fp4_status fp4_mxfp4_quantize_ceil(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                                   uint8_t *packed, uint8_t *scales, int32_t *status,
                                   cudaStream_t stream)
{
    return mxfp4_quantize_rule<true>(x, dtype, rows, cols, packed, scales, status, stream);
}

fp4_status fp4_dequantize(fp4_format fmt, const uint8_t *packed, const uint8_t *scales,
                          const float *global_scale, int64_t rows, int64_t cols, void *y,
                          fp4_dtype out_dtype, cudaStream_t stream)
{
    if ((fmt != FP4_NVFP4 && fmt != FP4_MXFP4) || !valid_dtype(out_dtype))
        return FP4_ERR_INVALID_ARG;
    const bool nv = fmt == FP4_NVFP4;
    fp4_status st = check_shape(rows, cols, nv ? 16 : 32);
    if (st != FP4_OK)
        return st;
    const int64_t n = rows * cols;
    if (n == 0)
        return FP4_OK;
    if (!packed || !scales || !y || (nv && !global_scale))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(y, 32) || (nv && !aligned(global_scale, 4)))
        return FP4_ERR_ALIGN;
    const uint2 *pk = reinterpret_cast<const uint2 *>(packed);
    auto run = [&](auto kernel, auto *yt) {
        return for_chunks(n / 16, [&](int64_t first, int count) {
            const int grid = grid_for(kernel, count, (int64_t)kThreads * fp4::kDequantUnits, kThreads, 0,
                                      fp4::kDequantCtasPerSm);
            if (grid <= 0)
                return FP4_ERR_CUDA;
            return launch(kernel, grid, stream, pk + first, scales + (nv ? first : first / 2),
                          global_scale, count, yt + first * 16);
        });
    };
    if (nv && out_dtype == FP4_BF16)
        return run(fp4::dequantize_kernel<true, uint16_t>, static_cast<uint16_t *>(y));
    if (nv)
        return run(fp4::dequantize_kernel<true, float>, static_cast<float *>(y));
    if (out_dtype == FP4_BF16)
        return run(fp4::dequantize_kernel<false, uint16_t>, static_cast<uint16_t *>(y));
    return run(fp4::dequantize_kernel<false, float>, static_cast<float *>(y));
}


fp4_status fp4_scale_search(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
                            uint8_t *packed, uint8_t *scales, float *global_scale,
                            float *block_loss, void *workspace, size_t workspace_bytes,
                            int32_t *status, cudaStream_t stream)
{
    if (!global_scale || !status || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    fp4_status st = check_shape(rows, cols, 16);
    if (st != FP4_OK)
        return st;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16) || !aligned(block_loss, 4))
        return FP4_ERR_ALIGN;
    if (!workspace || workspace_bytes < fp4_workspace_bytes(FP4_NVFP4, rows, cols) ||
        !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    uint32_t *ws = static_cast<uint32_t *>(workspace);
    float *amax = reinterpret_cast<float *>(ws + kWsAmax);
    st = launch_amax(x, dtype, n, ws, amax, status, stream);
    if (st != FP4_OK)
        return st;
    return launch_search(x, dtype, n, amax, packed, scales, global_scale, block_loss, status,
                         stream);
}

fp4_status fp4_scale_search_grid(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols, int n_cand, int p,
                                 int q, uint8_t *packed, uint8_t *scales, float *global_scale, float *block_loss,
                                 void *workspace, size_t workspace_bytes, int32_t *status, cudaStream_t stream)
{
    if (n_cand < 1 || p < 16 || q < 1 || (int64_t)p + n_cand - 1 > (1 << 20) || q > (1 << 20))
        return FP4_ERR_INVALID_ARG;
    if (!global_scale || !status || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    fp4_status st = check_shape(rows, cols, 16);
    if (st != FP4_OK)
        return st;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16) || !aligned(block_loss, 4))
        return FP4_ERR_ALIGN;
    if (!workspace || workspace_bytes < fp4_workspace_bytes(FP4_NVFP4, rows, cols) ||
        !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    uint32_t *ws = static_cast<uint32_t *>(workspace);
    float *amax = reinterpret_cast<float *>(ws + kWsAmax);
    st = launch_amax(x, dtype, n, ws, amax, status, stream);
    if (st != FP4_OK)
        return st;
    return launch_search(x, dtype, n, amax, packed, scales, global_scale, block_loss, status, stream, n_cand,
                         p, q);
}

fp4_status fp4_scale_search_with_amax(const void *x, fp4_dtype dtype, int64_t rows,
                                      int64_t cols, const float *amax, uint8_t *packed,
                                      uint8_t *scales, float *global_scale, float *block_loss,
                                      int32_t *status, cudaStream_t stream)
{
    if (!global_scale || !status || !amax || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    fp4_status st = check_shape(rows, cols, 16);
    if (st != FP4_OK)
        return st;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16) || !aligned(block_loss, 4) || !aligned(amax, 4))
        return FP4_ERR_ALIGN;
    return launch_search(x, dtype, n, amax, packed, scales, global_scale, block_loss, status,
                         stream);
}

fp4_status fp4_nvfp4_quantize_four_over_six(const void *x, fp4_dtype dtype, int64_t rows,
                                            int64_t cols, uint8_t *packed, uint8_t *scales,
                                            float *global_scale, float *block_loss,
                                            void *workspace, size_t workspace_bytes,
                                            int32_t *status, cudaStream_t stream)
{
    if (!global_scale || !status || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    fp4_status st = check_shape(rows, cols, 16);
    if (st != FP4_OK)
        return st;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16) || !aligned(block_loss, 4))
        return FP4_ERR_ALIGN;
    if (!workspace || workspace_bytes < fp4_workspace_bytes(FP4_NVFP4, rows, cols) ||
        !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    uint32_t *ws = static_cast<uint32_t *>(workspace);
    float *amax = reinterpret_cast<float *>(ws + kWsAmax);
    st = launch_amax(x, dtype, n, ws, amax, status, stream);
    if (st != FP4_OK)
        return st;
    if (dtype == FP4_BF16)
        return launch_block_kernel(fp4::nvfp4_four_over_six_kernel<uint16_t>,
                                   static_cast<const uint16_t *>(x), n, amax, packed, scales,
                                   global_scale, block_loss, status, stream);
    return launch_block_kernel(fp4::nvfp4_four_over_six_kernel<float>,
                               static_cast<const float *>(x), n, amax, packed, scales,
                               global_scale, block_loss, status, stream);
}

fp4_status fp4_e2m1_round(const float *v, uint8_t *codes, int64_t n, cudaStream_t stream)
{
    if (n < 0 || (n > 0 && (!v || !codes)))
        return FP4_ERR_INVALID_ARG;
    if (n == 0)
        return FP4_OK;
    const int grid = grid_for(fp4::e2m1_round_kernel, (n + 7) / 8, kThreads);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    return launch(fp4::e2m1_round_kernel, grid, stream, v, codes, n);
}

fp4_status fp4_e2m1_roundtrip(const float *v, float *out, int64_t n, cudaStream_t stream)
{
    if (n < 0 || (n > 0 && (!v || !out)))
        return FP4_ERR_INVALID_ARG;
    if (n == 0)
        return FP4_OK;
    const int grid = grid_for(fp4::e2m1_roundtrip_kernel, (n + 7) / 8, kThreads);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    return launch(fp4::e2m1_roundtrip_kernel, grid, stream, v, out, n);
}

fp4_status fp4_test_bounded_wait(uint32_t tries, int32_t *status, int64_t *elapsed_ns, cudaStream_t stream)
{
    if (tries < 1 || tries > fp4::kWaitTries || !status || !elapsed_ns)
        return FP4_ERR_INVALID_ARG;
    return launch_cfg(fp4::bounded_wait_test_kernel, dim3(1), 32, 0, stream, tries, status,
                      reinterpret_cast<long long *>(elapsed_ns));
}

fp4_status fp4_nv_encode_quotient(const float *x, const float *d, uint8_t *codes, int64_t n,
                                  cudaStream_t stream)
{
    if (n < 0 || (n > 0 && (!x || !d || !codes)))
        return FP4_ERR_INVALID_ARG;
    if (n == 0)
        return FP4_OK;
    const int grid = grid_for(fp4::nv_encode_quotient_kernel, n, kThreads);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    return launch(fp4::nv_encode_quotient_kernel, grid, stream, x, d, codes, n);
}

} // extern "C"
