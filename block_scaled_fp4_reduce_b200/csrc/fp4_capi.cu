// fp4_capi.cu -- the extern "C" entry points declared in include/fp4.h.
//
// Argument checking and launch configuration only: every step of the path
// runs in the kernels of fp4_kernels.cuh.  Nothing here allocates, frees or
// synchronises; every launch goes on the caller's stream.
#include <climits>
#include <cstdint>

#include <cuda_runtime.h>

#include "fp4.h"
#include "fp4_kernels.cuh"

namespace {

using fp4::kMaxPartials;
using fp4::kThreads;

constexpr int kMaxDevices = 64;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// SM count of the current device (cached per device).
int sm_count(int &dev)
{
    static int cache[kMaxDevices] = {0};
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return -1;
    if (dev < kMaxDevices && cache[dev] > 0)
        return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return -1;
    if (dev < kMaxDevices)
        cache[dev] = n;
    return n;
}

// Resident CTAs per SM of `kernel` at kThreads threads (cached per device
// and kernel instantiation).
template <typename K> int resident_ctas(K kernel, int dev)
{
    static int cache[kMaxDevices] = {0};
    if (dev < kMaxDevices && cache[dev] > 0)
        return cache[dev];
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, 0) != cudaSuccess ||
        n <= 0)
        n = 1;
    if (dev < kMaxDevices)
        cache[dev] = n;
    return n;
}

// Persistent grid: enough CTAs for `work` items at `per_cta` items each,
// at most SMs x resident CTAs, at least one.
template <typename K> int grid_for(K kernel, int64_t work, int64_t per_cta)
{
    int dev = 0;
    const int sms = sm_count(dev);
    if (sms <= 0)
        return -1;
    const int64_t cap = (int64_t)sms * resident_ctas(kernel, dev);
    int64_t want = (work + per_cta - 1) / per_cta;
    if (want < 1)
        want = 1;
    return (int)(want < cap ? want : cap);
}

fp4_status launched()
{
    return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

bool valid_dtype(fp4_dtype t) { return t == FP4_F32 || t == FP4_BF16; }

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

// Tensor amax, pass 1: returns the number of partials written (>= 0), or
// -1 on a launch-configuration failure.
int launch_amax_partials(const void *x, fp4_dtype dt, int64_t n, uint32_t *partials,
                         cudaStream_t stream)
{
    if (n == 0)
        return 0;
    const int64_t elems_per_vec = dt == FP4_BF16 ? 8 : 4;
    const int64_t nvec = n / elems_per_vec;
    const int64_t per_cta = (int64_t)kThreads * 4;
    int grid;
    if (dt == FP4_BF16)
        grid = grid_for(fp4::amax_partial_kernel<uint16_t>, nvec, per_cta);
    else
        grid = grid_for(fp4::amax_partial_kernel<float>, nvec, per_cta);
    if (grid <= 0)
        return -1;
    if (grid > kMaxPartials)
        grid = kMaxPartials;
    if (dt == FP4_BF16)
        fp4::amax_partial_kernel<uint16_t>
            <<<grid, kThreads, 0, stream>>>(static_cast<const uint16_t *>(x), n, partials);
    else
        fp4::amax_partial_kernel<float>
            <<<grid, kThreads, 0, stream>>>(static_cast<const float *>(x), n, partials);
    return grid;
}

fp4_status launch_nv_quantize(const void *x, fp4_dtype dt, int64_t n, const uint32_t *partials,
                              int nparts, uint8_t *packed, uint8_t *scales, float *global_scale,
                              int32_t *status, cudaStream_t stream)
{
    const int64_t n_units = n / 8;
    const int64_t per_cta = (int64_t)kThreads * 2;
    int grid;
    if (dt == FP4_BF16)
        grid = grid_for(fp4::nvfp4_quantize_kernel<uint16_t>, n_units, per_cta);
    else
        grid = grid_for(fp4::nvfp4_quantize_kernel<float>, n_units, per_cta);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    uint32_t *pk = reinterpret_cast<uint32_t *>(packed);
    if (dt == FP4_BF16)
        fp4::nvfp4_quantize_kernel<uint16_t><<<grid, kThreads, 0, stream>>>(
            static_cast<const uint16_t *>(x), n_units, partials, nparts, pk, scales, global_scale,
            status);
    else
        fp4::nvfp4_quantize_kernel<float><<<grid, kThreads, 0, stream>>>(
            static_cast<const float *>(x), n_units, partials, nparts, pk, scales, global_scale,
            status);
    return launched();
}

} // namespace

extern "C" {

const char *fp4_status_string(int status)
{
    switch (status) {
    case FP4_OK: return "ok";
    case FP4_ERR_INVALID_ARG: return "invalid argument";
    case FP4_ERR_SHAPE: return "shape: incomplete block or size overflow";
    case FP4_ERR_ALIGN: return "pointer not 16-byte aligned";
    case FP4_ERR_NONFINITE: return "non-finite input";
    case FP4_ERR_RANGE: return "global scale out of range";
    case FP4_ERR_WORKSPACE: return "workspace missing or too small";
    case FP4_ERR_CUDA: return "CUDA launch failure";
    default: return "unknown status";
    }
}

int fp4_version(void) { return 100; }

size_t fp4_workspace_bytes(fp4_format fmt, int64_t rows, int64_t cols)
{
    (void)fmt;
    (void)rows;
    (void)cols;
    return (size_t)kMaxPartials * sizeof(uint32_t);
}

fp4_status fp4_tensor_amax(const void *x, fp4_dtype dtype, int64_t n, float *amax,
                           void *workspace, size_t workspace_bytes, int32_t *status,
                           cudaStream_t stream)
{
    if (!amax || !status || !valid_dtype(dtype) || n < 0 || (n > 0 && !x))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 16))
        return FP4_ERR_ALIGN;
    if (!workspace || workspace_bytes < fp4_workspace_bytes(FP4_NVFP4, 1, n) ||
        !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    uint32_t *partials = static_cast<uint32_t *>(workspace);
    const int nparts = launch_amax_partials(x, dtype, n, partials, stream);
    if (nparts < 0)
        return FP4_ERR_CUDA;
    fp4::amax_finalize_kernel<<<1, kThreads, 0, stream>>>(partials, nparts, amax, status);
    return launched();
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
    if (!aligned(x, 16) || !aligned(packed, 16))
        return FP4_ERR_ALIGN;
    if (!workspace || workspace_bytes < fp4_workspace_bytes(FP4_NVFP4, rows, cols) ||
        !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    uint32_t *partials = static_cast<uint32_t *>(workspace);
    const int nparts = launch_amax_partials(x, dtype, n, partials, stream);
    if (nparts < 0)
        return FP4_ERR_CUDA;
    return launch_nv_quantize(x, dtype, n, partials, nparts, packed, scales, global_scale, status,
                              stream);
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
    if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(amax, 4))
        return FP4_ERR_ALIGN;
    return launch_nv_quantize(x, dtype, n, reinterpret_cast<const uint32_t *>(amax), 1, packed,
                              scales, global_scale, status, stream);
}

fp4_status fp4_mxfp4_quantize(const void *x, fp4_dtype dtype, int64_t rows, int64_t cols,
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
    if (!aligned(x, 16) || !aligned(packed, 16))
        return FP4_ERR_ALIGN;
    const int64_t n_units = n / 8;
    const int64_t per_cta = (int64_t)kThreads * 2;
    uint32_t *pk = reinterpret_cast<uint32_t *>(packed);
    if (dtype == FP4_BF16) {
        const int grid = grid_for(fp4::mxfp4_quantize_kernel<uint16_t>, n_units, per_cta);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        fp4::mxfp4_quantize_kernel<uint16_t><<<grid, kThreads, 0, stream>>>(
            static_cast<const uint16_t *>(x), n_units, pk, scales, status);
    } else {
        const int grid = grid_for(fp4::mxfp4_quantize_kernel<float>, n_units, per_cta);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        fp4::mxfp4_quantize_kernel<float><<<grid, kThreads, 0, stream>>>(
            static_cast<const float *>(x), n_units, pk, scales, status);
    }
    return launched();
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
    if (!aligned(packed, 16) || !aligned(y, 16) || (nv && !aligned(global_scale, 4)))
        return FP4_ERR_ALIGN;
    const int64_t n_units = n / 8;
    const int64_t per_cta = (int64_t)kThreads * 4;
    const uint32_t *pk = reinterpret_cast<const uint32_t *>(packed);
#define FP4_DEQ_LAUNCH(NV, TOUT)                                                                \
    do {                                                                                        \
        const int grid = grid_for(fp4::dequantize_kernel<NV, TOUT>, n_units, per_cta);          \
        if (grid <= 0)                                                                          \
            return FP4_ERR_CUDA;                                                                \
        fp4::dequantize_kernel<NV, TOUT><<<grid, kThreads, 0, stream>>>(                        \
            pk, scales, global_scale, n_units, static_cast<TOUT *>(y));                         \
    } while (0)
    if (nv && out_dtype == FP4_BF16)
        FP4_DEQ_LAUNCH(true, uint16_t);
    else if (nv)
        FP4_DEQ_LAUNCH(true, float);
    else if (out_dtype == FP4_BF16)
        FP4_DEQ_LAUNCH(false, uint16_t);
    else
        FP4_DEQ_LAUNCH(false, float);
#undef FP4_DEQ_LAUNCH
    return launched();
}

namespace {
fp4_status launch_search(const void *x, fp4_dtype dtype, int64_t n, const uint32_t *partials,
                         int nparts, uint8_t *packed, uint8_t *scales, float *global_scale,
                         float *block_loss, int32_t *status, cudaStream_t stream)
{
    const int64_t n_blocks = n / 16;
    uint2 *pk = reinterpret_cast<uint2 *>(packed);
    if (dtype == FP4_BF16) {
        const int grid = grid_for(fp4::scale_search_kernel<uint16_t>, n_blocks, kThreads);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        fp4::scale_search_kernel<uint16_t><<<grid, kThreads, 0, stream>>>(
            static_cast<const uint16_t *>(x), n_blocks, partials, nparts, pk, scales,
            global_scale, block_loss, status);
    } else {
        const int grid = grid_for(fp4::scale_search_kernel<float>, n_blocks, kThreads);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        fp4::scale_search_kernel<float><<<grid, kThreads, 0, stream>>>(
            static_cast<const float *>(x), n_blocks, partials, nparts, pk, scales, global_scale,
            block_loss, status);
    }
    return launched();
}
} // namespace

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
    if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(block_loss, 4))
        return FP4_ERR_ALIGN;
    if (!workspace || workspace_bytes < fp4_workspace_bytes(FP4_NVFP4, rows, cols) ||
        !aligned(workspace, 4))
        return FP4_ERR_WORKSPACE;
    uint32_t *partials = static_cast<uint32_t *>(workspace);
    const int nparts = launch_amax_partials(x, dtype, n, partials, stream);
    if (nparts < 0)
        return FP4_ERR_CUDA;
    return launch_search(x, dtype, n, partials, nparts, packed, scales, global_scale, block_loss,
                         status, stream);
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
    if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(block_loss, 4) || !aligned(amax, 4))
        return FP4_ERR_ALIGN;
    return launch_search(x, dtype, n, reinterpret_cast<const uint32_t *>(amax), 1, packed, scales,
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
    fp4::e2m1_round_kernel<<<grid, kThreads, 0, stream>>>(v, codes, n);
    return launched();
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
    fp4::nv_encode_quotient_kernel<<<grid, kThreads, 0, stream>>>(x, d, codes, n);
    return launched();
}

} // extern "C"
