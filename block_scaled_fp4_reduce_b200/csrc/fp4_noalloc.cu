// fp4_noalloc.cu -- fp4_nvfp4_quantize_noalloc: the NVFP4 quantiser for
// callers that cannot allocate device memory.
//
// fp4_nvfp4_quantize needs a small device workspace (the per-CTA maxima of
// the tensor amax, a CTA counter and the amax word) and asks its caller for
// it.  Some callers have no way to provide one: code running where
// allocation is forbidden -- the execute callback of an inference-engine
// plugin, or a serving loop that must not call cudaMalloc once requests are
// flowing -- or where the whole device memory budget was reserved up front
// and handed out as tensors only.  This entry point keeps that workspace in a
// file-scope __device__ array of the library instead, so the caller passes
// only its inputs and outputs.
//
// Costs and limits:
//   - The array is kScratchBytes (4128) bytes; every GPU that loads the
//     library holds it until the process exits.
//   - It serves every shape fp4_nvfp4_quantize accepts (the workspace that
//     function needs does not grow with the tensor); a shape needing more
//     would be rejected with FP4_ERR_WORKSPACE.
//   - All calls on a device share the one array.  Calls whose kernels
//     overlap on the GPU (different streams, or different host threads
//     without ordering) race on it and give wrong results: order them.
//   - The array keeps whatever the last call left in it; each call clears
//     the CTA counter (the only word that must start at zero) on its stream
//     before launching.
//   - The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current and caches it; make
//     that first call before any stream capture begins.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "fp4.h"
#include "fp4_kernels.cuh"

namespace {

constexpr size_t kScratchWords = fp4::kMaxPartials + 8; // maxima, counter, amax word
constexpr size_t kScratchBytes = kScratchWords * sizeof(uint32_t);
constexpr size_t kCounterWord = fp4::kMaxPartials;
constexpr size_t kAmaxWord = fp4::kMaxPartials + 1;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint32_t g_scratch[kScratchWords];

std::mutex g_setup_mutex;
uint32_t *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_scratch on the current device (looked up once per
// device; in host code the symbol name is only a host-side stand-in).
uint32_t *scratch_on_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return nullptr;
        }
        g_scratch_ptr[dev] = static_cast<uint32_t *>(p);
    }
    return g_scratch_ptr[dev];
}

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    return n;
}

template <typename K> int persistent_grid(K kernel, int64_t work, int64_t per_cta)
{
    const int sms = sm_count();
    int per_sm = 0;
    if (sms <= 0 ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, fp4::kThreads, 0) !=
            cudaSuccess)
        return -1;
    if (per_sm < 1)
        per_sm = 1;
    const int64_t cap = (int64_t)sms * per_sm;
    int64_t want = (work + per_cta - 1) / per_cta;
    if (want < 1)
        want = 1;
    return (int)(want < cap ? want : cap);
}

template <typename... KArgs, typename... Args>
fp4_status launch_chained(void (*kernel)(KArgs...), int grid, cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(fp4::kThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) {
        (void)cudaGetLastError();
        return FP4_ERR_CUDA;
    }
    return FP4_OK;
}

template <typename T>
fp4_status quantize_with_static_scratch(const T *x, int64_t rows, int64_t cols, uint8_t *packed,
                                        uint8_t *scales, float *global_scale, int32_t *status,
                                        cudaStream_t stream, uint32_t *ws)
{
    const int64_t n = rows * cols;
    float *amax = reinterpret_cast<float *>(ws + kAmaxWord);
    const int64_t nvec = n / (32 / (int64_t)sizeof(T));
    int grid = persistent_grid(fp4::amax_kernel<T>, nvec, (int64_t)fp4::kThreads * 4);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    if (grid > fp4::kMaxPartials)
        grid = fp4::kMaxPartials;
    fp4_status st = launch_chained(fp4::amax_kernel<T>, grid, stream, x, n, ws, amax, status);
    if (st != FP4_OK)
        return st;
    // 32-bit block indices in the kernel: chunks of at most 2^30 blocks, and
    // one launch even for an empty tensor (it publishes g).
    const int64_t n_blocks = n / 16;
    int64_t first = 0;
    do {
        const int64_t left = n_blocks - first;
        const int count = (int)(left < fp4::kMaxUnitsPerLaunch ? left : fp4::kMaxUnitsPerLaunch);
        grid = persistent_grid(fp4::nvfp4_quantize_kernel<T>, count, (int64_t)fp4::kThreads * 2);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        st = launch_chained(fp4::nvfp4_quantize_kernel<T>, grid, stream, x + first * 16, count,
                            static_cast<const float *>(amax),
                            reinterpret_cast<uint2 *>(packed) + first, scales + first,
                            global_scale, status);
        if (st != FP4_OK)
            return st;
        first += count;
    } while (first < n_blocks);
    return FP4_OK;
}

} // namespace

extern "C" fp4_status fp4_nvfp4_quantize_noalloc(const void *x, fp4_dtype dtype, int64_t rows,
                                                 int64_t cols, uint8_t *packed, uint8_t *scales,
                                                 float *global_scale, int32_t *status,
                                                 cudaStream_t stream)
{
    if (!global_scale || !status || (dtype != FP4_F32 && dtype != FP4_BF16))
        return FP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0)
        return FP4_ERR_INVALID_ARG;
    if (cols % 16 || (cols > 0 && rows > INT64_MAX / cols / 4))
        return FP4_ERR_SHAPE;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 31) || (reinterpret_cast<uintptr_t>(packed) & 15))
        return FP4_ERR_ALIGN;
    if (fp4_workspace_bytes(FP4_NVFP4, rows, cols) > kScratchBytes)
        return FP4_ERR_WORKSPACE;
    uint32_t *ws = scratch_on_current_device();
    if (!ws)
        return FP4_ERR_CUDA;
    if (cudaMemsetAsync(ws + kCounterWord, 0, sizeof(uint32_t), stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return FP4_ERR_CUDA;
    }
    if (dtype == FP4_BF16)
        return quantize_with_static_scratch(static_cast<const uint16_t *>(x), rows, cols, packed,
                                            scales, global_scale, status, stream, ws);
    return quantize_with_static_scratch(static_cast<const float *>(x), rows, cols, packed, scales,
                                        global_scale, status, stream, ws);
}
