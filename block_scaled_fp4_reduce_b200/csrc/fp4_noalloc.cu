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
// only its inputs and outputs.  It launches the same two kernels, through the
// same launch helpers, as fp4_nvfp4_quantize.
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
//   - In host code the array's name is only a host-side stand-in.  Every
//     call asks the runtime for the array's device address in the current
//     context (cudaGetSymbolAddress), so a call made in another context
//     than the last one -- a non-primary context, or the primary context
//     again after cudaDeviceReset -- gets that context's copy.  The first
//     call in a context also loads the library's device code there: make it
//     before any stream capture begins.
#include <cstdint>

#include <cuda_runtime.h>

#include "fp4.h"
#include "fp4_kernels.cuh"
#include "fp4_launch.cuh"

namespace {

constexpr size_t kScratchWords = fp4_launch::kWsWords; // maxima, counter, amax word
constexpr size_t kScratchBytes = kScratchWords * sizeof(uint32_t);
constexpr size_t kCounterWord = fp4::kMaxPartials;

static __device__ __align__(256) uint32_t g_scratch[kScratchWords];

// Device address of g_scratch in the current context, or nullptr.
uint32_t *scratch_in_current_context()
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
        (void)cudaGetLastError();
        return nullptr;
    }
    return static_cast<uint32_t *>(p);
}

} // namespace

extern "C" fp4_status fp4_nvfp4_quantize_noalloc(const void *x, fp4_dtype dtype, int64_t rows,
                                                 int64_t cols, uint8_t *packed, uint8_t *scales,
                                                 float *global_scale, int32_t *status,
                                                 cudaStream_t stream)
{
    using namespace fp4_launch;
    if (!global_scale || !status || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0)
        return FP4_ERR_INVALID_ARG;
    if (cols % 16 || (cols > 0 && rows > INT64_MAX / cols / 4))
        return FP4_ERR_SHAPE;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !packed || !scales))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 32) || !aligned(packed, 16))
        return FP4_ERR_ALIGN;
    if (fp4_workspace_bytes(FP4_NVFP4, rows, cols) > kScratchBytes)
        return FP4_ERR_WORKSPACE;
    uint32_t *ws = scratch_in_current_context();
    if (!ws)
        return FP4_ERR_CUDA;
    if (cudaMemsetAsync(ws + kCounterWord, 0, sizeof(uint32_t), stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return FP4_ERR_CUDA;
    }
    float *amax = reinterpret_cast<float *>(ws + kWsAmax);
    const fp4_status st = launch_amax(x, dtype, n, ws, amax, status, stream);
    if (st != FP4_OK)
        return st;
    return launch_nv_quantize(x, dtype, n, amax, packed, scales, global_scale, status, stream);
}
