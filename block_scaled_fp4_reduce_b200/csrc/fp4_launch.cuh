// fp4_launch.cuh -- host-side launch helpers shared by the C-ABI translation
// units: SM count, persistent grid size, launch with programmatic stream
// serialisation, and the split of a problem into launches of at most
// fp4::kMaxUnitsPerLaunch units.  Internal linkage (each translation unit
// keeps its own caches).
#pragma once

#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fp4.h"
#include "fp4_kernels.cuh"

namespace fp4_launch {

// Units per launch of the chunked calls: fp4::kMaxUnitsPerLaunch, or a
// smaller multiple of 64 set by fp4_set_launch_unit_limit (tests only).
// One definition, in fp4_capi.cu.
extern int64_t g_launch_unit_limit;

namespace {

using fp4::kThreads;

constexpr int kMaxDevices = 64;

// Workspace words of the single-tensor calls: fp4::kMaxPartials per-CTA
// maxima, the wrapping CTA counter, and the amax word the NVFP4 quantiser
// and the search read.
constexpr size_t kWsAmax = fp4::kMaxPartials + 1; // word kMaxPartials is the counter
constexpr size_t kWsWords = fp4::kMaxPartials + 8;

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

// Per-device facts about a kernel, cached by the kernel's address (kernels
// of different instantiations can share a function type).
struct KernelFacts {
    const void *kernel;
    int dev;
    int resident;   // resident CTAs per SM (0: not queried yet)
    bool smem_set;  // dynamic shared-memory limit raised
};

KernelFacts &kernel_facts(const void *kernel, int dev)
{
    static std::mutex mu;
    static KernelFacts table[256];
    static int used = 0;
    static KernelFacts spare;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (table[i].kernel == kernel && table[i].dev == dev)
            return table[i];
    if (used == 256) { // more kernels x devices than this library has: no caching
        spare = KernelFacts{kernel, dev, 0, false};
        return spare;
    }
    table[used] = KernelFacts{kernel, dev, 0, false};
    return table[used++];
}

// Resident CTAs per SM of `kernel` at `block` threads and `smem` bytes of
// dynamic shared memory (cached per device and kernel; a kernel is always
// queried with the same block and smem).
template <typename K> int resident_ctas(K kernel, int dev, int block = kThreads, size_t smem = 0)
{
    KernelFacts &f = kernel_facts(reinterpret_cast<const void *>(kernel), dev);
    if (f.resident > 0)
        return f.resident;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, block, smem) != cudaSuccess ||
        n <= 0) {
        (void)cudaGetLastError();
        n = 1;
    }
    f.resident = n;
    return n;
}

// Lets `kernel` launch with `bytes` of dynamic shared memory on the current
// device (above the default 48 KB); false on a CUDA error.
template <typename K> bool smem_attr(K kernel, int bytes)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    KernelFacts &f = kernel_facts(reinterpret_cast<const void *>(kernel), dev);
    if (f.smem_set)
        return true;
    if (cudaFuncSetAttribute(reinterpret_cast<const void *>(kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    f.smem_set = true;
    return true;
}

// Persistent grid: enough CTAs for `work` items at `per_cta` items each,
// at most SMs x resident CTAs (and at most SMs x max_per_sm when given), at
// least one.
template <typename K>
int grid_for(K kernel, int64_t work, int64_t per_cta, int block = kThreads, size_t smem = 0, int max_per_sm = 0)
{
    int dev = 0;
    const int sms = sm_count(dev);
    if (sms <= 0)
        return -1;
    int per_sm = resident_ctas(kernel, dev, block, smem);
    if (max_per_sm > 0 && per_sm > max_per_sm)
        per_sm = max_per_sm;
    const int64_t cap = (int64_t)sms * per_sm;
    int64_t want = (work + per_cta - 1) / per_cta;
    if (want < 1)
        want = 1;
    return (int)(want < cap ? want : cap);
}

// Launch with programmatic stream serialisation: the kernel is launched as
// the previous kernel on the stream retires its CTAs, and waits for it
// (griddepcontrol.wait) before touching memory.
template <typename... KArgs, typename... Args>
fp4_status launch_cfg(void (*kernel)(KArgs...), dim3 grid, int block, size_t smem,
                      cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3((unsigned)block);
    cfg.dynamicSmemBytes = smem;
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

template <typename... KArgs, typename... Args>
fp4_status launch(void (*kernel)(KArgs...), int grid, cudaStream_t stream, Args... args)
{
    return launch_cfg(kernel, grid, kThreads, 0, stream, args...);
}

// Runs one(first, count) over units [0, n) in chunks of at most
// g_launch_unit_limit (the kernels index units with 32-bit integers).
// At least one call is made, with count 0 for an empty problem, so that
// kernels with a prologue (the NVFP4 global scale) still run once.
template <typename F> fp4_status for_chunks(int64_t n, F &&one)
{
    int64_t first = 0;
    do {
        const int64_t left = n - first;
        const int64_t lim = g_launch_unit_limit;
        const int count = (int)(left < lim ? left : lim);
        const fp4_status st = one(first, count);
        if (st != FP4_OK)
            return st;
        first += count;
    } while (first < n);
    return FP4_OK;
}

// Runs one(first_row, count) over rows [0, rows) in chunks whose
// units (rows x units_per_row) stay within g_launch_unit_limit (a row larger
// than that is FP4_ERR_SHAPE); at least one call, as for_chunks.
// units_per_row >= 1.
template <typename F> fp4_status for_row_chunks(int64_t rows, int64_t units_per_row, F &&one)
{
    const int64_t per = g_launch_unit_limit / units_per_row;
    if (per < 1)
        return FP4_ERR_SHAPE;
    int64_t first = 0;
    do {
        const int64_t left = rows - first;
        const int64_t count = left < per ? left : per;
        const fp4_status st = one(first, count);
        if (st != FP4_OK)
            return st;
        first += count;
    } while (first < rows);
    return FP4_OK;
}

// Tensor amax (one launch) into *amax: at most fp4::kMaxPartials CTAs, whose
// maxima go to ws[0 ..), the CTA counter at ws[fp4::kMaxPartials].
inline fp4_status launch_amax(const void *x, fp4_dtype dt, int64_t n, uint32_t *ws, float *amax,
                       int32_t *status, cudaStream_t stream)
{
    const int64_t elems_per_vec = dt == FP4_BF16 ? 16 : 8; // one 32-byte vector
    const int64_t nvec = n / elems_per_vec;
    const int64_t per_cta = (int64_t)kThreads * 4;
    int grid;
    if (dt == FP4_BF16)
        grid = grid_for(fp4::amax_kernel<uint16_t>, nvec, per_cta);
    else
        grid = grid_for(fp4::amax_kernel<float>, nvec, per_cta);
    if (grid <= 0)
        return FP4_ERR_CUDA;
    if (grid > fp4::kMaxPartials)
        grid = fp4::kMaxPartials;
    if (dt == FP4_BF16)
        return launch(fp4::amax_kernel<uint16_t>, grid, stream, static_cast<const uint16_t *>(x), n,
                      ws, amax, status);
    return launch(fp4::amax_kernel<float>, grid, stream, static_cast<const float *>(x), n, ws, amax,
                  status);
}

template <typename T>
fp4_status launch_nv_quantize_t(const T *x, int64_t n, const float *amax, uint8_t *packed,
                                uint8_t *scales, float *global_scale, int32_t *status,
                                cudaStream_t stream)
{
    uint2 *pk = reinterpret_cast<uint2 *>(packed);
    return for_chunks(n / 16, [&](int64_t first, int count) {
        const int grid = grid_for(fp4::nvfp4_quantize_kernel<T>, count, (int64_t)kThreads * 2);
        if (grid <= 0)
            return FP4_ERR_CUDA;
        return launch(fp4::nvfp4_quantize_kernel<T>, grid, stream, x + first * 16, count, amax,
                      pk + first, scales + first, global_scale, status);
    });
}

// NVFP4 quantise pass given the tensor amax at *amax, in launches of at
// most g_launch_unit_limit blocks.
inline fp4_status launch_nv_quantize(const void *x, fp4_dtype dt, int64_t n, const float *amax,
                              uint8_t *packed, uint8_t *scales, float *global_scale,
                              int32_t *status, cudaStream_t stream)
{
    if (dt == FP4_BF16)
        return launch_nv_quantize_t(static_cast<const uint16_t *>(x), n, amax, packed, scales,
                                    global_scale, status, stream);
    return launch_nv_quantize_t(static_cast<const float *>(x), n, amax, packed, scales,
                                global_scale, status, stream);
}

bool valid_dtype(fp4_dtype t) { return t == FP4_F32 || t == FP4_BF16; }

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                 const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                 const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
EncodeTiled encode_tiled()
{
    static std::once_flag once;
    static EncodeTiled fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
        else
            (void)cudaGetLastError();
    });
    return fn;
}


} // namespace
} // namespace fp4_launch
