// fp4_grouped.cu -- the grouped entry points of include/fp4.h: many matrices
// per call, each quantised with its own scales, in a few launches.
//
// Host side only: argument checks, the split of the item list into launch
// tables (fp4_grouped.cuh), and the launches.  The item arrays are read
// during the call and not kept.
#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "fp4.h"
#include "fp4_grouped.cuh"
#include "fp4_launch.cuh"

namespace {

using namespace fp4_launch;
using fp4::kGroupMax;
using fp4::kThreads;

// One grid thread per entry publishes the entry's g (NVFP4).
static_assert(kGroupMax <= kThreads, "a one-CTA grid must cover every entry");

// Packs items into launch tables of at most kGroupMax entries and at most
// fp4::kMaxUnitsPerLaunch units.  An item that does not fit in what is left
// of a launch is split at a multiple of 64 units (so that an MXFP4 dequant
// piece starts on an even unit); an empty item still gets an entry.
// set(table, k, item, first_unit_of_piece, units) fills entry k; go(table)
// launches a full table.  max_units (>= 64) and max_entries (1 ..
// kGroupMax) are lowered only by the planner test below.
template <typename Table, typename Units, typename Set, typename Go>
fp4_status plan(int n_items, Units &&units_of, Set &&set, Go &&go,
                int64_t max_units = 0, int max_entries = kGroupMax)
{
    if (max_units <= 0)
        max_units = g_launch_unit_limit;
    Table t;
    std::memset(&t, 0, sizeof(t));
    int64_t total = 0;
    for (int it = 0; it < n_items; ++it) {
        const int64_t units = units_of(it);
        int64_t off = 0;
        for (;;) {
            const int64_t cap = max_units - total;
            if (t.n == max_entries || (cap < 64 && off < units)) {
                const fp4_status st = go(t);
                if (st != FP4_OK)
                    return st;
                std::memset(&t, 0, sizeof(t));
                total = 0;
                continue;
            }
            const int64_t left = units - off;
            const int64_t take = left <= cap ? left : (cap & ~(int64_t)63);
            set(t, t.n, it, off, take);
            t.first[t.n + 1] = t.first[t.n] + (int)take;
            ++t.n;
            total += take;
            off += take;
            if (off >= units)
                break;
        }
    }
    if (t.n > 0)
        return go(t);
    return FP4_OK;
}

// What a call reads or writes of an item, for the checks.
enum ItemUse { kInputOnly, kMx, kNv };

// Shape and pointer checks of one quantisation item.
fp4_status check_quant_item(const fp4_quant_item &q, int64_t block, ItemUse use)
{
    if (q.rows < 0 || q.cols < 0)
        return FP4_ERR_INVALID_ARG;
    if (q.cols % block || (q.cols > 0 && q.rows > INT64_MAX / q.cols / 4))
        return FP4_ERR_SHAPE;
    const bool outputs = use != kInputOnly, nv = use == kNv;
    if (nv && !q.global_scale)
        return FP4_ERR_INVALID_ARG;
    if (q.rows * q.cols > 0 && (!q.x || (outputs && (!q.packed || !q.scales))))
        return FP4_ERR_INVALID_ARG;
    if (!aligned(q.x, 32) || (outputs && !aligned(q.packed, 16)) ||
        (nv && !aligned(q.global_scale, 4)))
        return FP4_ERR_ALIGN;
    return FP4_OK;
}

template <typename T>
fp4_status amax_grouped(const fp4_quant_item *items, int n_items, uint32_t *amax_words,
                        int32_t *status, cudaStream_t stream)
{
    constexpr int64_t kPerVec = 32 / (int64_t)sizeof(T);
    if (cudaMemsetAsync(amax_words, 0, (size_t)n_items * sizeof(uint32_t), stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return FP4_ERR_CUDA;
    }
    auto nvec = [&](int it) { return items[it].rows * items[it].cols / kPerVec; };
    return plan<fp4::AmaxGroup>(
        n_items,
        [&](int it) { return (nvec(it) + fp4::kAmaxChunkVecs - 1) / fp4::kAmaxChunkVecs; },
        [&](fp4::AmaxGroup &t, int k, int it, int64_t off, int64_t take) {
            const int64_t v0 = off * fp4::kAmaxChunkVecs;
            const int64_t left = nvec(it) - v0;
            t.x[k] = static_cast<const T *>(items[it].x) + v0 * kPerVec;
            t.nvec[k] = left < take * fp4::kAmaxChunkVecs ? left : take * fp4::kAmaxChunkVecs;
            t.amax[k] = amax_words + it;
        },
        [&](const fp4::AmaxGroup &t) {
            const int grid = grid_for(fp4::amax_grouped_kernel<T>, t.first[t.n], 1);
            if (grid <= 0)
                return FP4_ERR_CUDA;
            return launch(fp4::amax_grouped_kernel<T>, grid, stream, t, status);
        });
}

template <typename T>
fp4_status nv_grouped_with_amax(const fp4_quant_item *items, int n_items,
                                const uint32_t *amax_words, int32_t *status, cudaStream_t stream)
{
    return plan<fp4::NvGroup>(
        n_items, [&](int it) { return items[it].rows * items[it].cols / 16; },
        [&](fp4::NvGroup &t, int k, int it, int64_t off, int64_t take) {
            t.x[k] = static_cast<const T *>(items[it].x) + off * 16;
            t.packed[k] = reinterpret_cast<uint2 *>(items[it].packed) + off;
            t.scales[k] = items[it].scales + off;
            t.amax[k] = amax_words + it;
            t.global_scale[k] = items[it].global_scale;
            t.tile_first[k + 1] = t.tile_first[k] + fp4::grouped_tile_count(take, fp4::kNvGroupedU);
        },
        [&](const fp4::NvGroup &t) {
            // one CTA at least: its first threads publish every entry's g
            const int grid = grid_for(fp4::nvfp4_quantize_grouped_kernel<T>, t.tile_first[t.n], 1);
            if (grid <= 0)
                return FP4_ERR_CUDA;
            return launch(fp4::nvfp4_quantize_grouped_kernel<T>, grid, stream, t, status);
        });
}

fp4_status check_quant_items(const fp4_quant_item *items, int n_items, fp4_dtype dtype,
                             const int32_t *status, int64_t block, ItemUse use)
{
    if (n_items < 0 || (n_items > 0 && !items) || !status || !valid_dtype(dtype))
        return FP4_ERR_INVALID_ARG;
    for (int i = 0; i < n_items; ++i) {
        const fp4_status st = check_quant_item(items[i], block, use);
        if (st != FP4_OK)
            return st;
    }
    return FP4_OK;
}

fp4_status check_workspace(const void *workspace, size_t bytes, int n_items)
{
    if (!workspace || bytes < fp4_grouped_workspace_bytes(n_items) ||
        (reinterpret_cast<uintptr_t>(workspace) & 3))
        return FP4_ERR_WORKSPACE;
    return FP4_OK;
}

template <typename T, bool kCeil>
fp4_status mx_grouped(const fp4_quant_item *items, int n_items, int32_t *status, cudaStream_t stream)
{
    return plan<fp4::MxGroup>(
        n_items, [&](int it) { return items[it].rows * items[it].cols / 32; },
        [&](fp4::MxGroup &t, int k, int it, int64_t off, int64_t take) {
            t.x[k] = static_cast<const T *>(items[it].x) + off * 32;
            t.packed[k] = reinterpret_cast<uint4 *>(items[it].packed) + off;
            t.scales[k] = items[it].scales + off;
            t.tile_first[k + 1] = t.tile_first[k] + fp4::grouped_tile_count(take, fp4::kMxGroupedU);
        },
        [&](const fp4::MxGroup &t) {
            const int grid = grid_for(fp4::mxfp4_quantize_grouped_kernel<T, kCeil>, t.tile_first[t.n], 1);
            if (grid <= 0)
                return FP4_ERR_CUDA;
            return launch(fp4::mxfp4_quantize_grouped_kernel<T, kCeil>, grid, stream, t, status);
        });
}

template <bool kNv, typename TOut>
fp4_status dq_grouped(const fp4_dequant_item *items, int n_items, cudaStream_t stream)
{
    return plan<fp4::DqGroup>(
        n_items, [&](int it) { return items[it].rows * items[it].cols / 16; },
        [&](fp4::DqGroup &t, int k, int it, int64_t off, int64_t take) {
            t.packed[k] = reinterpret_cast<const uint2 *>(items[it].packed) + off;
            t.scales[k] = items[it].scales + (kNv ? off : off / 2);
            t.global_scale[k] = items[it].global_scale;
            t.y[k] = static_cast<TOut *>(items[it].y) + off * 16;
            t.tile_first[k + 1] = t.tile_first[k] + fp4::grouped_tile_count(take, fp4::kDequantUnits);
        },
        [&](const fp4::DqGroup &t) {
            const int grid = grid_for(fp4::dequantize_grouped_kernel<kNv, TOut>, t.tile_first[t.n], 1,
                                      kThreads, 0, fp4::kDequantCtasPerSm);
            if (grid <= 0)
                return FP4_ERR_CUDA;
            return launch(fp4::dequantize_grouped_kernel<kNv, TOut>, grid, stream, t);
        });
}

template <bool kCeil>
fp4_status mx_quantize_grouped_rule(const fp4_quant_item *items, int n_items, fp4_dtype dtype,
                                    int32_t *status, cudaStream_t stream)
{
    const fp4_status st = check_quant_items(items, n_items, dtype, status, 32, kMx);
    if (st != FP4_OK)
        return st;
    if (dtype == FP4_BF16)
        return mx_grouped<uint16_t, kCeil>(items, n_items, status, stream);
    return mx_grouped<float, kCeil>(items, n_items, status, stream);
}

} // namespace

extern "C" {

size_t fp4_grouped_workspace_bytes(int n_items)
{
    if (n_items < 0)
        return 0;
    return ((size_t)n_items * sizeof(uint32_t) + 255) / 256 * 256;
}

fp4_status fp4_tensor_amax_grouped(const fp4_quant_item *items, int n_items, fp4_dtype dtype,
                                   void *workspace, size_t workspace_bytes, int32_t *status,
                                   cudaStream_t stream)
{
    fp4_status st = check_quant_items(items, n_items, dtype, status, 16, kInputOnly);
    if (st != FP4_OK || n_items == 0)
        return st;
    if ((st = check_workspace(workspace, workspace_bytes, n_items)) != FP4_OK)
        return st;
    uint32_t *words = static_cast<uint32_t *>(workspace);
    if (dtype == FP4_BF16)
        return amax_grouped<uint16_t>(items, n_items, words, status, stream);
    return amax_grouped<float>(items, n_items, words, status, stream);
}

fp4_status fp4_nvfp4_quantize_grouped_with_amax(const fp4_quant_item *items, int n_items,
                                                fp4_dtype dtype, const void *amax_words,
                                                int32_t *status, cudaStream_t stream)
{
    fp4_status st = check_quant_items(items, n_items, dtype, status, 16, kNv);
    if (st != FP4_OK || n_items == 0)
        return st;
    if (!amax_words || (reinterpret_cast<uintptr_t>(amax_words) & 3))
        return FP4_ERR_INVALID_ARG;
    const uint32_t *words = static_cast<const uint32_t *>(amax_words);
    if (dtype == FP4_BF16)
        return nv_grouped_with_amax<uint16_t>(items, n_items, words, status, stream);
    return nv_grouped_with_amax<float>(items, n_items, words, status, stream);
}

fp4_status fp4_nvfp4_quantize_grouped(const fp4_quant_item *items, int n_items, fp4_dtype dtype,
                                      void *workspace, size_t workspace_bytes, int32_t *status,
                                      cudaStream_t stream)
{
    fp4_status st = check_quant_items(items, n_items, dtype, status, 16, kNv);
    if (st != FP4_OK || n_items == 0)
        return st;
    if ((st = check_workspace(workspace, workspace_bytes, n_items)) != FP4_OK)
        return st;
    st = fp4_tensor_amax_grouped(items, n_items, dtype, workspace, workspace_bytes, status, stream);
    if (st != FP4_OK)
        return st;
    return fp4_nvfp4_quantize_grouped_with_amax(items, n_items, dtype, workspace, status, stream);
}

fp4_status fp4_mxfp4_quantize_grouped(const fp4_quant_item *items, int n_items, fp4_dtype dtype,
                                      int32_t *status, cudaStream_t stream)
{
    return mx_quantize_grouped_rule<false>(items, n_items, dtype, status, stream);
}

fp4_status fp4_mxfp4_quantize_ceil_grouped(const fp4_quant_item *items, int n_items,
                                           fp4_dtype dtype, int32_t *status, cudaStream_t stream)
{
    return mx_quantize_grouped_rule<true>(items, n_items, dtype, status, stream);
}

fp4_status fp4_dequantize_grouped(fp4_format fmt, const fp4_dequant_item *items, int n_items,
                                  fp4_dtype out_dtype, cudaStream_t stream)
{
    if ((fmt != FP4_NVFP4 && fmt != FP4_MXFP4) || !valid_dtype(out_dtype) || n_items < 0 ||
        (n_items > 0 && !items))
        return FP4_ERR_INVALID_ARG;
    const bool nv = fmt == FP4_NVFP4;
    for (int i = 0; i < n_items; ++i) {
        const fp4_dequant_item &d = items[i];
        if (d.rows < 0 || d.cols < 0)
            return FP4_ERR_INVALID_ARG;
        if (d.cols % (nv ? 16 : 32) || (d.cols > 0 && d.rows > INT64_MAX / d.cols / 4))
            return FP4_ERR_SHAPE;
        if (d.rows * d.cols > 0 && (!d.packed || !d.scales || !d.y || (nv && !d.global_scale)))
            return FP4_ERR_INVALID_ARG;
        if (!aligned(d.packed, 16) || !aligned(d.y, 32) || (nv && !aligned(d.global_scale, 4)))
            return FP4_ERR_ALIGN;
    }
    if (nv && out_dtype == FP4_BF16)
        return dq_grouped<true, uint16_t>(items, n_items, stream);
    if (nv)
        return dq_grouped<true, float>(items, n_items, stream);
    if (out_dtype == FP4_BF16)
        return dq_grouped<false, uint16_t>(items, n_items, stream);
    return dq_grouped<false, float>(items, n_items, stream);
}

int fp4_grouped_plan(const int64_t *units, int n_items, int64_t max_units, int max_entries,
                     int32_t *launch_of, int32_t *item_of, int64_t *first_of, int64_t *count_of,
                     int max_pieces)
{
    if (n_items < 0 || (n_items > 0 && !units) || max_units < 64 ||
        max_units > fp4::kMaxUnitsPerLaunch || max_entries < 1 || max_entries > kGroupMax ||
        max_pieces < 0)
        return -1;
    struct Table {
        int n;
        int first[kGroupMax + 1];
    };
    int pieces = 0, launches = 0;
    const fp4_status st = plan<Table>(
        n_items, [&](int it) { return units[it]; },
        [&](Table &, int, int it, int64_t off, int64_t take) {
            if (pieces < max_pieces) {
                launch_of[pieces] = launches;
                item_of[pieces] = it;
                first_of[pieces] = off;
                count_of[pieces] = take;
            }
            ++pieces;
        },
        [&](const Table &) {
            ++launches;
            return FP4_OK;
        },
        max_units, max_entries);
    return st == FP4_OK ? pieces : -1;
}

} // extern "C"
