// fp4_async.cuh -- shared-memory barriers (mbarrier) and bulk copies into
// shared memory, for the kernels that stage their operands with the copy
// engine (the tensor-core GEMMs).  Every wait is bounded (kWaitTries polls);
// a kernel whose wait runs out records FP4_ERR_TIMEOUT (kStatusTimeout),
// waits (bounded) for the copies it has issued, and returns.
#pragma once

#include <cstdint>

namespace fp4 {

constexpr int32_t kStatusTimeout = 8;
// Polls of a bounded wait.  A poll (mbarrier.try_wait) that finds the phase
// incomplete suspends the thread for about 4 us on B200 (measured with the
// bounded-wait test entry point), so a wait gives up after about a second.
constexpr uint32_t kWaitTries = 1u << 18;

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// Bounded wait for phase `parity` of the barrier; false when the tries run out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t tries = kWaitTries)
{
    for (uint32_t t = 0; t < tries; ++t) {
        uint32_t done;
        asm volatile("{\n\t"
                     ".reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t"
                     "}"
                     : "=r"(done)
                     : "r"(smem_addr(bar)), "r"(parity)
                     : "memory");
        if (done)
            return true;
    }
    return false;
}

// Makes the barriers' initialisation visible to the copy engine.
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Untiled bulk copy of `bytes` (a multiple of 16; both addresses 16-byte
// aligned) from global into shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// Test of the bounded wait: one warp waits on a barrier that nothing
// arrives on (`tries` polls), records FP4_ERR_TIMEOUT when the wait runs out
// as the kernels that copy do, and reports the wait's duration (globaltimer
// nanoseconds) in *elapsed_ns.
static __global__ void bounded_wait_test_kernel(uint32_t tries, int32_t *status, long long *elapsed_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_init_fence();
    }
    __syncwarp();
    long long t0, t1;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bar, 0, tries));
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
    if (threadIdx.x == 0) {
        if (!ok)
            atomicCAS(status, 0, kStatusTimeout);
        *elapsed_ns = t1 - t0;
    }
}

} // namespace fp4
