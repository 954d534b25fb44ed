// mbarrier_sm100.cuh -- shared-memory mbarrier helpers with BOUNDED waits
// (every wait gives up after a time limit, or at once when another thread
// of the CTA has given up, so no kernel here can spin forever).
#pragma once

#include <stdint.h>

namespace gdn {
namespace sync {

// Time limit of every bounded wait: 0.5 s.  The timeout tests build a copy
// of the library (tests/timeout_probe/) with a limit of a few milliseconds.
#ifndef GDN_WAIT_LIMIT_NS
#define GDN_WAIT_LIMIT_NS (500ull * 1000ull * 1000ull)
#endif
constexpr uint64_t WAIT_LIMIT_NS = GDN_WAIT_LIMIT_NS;

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(unsigned long long *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// The expect-tx arrival paired with a kernel's first bulk copy of a
// sequence's data -- its state, or the first piece's record for a kernel that
// loads the state with plain loads (the barrier phase completes when this
// arrival and the copy's bytes are both in).  The test copy of the library (tests/timeout_probe/) is compiled with
// GDN_TEST_WITHHOLD_STATE_ARRIVAL, which drops the arrival: the copy still
// lands, its phase never completes, and the kernel's bounded wait for it runs
// out -- how the timeout paths are made to fire on a GPU without a fault.
// Product builds never define it.
__device__ __forceinline__ void mbar_arrive_expect_state_tx(unsigned long long *bar, uint32_t bytes)
{
#ifdef GDN_TEST_WITHHOLD_STATE_ARRIVAL
    (void)bar;
    (void)bytes;
#else
    mbar_arrive_expect_tx(bar, bytes);
#endif
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase.  Gives up (returns false) after
// WAIT_LIMIT_NS, or at once when another thread of the CTA has given up.
__device__ __forceinline__ bool mbar_wait(unsigned long long *bar, uint32_t parity, volatile int *failed)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((n & 63u) == 0u && (*failed || global_ns() - t0 > WAIT_LIMIT_NS))
            return false;
    }
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Plain (untiled, non-multicast) bulk copies between global and this CTA's
// shared memory.  Addresses 16-byte aligned, sizes multiples of 16 bytes.
// A load completes `bytes` transactions on the mbarrier `bar`.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                          unsigned long long *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(smem_dst)),
                 "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void bulk_store(void *gmem_dst, const void *smem_src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
                 "r"(smem_addr(smem_src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// generic-proxy shared-memory writes -> visible to the async proxy (bulk copies)
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Per-thread 16-byte asynchronous copy global -> shared.  Both addresses 16-byte
// aligned; `src_bytes` (0 or 16) bytes are read and the rest of the 16 zero-filled.
// Complete with cp_async_wait_all() in the issuing thread (before the CTA exits).
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(smem_dst)), "l"(gmem_src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Hint: bring `bytes` of global memory (16-byte aligned, a multiple of 16) into L2.
__device__ __forceinline__ void prefetch_l2(const void *gmem_src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gmem_src), "r"(bytes) : "memory");
}

}  // namespace sync
}  // namespace gdn
