// ssq_pipe.cuh -- PTX wrappers for the asynchronous copy pipelines of the
// libssq kernels: mbarriers (init, arrive, expect-tx, bounded waits), bulk
// copies between global and shared memory (cp.async.bulk) and cp.async.
//
// Every wait is bounded: a wait that sees no progress for about a second
// returns false and the caller records SSQ_DEVERR_TIMEOUT and winds down.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssq {

constexpr long long kWaitLimit = 2000000000LL;  // clock cycles, about one second

// ---- PTX wrappers -------------------------------------------------------
__device__ __forceinline__ unsigned saddr(const void* p)
{
    return (unsigned)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* b, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
// Arrive from the lanes where `pred` holds (predicated inside the
// instruction, so the warp does not branch).
__device__ __forceinline__ void mbar_arrive_if(uint64_t* b, bool pred)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %1, 0;\n"
                 " @p mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n}\n"
                 ::"r"(saddr(b)), "r"((unsigned)pred) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(saddr(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, unsigned parity)
{
    unsigned ok;
    asm volatile("{\n .reg .pred p;\n"
                 " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
                 " selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok) : "r"(saddr(b)), "r"(parity) : "memory");
    return ok != 0;
}
// Wait for the phase of the given parity to complete, sleeping between
// tries (exponential back-off up to kMaxSleepNs, so a waiting warp takes
// few issue slots from the warps that compute); false after `limit` clock
// cycles without progress (about a second by default).
template <unsigned kMaxSleepNs>
__device__ __forceinline__ bool mbar_wait(uint64_t* b, unsigned parity,
                                          long long limit = kWaitLimit)
{
    if (mbar_try(b, parity)) return true;
    const long long t0 = clock64();
    unsigned ns = 64;
    while (!mbar_try(b, parity)) {
        __nanosleep(ns);
        ns = ns < kMaxSleepNs ? 2 * ns : kMaxSleepNs;
        if (clock64() - t0 > limit) return false;
    }
    return true;
}
constexpr unsigned kProducerSleep = 2048;  // the producer waits for a stage to drain
constexpr unsigned kConsumerSleep = 256;   // consumers wait for data to land

// One test of the phase in which the thread may be suspended by the
// hardware until the phase completes or about `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_suspend(uint64_t* b, unsigned parity, unsigned hint_ns)
{
    unsigned ok;
    asm volatile("{\n .reg .pred p;\n"
                 " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
                 " selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok) : "r"(saddr(b)), "r"(parity), "r"(hint_ns) : "memory");
    return ok != 0;
}
// Wait for the phase of the given parity to complete with the thread
// suspended in the barrier instead of polling (a waiting warp issues a few
// instructions per suspension, not one loop per few cycles); false after
// `limit` clock cycles without progress.
__device__ __forceinline__ bool mbar_wait_suspend(uint64_t* b, unsigned parity,
                                                  long long limit = kWaitLimit)
{
    if (mbar_try_suspend(b, parity, 20000u)) return true;
    const long long t0 = clock64();
    while (!mbar_try_suspend(b, parity, 20000u)) {
        if (clock64() - t0 > limit) return false;
    }
    return true;
}
// Bulk prefetch of global memory into L2 (no completion to wait for).
// Address 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, unsigned bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// Bulk copy global -> shared; completion counted in bytes on `bar`.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(saddr(dst)), "l"(src), "r"(bytes), "r"(saddr(bar)) : "memory");
}
__device__ __forceinline__ void cpa4(void* dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(saddr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa16(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr(dst)), "l"(src) : "memory");
}
// The mbarrier's current phase also waits for this thread's earlier cp.async.
__device__ __forceinline__ void cpa_arrive(uint64_t* b)
{
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(saddr(b)) : "memory");
}

// Bulk copy shared -> global (completion tracked per thread in bulk groups).
// Both addresses 16-byte aligned, size a multiple of 16.  The shared data
// must be made visible to the async proxy first (fence_proxy_async).
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, unsigned bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst), "r"(saddr(src)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's bulk groups still read their source.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N of this thread's bulk groups are still in flight.
template <int N>
__device__ __forceinline__ void bulk_wait()
{
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Order this thread's generic-proxy shared-memory writes before later
// async-proxy accesses (a bulk store reading them).
__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace ssq
