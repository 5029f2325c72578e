// q8_ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, 1-D bulk
// (TMA) copies global -> shared without multicast, programmatic dependent
// launch control, named barriers and bounded waits.
//
// Every wait here is bounded: after about two seconds it records
// Q8_WAIT_TIMEOUT in the calling translation unit's device error word and
// returns false instead of spinning forever; callers carry on (the results
// are then wrong, and q8_check reports it) so that no barrier is left
// waiting for a warp that gave up.
#pragma once

#include <stdint.h>

// Trace points of the kernels (numbered phases of a CTA's timeline).  They
// compile to nothing unless the build defines Q8_TRACE(id) to a recorder
// before this header is included.
#ifndef Q8_TRACE
#define Q8_TRACE(id) ((void)0)
#endif

namespace q8 {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Make initialized barriers visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

constexpr int Q8_WAIT_TIMEOUT = 1;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Wait for the phase with the given parity to complete; false after
// limit_ns (the error word then holds Q8_WAIT_TIMEOUT).
__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, uint32_t parity, int *err_word,
                                              uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 256; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(err_word, Q8_WAIT_TIMEOUT);
            return false;
        }
    }
}

// Wait for the phase with the given parity to complete; false after ~2 s.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *err_word) {
    return mbar_wait_for(bar, parity, err_word, kWaitLimitNs);
}

// 1-D bulk copy global -> this CTA's shared memory, completing `bytes` of
// transaction count on `bar`.  dst, src 16-byte aligned, bytes % 16 == 0.
// The weights are read once per call: L2 evict-first.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b64 pol;\n\t"
        "createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n\t"
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], pol;\n\t}" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// The same without an L2 eviction hint, for data that other CTAs read too.
__device__ __forceinline__ void bulk_g2s_keep(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Per-thread asynchronous copies global -> shared (the non-bulk form): the
// thread continues at once; cp_async_commit closes a group of its copies and
// cp_async_wait<N> returns when at most N of its groups are still in flight.
// 16-byte copies: both addresses 16-byte aligned, L2 only; 4-byte copies:
// both addresses 4-byte aligned.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)),
                 "l"(__cvta_generic_to_global(src))
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)),
                 "l"(__cvta_generic_to_global(src))
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch: wait until the grids this one depends on
// have completed and their memory is visible; allow dependents to launch.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Barrier among `nthreads` threads (whole warps) on hardware barrier `id`.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace q8
