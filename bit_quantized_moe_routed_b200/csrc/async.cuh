// async.cuh -- mbarrier, bulk-copy (TMA) and bounded-wait helpers for sm_100a.
#pragma once

#include <stdint.h>

#include "internal.cuh"

namespace moeq {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// cnt arrivals at once
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t *bar, uint32_t cnt) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(cnt) : "memory");
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

// Non-blocking probe of phase `parity` of `bar` (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, giving up after about
// `max_cycles` SM clocks (about a second at the default).  Returns false on
// timeout; the caller reports MOEQ_ERR_TIMEOUT and unwinds.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  long long max_cycles = 2000000000LL) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > max_cycles) return false;
    }
    return true;
}

// Wait for phase `parity` of `bar` unless another role of the CTA has given
// up (*abort != 0), for at most `max_cycles` SM clocks; on expiry this
// thread raises *abort itself.  Returns false when it did not see the phase
// complete.  The first probe is the fast path; the loop re-reads the flag
// between suspended probes.
__device__ __forceinline__ bool mbar_wait_abort(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                long long max_cycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > max_cycles) {
            *abort = 1;
            return false;
        }
    }
    return true;
}

// mbar_wait_abort with non-suspending probes (test_wait): for a wait that
// the whole CTA makes once, where a suspended thread would only add
// latency; with a short limit it gives up as soon as the phase is not
// complete.
__device__ __forceinline__ bool mbar_poll_abort(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                long long max_cycles) {
    if (mbar_test_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_test_wait(bar, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > max_cycles) {
            *abort = 1;
            return false;
        }
    }
    return true;
}

// The limit of the drains that run before a CTA exits (its own copies in
// flight, its own tensor-core operations): fixed and long, so that no
// asynchronous operation outlives the CTA whatever limit the other waits
// were given (about 0.1 s).
constexpr long long kDrainCycles = 200000000LL;

// Global -> shared bulk copy (no tensor map).  dst and src 16-byte aligned,
// bytes a multiple of 16; completion is signalled on `bar` as tx bytes.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// An L2 policy that evicts first: for data read exactly once per call (the
// decode weights), so that it does not push the small, reused data (kernel
// code, routing, activations) out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// bulk_g2s with an L2 cache policy for the source.
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint4 lds128(const void *p) {
    return *reinterpret_cast<const uint4 *>(p);
}
__device__ __forceinline__ uint32_t lds32(const void *p) { return *reinterpret_cast<const uint32_t *>(p); }

// Programmatic dependent launch controls (no-ops when the launch does not use PDL).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace moeq
