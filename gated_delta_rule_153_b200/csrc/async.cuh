// async.cuh -- mbarrier and bulk-copy (TMA engine) helpers for sm_100a.
//
// Loads are 1-D bulk copies (cp.async.bulk) of contiguous global ranges into
// shared memory, completing on an mbarrier with a transaction byte count;
// stores are bulk copies from shared memory back to global memory.  Every
// copy targets only the issuing CTA's own shared memory.
//
// Every wait is bounded: a waiter that has not seen its phase complete after
// kWaitNs nanoseconds sets bit 0 of the caller's device status word (read by
// gdn_query_device_status) and reports failure, so the kernel can return
// instead of spinning forever.
#pragma once

#include <stdint.h>

#include "mma.cuh"

namespace gdn {

constexpr unsigned long long kWaitNs = 1000000000ull;  // 1 s

GDN_DEV uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

GDN_DEV void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

GDN_DEV void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive once and add `bytes` to the barrier's expected transaction count.
GDN_DEV void mbar_arrive_expect(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Plain arrival (no transaction bytes).
GDN_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

GDN_DEV bool mbar_try(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of `bar`.  Returns false (and flags the
// status word) if it did not complete within `limit_ns` (default kWaitNs).
// A wait that guards a copy or an MMA still in flight when the CTA is about
// to exit (the drains before teardown) always uses the default limit.
GDN_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned int* status,
                       unsigned long long limit_ns = kWaitNs) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) {
            if (status) atomicOr(status, 1u);
            return false;
        }
    }
}

// Bulk copy `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global memory into shared memory, completing on `bar`.
GDN_DEV void bulk_g2s(void* smem, const void* gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem)), "l"(gmem), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Hint: pull `bytes` (multiple of 16) of global memory into L2 ahead of use.
GDN_DEV void bulk_prefetch_l2(const void* gmem, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gmem), "r"(bytes) : "memory");
}

// Hint: pull the cache line holding `gmem` into L2.
GDN_DEV void prefetch_l2(const void* gmem) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(gmem) : "memory");
}

// Bulk copy from shared memory to global memory (bulk-group completion).
GDN_DEV void bulk_s2g(void* gmem, const void* smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(gmem), "r"(smem_u32(smem)), "r"(bytes) : "memory");
}
GDN_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N bulk groups of this thread are still reading shared memory.
template <int N>
GDN_DEV void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
template <int N>
GDN_DEV void bulk_wait() { asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (bulk copies) -- required before a bulk store reads them.
GDN_DEV void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

}  // namespace gdn
