// focus_pipeline.cuh -- shared-memory staging primitives for sm_100a.
//
// A CTA streams its tiles through a ring of shared-memory stages: one
// producer thread issues 1-D bulk asynchronous copies (cp.async.bulk, global
// to shared, completion counted in bytes on an mbarrier) and consumer warps
// compute from the staged data, releasing each stage through a second
// mbarrier.  Where the consumers leave their outputs in the stage, the
// producer writes them out with bulk copies the other way (shared to global,
// completion tracked by bulk groups) before it fills the stage again.  No copy
// uses cluster multicast: every copy reads or writes this GPU's own global
// memory and the issuing CTA's shared memory.
//
// Every wait is bounded: after WAIT_LIMIT_NS of wall time (read from
// %globaltimer), or a hard iteration cap, it gives up and returns false; the
// caller then records an error and leaves its loop, so a kernel never waits
// forever.  Between its tests a waiting thread is suspended by the hardware
// (the try_wait suspend-time hint) rather than polling.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace focus {

constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s
constexpr uint32_t WAIT_MAX_ITERS = 1u << 26;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes the initialised barriers visible to the asynchronous (bulk copy) proxy.
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar) : "memory");
}

// Arrive and add `bytes` to the transaction count the phase waits for.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// The same test, but a thread whose phase is not yet complete is suspended by
// the hardware until it completes or about HINT_NS nanoseconds have passed:
// a waiting warp then takes no issue slots from the warps that compute.
template <uint32_t HINT_NS>
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "n"(HINT_NS)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits until the phase of parity `parity` of the barrier has completed,
// suspended (not polling) between tests.  Returns false if that does not
// happen within `limit_ns` of wall time (or WAIT_MAX_ITERS tests).
constexpr uint32_t WAIT_SLEEP_NS = 1000;

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns = WAIT_LIMIT_NS) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1; i < WAIT_MAX_ITERS; ++i) {
        if (mbar_try_wait_sleep<WAIT_SLEEP_NS>(bar, parity)) return true;
        if ((i & 15u) == 0 && global_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// global memory into this CTA's shared memory; completion is counted on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// this CTA's shared memory to global memory, in the thread's current bulk
// group.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until every bulk group of this thread has finished reading its shared
// memory source (the stage may then be written again).
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Waits until every bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Makes this thread's writes to shared memory visible to later bulk copies
// (the asynchronous proxy) that read it.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace focus
