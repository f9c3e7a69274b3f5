// kq_ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, bulk and
// tensor (TMA) copies, programmatic dependent launch, packed fp32 math.
// Every wait on an mbarrier is bounded: after `KQ_SPIN_LIMIT` polls (each
// suspending at most ~1 us, so a few seconds at most) it gives up, sets the
// device error word and reports failure to the caller.
#pragma once

#include "kq_common.cuh"

#ifndef KQ_SPIN_LIMIT
#define KQ_SPIN_LIMIT (1u << 22)
#endif

namespace kq {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// One poll; the thread may be suspended up to ~1 us inside it (time hint),
// so a waiting warp does not spin through issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(1000u)
        : "memory");
    return ok != 0;
}

// Non-blocking poll of a phase.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait; returns false (and flags the device error word) on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned int *err) {
    for (uint32_t i = 0; i < KQ_SPIN_LIMIT; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    atomicOr(err, ERR_TIMEOUT);
    return false;
}

// Bounded wait that polls without suspending: a non-blocking test, then a
// short sleep.  For phases completed by other threads' arrivals, where a
// suspended try_wait can stay asleep up to its whole time hint after the
// phase completes.  Gives up after about as long as mbar_wait.
__device__ __forceinline__ bool mbar_wait_poll(uint64_t *bar, uint32_t parity, unsigned int *err) {
    for (uint32_t i = 0; i < (KQ_SPIN_LIMIT << 4); ++i) {
        if (mbar_test_wait(bar, parity)) return true;
        __nanosleep(32);
    }
    atomicOr(err, ERR_TIMEOUT);
    return false;
}

// Contiguous global -> shared bulk copy; completion counted on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Prefetch a contiguous global range into L2 (bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Programmatic dependent launch (no-ops when the launch did not enable it).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Packed fp32 pair fused multiply-add (sm_100): (a.x*b.x + c.x, a.y*b.y + c.y),
// each lane rounded once like fmaf.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long A, B, C;
    asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(B) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(C) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(C) : "l"(A), "l"(B));
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(C));
    return r;
}

}  // namespace kq
