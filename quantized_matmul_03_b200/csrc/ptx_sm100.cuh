// ptx_sm100.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, bulk and
// tensor (TMA) copies, bounded waits.  No cluster multicast anywhere.
#pragma once

#include <stdint.h>

#include "qmm_internal.cuh"

namespace qmm {
namespace ptx {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// Make mbarrier initialisation visible to the async proxy (TMA / bulk copies).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// Test the phase once, without blocking.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Test the phase; if it is not complete, the thread may be suspended for up
// to ~1 ms (or until the phase completes, whichever is first) instead of
// spinning, so waiting warps leave the issue slots to working ones.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}

// Wait for the phase of parity `parity` to complete, for at most the
// library's wait limit (2 s unless qmm_set_wait_limit_ns changed it).  On
// timeout the device error word gets QMM_ERR_TIMEOUT and false is returned;
// callers then carry on without the data (their shared-memory accesses stay
// in bounds), so every thread still reaches the kernel's end.  SLEEP selects
// suspending waits (long, off the critical path) or spinning ones (short
// hand-offs where a wake-up delay would cost throughput).
template <bool SLEEP = true>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int *err) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = wait_limit_ns(err);
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (SLEEP ? mbar_try_wait(bar, parity) : mbar_test(bar, parity)) return true;
        const uint64_t dt = globaltimer_ns() - t0;
        if (dt > limit) {
            record_device_error(err, QMM_ERR_TIMEOUT);
            return false;
        }
        // After 1 ms, give up at once if another wait already timed out (the
        // error word is global memory: never read it on the fast path).
        if (dt > 1000000ull && *reinterpret_cast<volatile int *>(err) != 0) return false;
    }
}

// Wait for this CTA's own asynchronous operations (copies into its shared
// memory, its tensor-core work) before it exits or frees tensor memory.  The
// limit is the fixed default, never the settable one: a CTA must not leave
// while its copies can still land.
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity, int *err) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kDefaultWaitNs) {
            record_device_error(err, QMM_ERR_TIMEOUT);
            return false;
        }
    }
}

// ---- programmatic dependent launch -----------------------------------------
// Block until every grid this one depends on (the preceding work in the
// stream) has completed and its memory is visible.  No-op without PDL.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next kernel in the stream (launched with programmatic stream
// serialization) to start its prologue while this grid is still running.
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- bulk copies (global -> shared, completion on an mbarrier) -------------
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Per 16-bit half, the unsigned maximum of a and b (sm_90 and later).
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Two fp32 values in one 64-bit register (x in the low half), and the packed
// two-lane fp32 operations of sm_100 (each lane one IEEE operation, round to
// nearest even).
__device__ __forceinline__ unsigned long long f2pack(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ unsigned long long u2pack(uint32_t a, uint32_t b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ void f2unpack(unsigned long long v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2sub(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long f2add(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long f2mul(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

}  // namespace ptx
}  // namespace qmm
