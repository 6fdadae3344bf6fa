// Shared device helpers for the sm_100a kernels: the per-device error word,
// bounded mbarrier waits, bulk-copy and programmatic-dependent-launch PTX.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "mrgemm.h"

#ifndef MR_WAIT_TEST_FIRST
#define MR_WAIT_TEST_FIRST 1
#endif

namespace mr {

// Per-device error word: bits MR_DEVERR_*, set by a kernel whose bounded wait
// ran out; read and cleared by mr_poll_errors.  The library is one translation
// unit (mrgemm_lib.cu includes every kernel file), so this is its only copy.
__device__ uint32_t g_error_word = 0;

// Default bound on any single wait inside a kernel (nanoseconds of
// %globaltimer).  Every legitimate wait ends in microseconds.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_error(uint32_t bits) {
    atomicOr(&g_error_word, bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier -----------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make initialised barriers visible to the async proxy (bulk copies, TMA).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of phase `parity` (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of the barrier to complete, for at most limit_ns.
// Returns false (after recording `err_bits`) when the limit runs out.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint32_t err_bits,
                                                  uint64_t limit_ns = kWaitLimitNs) {
#if MR_WAIT_TEST_FIRST
    if (mbar_test_wait(bar, parity)) return true;
#endif
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_error(err_bits);
            return false;
        }
    }
}

// ---- bulk copies (non-tensor, into the issuing CTA only) ------------------

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned) whose completion is counted on `bar` as tx bytes.
__device__ __forceinline__ void bulk_g2s(uint32_t dst_smem, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst_smem), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ---- programmatic dependent launch ----------------------------------------

// Block until the kernels this grid depends on have completed and their
// memory is visible (a no-op when the launch had no programmatic dependency).
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Allow the next kernel in the stream to begin launching.
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace mr

// Host-side helpers shared by the entry points (defined in api.cu).
namespace mr_host {
mr_status cuda_status(cudaError_t e);
int sm_count();             // SMs of the current device (cached per device)
int max_smem_optin();       // opt-in shared memory per block (bytes)
}  // namespace mr_host
