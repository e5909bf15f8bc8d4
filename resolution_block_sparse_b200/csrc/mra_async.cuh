// mra_async.cuh - mbarrier helpers (PTX) shared by the kernels whose copies
// or tensor-core work complete on mbarriers (the tcgen05 attention and the
// layer's projection GEMM).
//
// Every wait is bounded: a waiting thread sleeps up to kSuspendHintNs per
// try_wait and gives up after kWaitLimit tries (a few seconds), so a copy that
// never lands ends in an error status instead of a hung GPU.
#pragma once

#include <cstdint>

namespace mra {
namespace async {

constexpr unsigned kSuspendHintNs = 20000;   // per try_wait
constexpr unsigned kWaitLimit = 1u << 17;    // x hint: a few seconds at most

__device__ __forceinline__ uint32_t saddr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
// makes initialised barriers visible to the copy engine and the other threads
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// try_wait with a suspend-time hint: a waiting thread sleeps (up to the hint)
// until the phase completes instead of spinning on issue slots
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}
// Bounded wait on one phase of an mbarrier; false when the limit expired.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (unsigned i = 0; i < kWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

}  // namespace async
}  // namespace mra
