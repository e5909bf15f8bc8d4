// mra_async.cuh - mbarrier helpers (PTX) shared by the kernels whose copies
// or tensor-core work complete on mbarriers (the tcgen05 attention and the
// layer's projection GEMM).
//
// Every wait is bounded: a waiting thread polls the barrier with try_wait
// without a suspend-time hint (polling measured faster than suspending with a
// 20 us hint: the tcgen05 attention on the N=16384 map 286 -> 255 us) and
// gives up once kWaitNs of %globaltimer time have passed, so a copy that never
// lands ends in an error status instead of a hung GPU.
#pragma once

#include <cstdint>

namespace mra {
namespace async {

constexpr unsigned long long kWaitNs = 2000000000ull;   // 2 s per wait at most
constexpr unsigned kWaitLimit = 1u << 30;                // polls, a second bound that needs no timer

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
// One poll of a phase: try_wait blocks for at most a short, system-dependent
// time and reports whether the phase with this parity has completed.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Polls until the phase completes (true) or kWaitNs have passed (false).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (unsigned i = 0; i < kWaitLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u && global_ns() - t0 > kWaitNs) return false;
    }
    return false;
}

}  // namespace async
}  // namespace mra
