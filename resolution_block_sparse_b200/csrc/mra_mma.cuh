// mra_mma.cuh - warp-level tensor-core helpers (mma.sync m16n8k16 bf16 with
// fp32 accumulation, ldmatrix, cp.async) and the XOR-swizzled layout of a
// [32][D] bf16 tile in shared memory, shared by the forward attention kernel
// and the backward kernel.
#pragma once

#include <cuda_bf16.h>

namespace mra {
namespace mma {

__device__ __forceinline__ unsigned smem_u32(const void *p) {
    return (unsigned)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void ldsm_x4(unsigned &r0, unsigned &r1, unsigned &r2, unsigned &r3,
                                        unsigned addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(unsigned &r0, unsigned &r1, unsigned &r2, unsigned &r3,
                                          unsigned addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float *c, const unsigned *a, unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 2^x on the special-function unit (ex2.approx.ftz, about 2 ulp)
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ unsigned pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<unsigned *>(&v);
}

// Element offset of (row, 8-element chunk j) in a swizzled [32][D] bf16 tile:
// chunk j of a row is stored at position j ^ f(row), which keeps the eight
// rows read by one ldmatrix phase in distinct 16-byte bank groups.
template <int D>
__device__ __forceinline__ int swz(int row, int j) {
    if constexpr (D == 64) return row * D + ((j ^ (row & 7)) << 3);
    else return row * D + ((j ^ ((row >> 1) & 3)) << 3);
}

template <int D, int NT>
__device__ __forceinline__ void load_tile_async(__nv_bfloat16 *tile, const __nv_bfloat16 *g, int tid) {
    constexpr int kCpr = D / 8;
    constexpr int kChunks = 32 * kCpr;
#pragma unroll
    for (int e = tid; e < kChunks; e += NT) {
        const int row = e / kCpr, j = e % kCpr;
        cp_async16(tile + swz<D>(row, j), g + (size_t)row * D + j * 8);
    }
}

}  // namespace mma
}  // namespace mra
