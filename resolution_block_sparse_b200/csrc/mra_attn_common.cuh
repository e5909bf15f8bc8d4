// mra_attn_common.cuh - epilogue shared by the attention kernels: merge of
// (max, sum, output) partials of one block row with the low-resolution part
// (page "深入解析 Transformers 中的 MRA 模型", section "源码级原理", step four:
// both parts brought to a shared maximum, normalisers added) and the output
// write.  Sync is the barrier of the participating threads (whole CTA, or a
// named barrier when a producer warp sits outside the epilogue).
#pragma once

#include <cuda_bf16.h>

#include "mra_internal.cuh"

namespace mra {
namespace attn {

constexpr float kLog2e = 1.4426950408889634f;

struct SyncAll {
    __device__ __forceinline__ static void sync() { __syncthreads(); }
};
struct SyncNamed128 {   // barrier 1 over threads 0..127
    __device__ __forceinline__ static void sync() { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }
};

template <bool G>
__device__ __forceinline__ float ldp(const float *p) {
    if constexpr (G) return __ldcg(p);
    else return *p;
}

template <typename T>
__device__ __forceinline__ T to_out(float x);
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <>
__device__ __forceinline__ float to_out<float>(float x) { return x; }

struct MergeSmem {
    float w[32][33];
    float M[32], inv[32], beta[32];
};

// Merge nchunks partials (layout per slot: m[32], l[32], O[32][D]; m in log2
// units, l and O relative to exp2(m)) with the low-resolution part of the row
// (full mode) and write the 32 x D output block.
template <int D, int NT, bool G, typename OutT, typename Sync>
__device__ void merge_write(const float *src0, size_t slot_stride, int nchunks, int full,
                            float m_lo2, float l_lo, const float *olo_row, const float *qmask,
                            OutT *out_blk, MergeSmem &sm) {
    const int tid = threadIdx.x;
    if (tid < 32) {
        const int q = tid;
        float M = -INFINITY;
        for (int c = 0; c < nchunks; ++c) {
            const float *P = src0 + (size_t)c * slot_stride;
            if (ldp<G>(P + 32 + q) > 0.0f) M = fmaxf(M, ldp<G>(P + q));
        }
        const bool lo = full && l_lo > 0.0f;
        if (lo) M = fmaxf(M, m_lo2);
        float inv = 0.0f, beta = 0.0f;
        if (M != -INFINITY && (!qmask || qmask[q] > 0.0f)) {
            float den = 0.0f;
            for (int c = 0; c < nchunks; ++c) {
                const float *P = src0 + (size_t)c * slot_stride;
                const float l = ldp<G>(P + 32 + q);
                if (l > 0.0f) den += exp2f(ldp<G>(P + q) - M) * l;
            }
            if (lo) {
                beta = exp2f(m_lo2 - M);
                den += beta * l_lo;
            }
            inv = den > 0.0f ? 1.0f / den : 0.0f;
        }
        sm.M[q] = (M == -INFINITY) ? 0.0f : M;
        sm.inv[q] = inv;
        sm.beta[q] = beta;
    }
    Sync::sync();
    constexpr int E = 32 * D / NT;
    float acc[E];
#pragma unroll
    for (int i = 0; i < E; ++i) acc[i] = 0.0f;
    for (int cg = 0; cg < nchunks; cg += 32) {
        const int nc = min(32, nchunks - cg);
        for (int e = tid; e < nc * 32; e += NT) {
            const int c = e / 32, q = e % 32;
            const float *P = src0 + (size_t)(cg + c) * slot_stride;
            sm.w[c][q] = ldp<G>(P + 32 + q) > 0.0f ? exp2f(ldp<G>(P + q) - sm.M[q]) : 0.0f;
        }
        Sync::sync();
        for (int c = 0; c < nc; ++c) {
            const float *O = src0 + (size_t)(cg + c) * slot_stride + 64;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const int e = tid + i * NT;
                acc[i] = fmaf(sm.w[c][e / D], ldp<G>(O + e), acc[i]);
            }
        }
        Sync::sync();
    }
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int e = tid + i * NT;
        const int q = e / D, d = e % D;
        float val = acc[i];
        if (full) val = fmaf(sm.beta[q], olo_row[d], val);
        out_blk[e] = to_out<OutT>(val * sm.inv[q]);
    }
}

// Shared epilogue: the item's (m, l, O) sit in `stage` (shared, slot layout).
template <int D, int NT, typename OutT, typename Sync>
__device__ void finish_item(float *stage, int slot, int chunk, int nchunks, int row, int full,
                            const float *mlo, const float *olo, const float *llo,
                            float *partial, int *row_arrive, const float *qmask, OutT *out_blk,
                            MergeSmem &sm, int *s_last) {
    const int tid = threadIdx.x;
    const size_t stride = (size_t)32 * (D + 2);
    const float m_lo2 = full ? mlo[row] * kLog2e : 0.0f;
    const float l_lo = full ? llo[row] : 0.0f;
    const float *olo_row = full ? olo + (size_t)row * D : nullptr;
    if (nchunks == 1) {
        merge_write<D, NT, false, OutT, Sync>(stage, stride, 1, full, m_lo2, l_lo, olo_row, qmask, out_blk, sm);
        return;
    }
    float *dst = partial + (size_t)slot * stride;
    for (int e = tid; e < (int)stride; e += NT) dst[e] = stage[e];
    __threadfence();
    Sync::sync();
    if (tid == 0) *s_last = (atomicAdd(&row_arrive[row], 1) == nchunks - 1);
    Sync::sync();
    if (!*s_last) return;
    __threadfence();
    merge_write<D, NT, true, OutT, Sync>(partial + (size_t)(slot - chunk) * stride, stride, nchunks, full,
                                   m_lo2, l_lo, olo_row, qmask, out_blk, sm);
    if (tid == 0) row_arrive[row] = 0;
}

}  // namespace attn
}  // namespace mra
