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

// four consecutive outputs (8-byte store for bf16, 16-byte for fp32)
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<unsigned *>(&a);
    u.y = *reinterpret_cast<unsigned *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}
__device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }

// four consecutive partial-output elements as fp32 (16-byte load for fp32
// partials, 8-byte for bf16 ones); G: through L2 only (written by other CTAs)
template <bool G>
__device__ __forceinline__ float4 ld_quad(const float *p) {
    if constexpr (G) return __ldcg(reinterpret_cast<const float4 *>(p));
    else return *reinterpret_cast<const float4 *>(p);
}
template <bool G>
__device__ __forceinline__ float4 ld_quad(const __nv_bfloat16 *p) {
    uint2 u;
    if constexpr (G) u = __ldcg(reinterpret_cast<const uint2 *>(p));
    else u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

constexpr int kMergeGroup = 16;   // partials whose (m, l) are staged at once

struct MergeSmem {
    float w[kMergeGroup][32];   // m of (chunk, row), then its weight
    float l[kMergeGroup][32];
    float M[32], den[32], resc[32];
    float lse2[32], dsum[32];   // per-row statistics for the backward pass
};

// Bytes of one partial slot: m[32] and l[32] in fp32, then O[32][D] in PartT.
template <int D, typename PartT>
__host__ __device__ constexpr size_t partial_slot_bytes() {
    return 64 * sizeof(float) + (size_t)32 * D * sizeof(PartT);
}

// Merge nchunks partials (slot layout above; m in log2 units, l and O
// relative to exp2(m)) with the low-resolution part of the row (full mode)
// and write the 32 x D output block.  Run by NT threads, tid = 0..NT-1 their
// index, that Sync synchronises.
//
// The partials are taken in groups of kMergeGroup: all (m, l) pairs of a group
// are loaded at once, the running per-row maximum and normaliser move to the
// group's maximum (earlier groups rescaled), and the O tiles of several
// partials are in flight together, so the merge costs a few memory round
// trips rather than two per partial.
template <int D, int NT, bool G, typename OutT, typename PartT, typename Sync>
__device__ void merge_write(const unsigned char *src0, size_t slot_bytes, int nchunks, int full,
                            float m_lo2, float l_lo, const float *olo_row, const float *qmask,
                            OutT *out_blk, int orow, MergeSmem &sm, int tid, const GradStats &gs) {
    static_assert((8 * D) % NT == 0, "a chunk's O tile must split evenly into quads per thread");
    constexpr int F = 8 * D / NT;   // quads (4 elements) of one partial's O tile per thread
    constexpr int kRowQ = D / 4;
    constexpr int kQuadBytes = 4 * (int)sizeof(PartT);
    // partial tiles in flight per thread: at most 128 bytes of registers
    constexpr int kMergeUnroll = F * kQuadBytes >= 128 ? 1 : 128 / (F * kQuadBytes);
    constexpr int kML = kMergeGroup * 32 / NT;   // (m, l) pairs per thread per group
    static_assert(kML >= 1 && (kMergeGroup * 32) % NT == 0, "merge group layout");
    float4 acc[F];
#pragma unroll
    for (int i = 0; i < F; ++i) acc[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (tid < 32) {
        sm.M[tid] = -INFINITY;
        sm.den[tid] = 0.0f;
    }
    for (int cg = 0; cg < nchunks; cg += kMergeGroup) {
        const int nc = min(kMergeGroup, nchunks - cg);
        {
            float mv[kML], lv[kML];
#pragma unroll
            for (int i = 0; i < kML; ++i) {
                const int e = tid + i * NT;
                const int c = e >> 5, q = e & 31;
                mv[i] = -INFINITY;
                lv[i] = 0.0f;
                if (c < nc) {
                    const float *P = reinterpret_cast<const float *>(src0 + (size_t)(cg + c) * slot_bytes);
                    lv[i] = ldp<G>(P + 32 + q);
                    mv[i] = ldp<G>(P + q);
                }
            }
#pragma unroll
            for (int i = 0; i < kML; ++i) {
                const int e = tid + i * NT;
                const int c = e >> 5, q = e & 31;
                if (c < nc) {
                    sm.w[c][q] = lv[i] > 0.0f ? mv[i] : -INFINITY;
                    sm.l[c][q] = lv[i] > 0.0f ? lv[i] : 0.0f;
                }
            }
        }
        Sync::sync();
        if (tid < 32) {
            const int q = tid;
            const float m_old = sm.M[q];
            float m_new = m_old;
            for (int c = 0; c < nc; ++c) m_new = fmaxf(m_new, sm.w[c][q]);
            const float resc = (m_old == -INFINITY) ? 0.0f : exp2f(m_old - m_new);
            float den = sm.den[q] * resc;
            for (int c = 0; c < nc; ++c) {
                const float m = sm.w[c][q];
                const float wgt = (m == -INFINITY) ? 0.0f : exp2f(m - m_new);
                den = fmaf(wgt, sm.l[c][q], den);
                sm.w[c][q] = wgt;
            }
            sm.M[q] = m_new;
            sm.den[q] = den;
            sm.resc[q] = resc;
        }
        Sync::sync();
        if (cg > 0) {
#pragma unroll
            for (int i = 0; i < F; ++i) {
                const float r = sm.resc[(tid + i * NT) / kRowQ];
                acc[i].x *= r;
                acc[i].y *= r;
                acc[i].z *= r;
                acc[i].w *= r;
            }
        }
#pragma unroll kMergeUnroll
        for (int c = 0; c < nc; ++c) {
            const PartT *O = reinterpret_cast<const PartT *>(src0 + (size_t)(cg + c) * slot_bytes +
                                                            64 * sizeof(float));
#pragma unroll
            for (int i = 0; i < F; ++i) {
                const int f = tid + i * NT;
                const float wgt = sm.w[c][f / kRowQ];
                const float4 v = ld_quad<G>(O + 4 * f);
                acc[i].x = fmaf(wgt, v.x, acc[i].x);
                acc[i].y = fmaf(wgt, v.y, acc[i].y);
                acc[i].z = fmaf(wgt, v.z, acc[i].z);
                acc[i].w = fmaf(wgt, v.w, acc[i].w);
            }
        }
        Sync::sync();
    }
    // low-resolution part at the shared maximum, normaliser, padded queries
    if (tid < 32) {
        const int q = tid;
        const float m_hi = sm.M[q];
        const bool lo = full && l_lo > 0.0f;
        const float M = lo ? fmaxf(m_hi, m_lo2) : m_hi;
        float a_hi = 0.0f, beta = 0.0f, inv = 0.0f, lse2 = INFINITY;
        if (M != -INFINITY && (!qmask || qmask[q] > 0.0f)) {
            a_hi = (m_hi == -INFINITY) ? 0.0f : exp2f(m_hi - M);
            beta = lo ? exp2f(m_lo2 - M) : 0.0f;
            const float den = a_hi * sm.den[q] + beta * l_lo;
            inv = den > 0.0f ? 1.0f / den : 0.0f;
            if (den > 0.0f) lse2 = M + log2f(den);
        }
        sm.resc[q] = a_hi * inv;   // factor of the merged high-resolution O
        sm.den[q] = beta * inv;    // factor of the low-resolution output
        sm.lse2[q] = lse2;
        sm.dsum[q] = 0.0f;
    }
    Sync::sync();
#pragma unroll
    for (int i = 0; i < F; ++i) {
        const int f = tid + i * NT;
        const int q = f / kRowQ, d = (f % kRowQ) * 4;
        const float fa = sm.resc[q], fb = sm.den[q];
        float4 ol = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (full) ol = *reinterpret_cast<const float4 *>(olo_row + d);
        const float4 ov = make_float4(fmaf(acc[i].x, fa, ol.x * fb), fmaf(acc[i].y, fa, ol.y * fb),
                                      fmaf(acc[i].z, fa, ol.z * fb), fmaf(acc[i].w, fa, ol.w * fb));
        store4(out_blk + (size_t)q * orow + d, ov);
        if (gs.lse2) {
            const size_t gi = (gs.qbase + q) * D + d;
            atomicAdd(&sm.dsum[q], ov.x * gs.dout_at(gi) + ov.y * gs.dout_at(gi + 1) +
                                       ov.z * gs.dout_at(gi + 2) + ov.w * gs.dout_at(gi + 3));
        }
    }
    if (gs.lse2) {
        Sync::sync();
        if (tid < 32) {
            gs.lse2[gs.qbase + tid] = sm.lse2[tid];
            gs.delta[gs.qbase + tid] = sm.dsum[tid];
        }
    }
}

// Partials of a split row are combined as a tree: the items of the row form
// groups of kTreeGroup consecutive items; the last item of a group to finish
// combines the group's partials into one (same slot format, in the group's
// first slot), and the last group to finish merges the group partials into
// the output.  Every hand-off is "the last to arrive continues" (arrival
// counters, no waiting), and the critical path of a row is one item plus two
// short merges instead of one merge over every partial.
constexpr int kTreeGroup = 4;

// Combines n <= kTreeGroup partials (slot layout of partial_slot_bytes, m in
// log2 units, l and O relative to exp2(m)) at src0, src0 + slot_bytes, ...
// into one partial of the same layout written over the first.  Run by the NT
// threads that Sync synchronises; tid = 0..NT-1.
template <int D, int NT, typename PartT, typename Sync>
__device__ void combine_group(unsigned char *src0, size_t slot_bytes, int n, MergeSmem &sm, int tid) {
    static_assert((8 * D) % NT == 0, "a partial's O tile must split evenly into quads per thread");
    constexpr int F = 8 * D / NT;   // quads of the O tile per thread
    constexpr int kRowQ = D / 4;
    if (tid < 32) {
        const int q = tid;
        float mv[kTreeGroup], lv[kTreeGroup];
#pragma unroll
        for (int c = 0; c < kTreeGroup; ++c) {
            const float *P = reinterpret_cast<const float *>(src0 + (size_t)c * slot_bytes);
            mv[c] = c < n ? __ldcg(P + q) : -INFINITY;
            lv[c] = c < n ? __ldcg(P + 32 + q) : 0.0f;
        }
        float M = -INFINITY;
#pragma unroll
        for (int c = 0; c < kTreeGroup; ++c)
            if (lv[c] > 0.0f) M = fmaxf(M, mv[c]);
        float L = 0.0f;
#pragma unroll
        for (int c = 0; c < kTreeGroup; ++c) {
            const float wgt = (lv[c] > 0.0f) ? exp2f(mv[c] - M) : 0.0f;
            sm.w[c][q] = wgt;
            L = fmaf(wgt, lv[c], L);
        }
        sm.M[q] = M;
        sm.den[q] = L;
    }
    Sync::sync();
    float4 acc[F];
#pragma unroll
    for (int i = 0; i < F; ++i) acc[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int c = 0; c < kTreeGroup; ++c) {
        if (c < n) {
            const PartT *O = reinterpret_cast<const PartT *>(src0 + (size_t)c * slot_bytes + 64 * sizeof(float));
#pragma unroll
            for (int i = 0; i < F; ++i) {
                const int f = tid + i * NT;
                const float wgt = sm.w[c][f / kRowQ];
                const float4 v = ld_quad<true>(O + 4 * f);
                acc[i].x = fmaf(wgt, v.x, acc[i].x);
                acc[i].y = fmaf(wgt, v.y, acc[i].y);
                acc[i].z = fmaf(wgt, v.z, acc[i].z);
                acc[i].w = fmaf(wgt, v.w, acc[i].w);
            }
        }
    }
    Sync::sync();   // every read of the group's slots is done before the first is overwritten
    float *P0 = reinterpret_cast<float *>(src0);
    if (tid < 32) {
        P0[tid] = sm.M[tid];
        P0[32 + tid] = sm.den[tid];
    }
    PartT *O0 = reinterpret_cast<PartT *>(src0 + 64 * sizeof(float));
#pragma unroll
    for (int i = 0; i < F; ++i) store4(O0 + 4 * (tid + i * NT), acc[i]);
}

// Shared epilogue: the item's (m, l, O) sit in `stage` (shared memory, slot
// layout of partial_slot_bytes<D, PartT>).  A row that fits one item merges
// and writes at once; otherwise the slot is copied to the partial buffer and
// the row's partials are combined as a tree (kTreeGroup above): slot_arrive
// counts the arrivals of a group at its first slot, row_arrive the groups of
// the row.
template <int D, int NT, typename OutT, typename PartT, typename Sync>
__device__ void finish_item(const unsigned char *stage, int slot, int chunk, int nchunks, int row, int full,
                            const float *mlo, const float *olo, const float *llo,
                            unsigned char *partial, int *row_arrive, int *slot_arrive, const float *qmask,
                            OutT *out_blk, int orow, MergeSmem &sm, int *s_last, const GradStats &gs) {
    constexpr size_t kSlot = partial_slot_bytes<D, PartT>();
    static_assert(kSlot % 16 == 0, "partial slots stay 16-byte aligned");
    const int tid = threadIdx.x;
    const float m_lo2 = full ? mlo[row] * kLog2e : 0.0f;
    const float l_lo = full ? llo[row] : 0.0f;
    const float *olo_row = full ? olo + (size_t)row * D : nullptr;
    if (nchunks == 1) {
        merge_write<D, NT, false, OutT, PartT, Sync>(stage, kSlot, 1, full, m_lo2, l_lo, olo_row, qmask,
                                                     out_blk, orow, sm, tid, gs);
        return;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(partial + (size_t)slot * kSlot);
    const uint4 *src = reinterpret_cast<const uint4 *>(stage);
    for (int e = tid; e < (int)(kSlot / 16); e += NT) dst[e] = src[e];
    __threadfence();
    Sync::sync();
    const int row_slot0 = slot - chunk;
    const int first = (chunk / kTreeGroup) * kTreeGroup;
    const int gsize = min(kTreeGroup, nchunks - first);
    const int ngroups = (nchunks + kTreeGroup - 1) / kTreeGroup;
    unsigned char *grp0 = partial + (size_t)(row_slot0 + first) * kSlot;
    if (gsize > 1) {
        if (tid == 0) *s_last = (atomicAdd(&slot_arrive[row_slot0 + first], 1) == gsize - 1);
        Sync::sync();
        if (!*s_last) return;
        __threadfence();
        combine_group<D, NT, PartT, Sync>(grp0, kSlot, gsize, sm, tid);
        if (tid == 0) slot_arrive[row_slot0 + first] = 0;
        __threadfence();
        Sync::sync();
    }
    if (ngroups > 1) {
        if (tid == 0) *s_last = (atomicAdd(&row_arrive[row], 1) == ngroups - 1);
        Sync::sync();
        if (!*s_last) return;
        __threadfence();
    }
    // the group partials sit kTreeGroup slots apart from the row's first slot
    merge_write<D, NT, true, OutT, PartT, Sync>(partial + (size_t)row_slot0 * kSlot, kTreeGroup * kSlot, ngroups,
                                                full, m_lo2, l_lo, olo_row, qmask, out_blk, orow, sm, tid, gs);
    if (tid == 0 && ngroups > 1) row_arrive[row] = 0;
}

}  // namespace attn
}  // namespace mra
