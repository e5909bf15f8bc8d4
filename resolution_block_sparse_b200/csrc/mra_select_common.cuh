// mra_select_common.cuh - device helpers shared by the kernels of the global
// top-k (radix select over per-head histograms; page "深入解析 Transformers 中
// 的 MRA 模型", section "源码级原理", step two: global top-k, k = num_block).
#pragma once

#include "mra_internal.cuh"

namespace mra {

// Histogram increment, one shared-memory atomic per counted key (measured
// faster than aggregating the lanes of a warp that carry the same bin with
// __match_any_sync first: the N=16384 keys kernel 3.3 us faster).
static __device__ __forceinline__ void hist_add(unsigned int *h, unsigned int bin, bool active) {
    if (active) atomicAdd(&h[bin], 1u);
}

// Finds, in the histogram h[0..nbins) of one head, the bucket that holds the
// need-th largest element counted from the top.  Runs on all NT threads of
// the block; `load` reads one bin (global memory through L2, or shared).
// Writes the bucket and the count still needed inside it to *out_bin /
// *out_need (shared memory).
template <int NT, typename Load>
static __device__ __forceinline__ void find_bucket(Load load, int nbins, unsigned int need,
                                                   unsigned int *s_tmp /* >= NT */,
                                                   int *out_bin, unsigned int *out_need) {
    const int t = threadIdx.x;
    const int per = nbins / NT;
    if (t == 0) {  // defined result even if no bucket qualifies (cannot happen when need <= total)
        *out_bin = 0;
        *out_need = 1;
    }
    unsigned int local = 0;
    for (int i = 0; i < per; ++i) local += load(t * per + i);
    s_tmp[t] = local;
    __syncthreads();
    // inclusive suffix sum over threads (Hillis-Steele)
    for (int off = 1; off < NT; off <<= 1) {
        const unsigned int add = (t + off < NT) ? s_tmp[t + off] : 0u;
        __syncthreads();
        s_tmp[t] += add;
        __syncthreads();
    }
    const unsigned int above = (t + 1 < NT) ? s_tmp[t + 1] : 0u;  // bins above my range
    if (above < need && need <= above + local) {
        unsigned int cum = above;
        for (int i = per - 1; i >= 0; --i) {
            const unsigned int hb = load(t * per + i);
            if (cum + hb >= need) {
                *out_bin = t * per + i;
                *out_need = need - cum;
                break;
            }
            cum += hb;
        }
    }
    __syncthreads();
}

// Same result as find_bucket for a histogram in shared memory, with two block
// barriers: each warp sums a contiguous segment of the bins; in the warp whose
// segment holds the bucket every lane sums its own run of NBINS / NT bins, a
// shuffle suffix sum over the lanes finds the run, and that lane walks it.
template <int NT, int NBINS>
static __device__ __forceinline__ void find_bucket_smem(const unsigned int *h, unsigned int need,
                                                        unsigned int *s_tot /* >= NT / 32 */,
                                                        int *out_bin, unsigned int *out_need) {
    constexpr int W = NT / 32;
    constexpr int kSeg = NBINS / W;   // bins per warp
    constexpr int kPer = kSeg / 32;   // bins per lane
    static_assert(kPer >= 4 && kPer % 4 == 0 && kPer <= 16, "bins per lane");
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const unsigned int *hl = h + warp * kSeg + lane * kPer;
    unsigned int v[kPer];
#pragma unroll
    for (int i = 0; i < kPer; i += 4) {
        const uint4 x = *reinterpret_cast<const uint4 *>(hl + i);
        v[i] = x.x;
        v[i + 1] = x.y;
        v[i + 2] = x.z;
        v[i + 3] = x.w;
    }
    unsigned int mine = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) mine += v[i];
    const unsigned int sum = __reduce_add_sync(0xffffffffu, mine);
    if (lane == 0) s_tot[warp] = sum;
    if (t == 0) {
        *out_bin = 0;
        *out_need = 1;
    }
    __syncthreads();
    unsigned int above = 0;
    for (int w2 = warp + 1; w2 < W; ++w2) above += s_tot[w2];
    if (above < need && need <= above + sum) {   // warp-uniform
        unsigned int sfx = mine;   // runs of lanes lane..31
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned int y = __shfl_down_sync(0xffffffffu, sfx, o);
            if (lane + o < 32) sfx += y;
        }
        unsigned int cum = above + sfx - mine;   // bins above this lane's run
        if (cum < need && need <= cum + mine) {
#pragma unroll
            for (int i = kPer - 1; i >= 0; --i) {
                if (cum + v[i] >= need) {
                    *out_bin = warp * kSeg + lane * kPer + i;
                    *out_need = need - cum;
                    break;
                }
                cum += v[i];
            }
        }
    }
    __syncthreads();
}

// The global-memory form used by the multi-CTA passes (histogram in L2).
static __device__ __forceinline__ void find_bucket_256(const unsigned int *gh, int nbins,
                                                       unsigned int need, unsigned int *s_tmp,
                                                       int *out_bin, unsigned int *out_need) {
    find_bucket<256>([gh](int i) { return __ldcg(gh + i); }, nbins, need, s_tmp, out_bin, out_need);
}

}  // namespace mra
