// mra_select_common.cuh - device helper shared by the kernels that locate
// the bucket of the k-th largest selection key (radix select over per-head
// histograms, page "深入解析 Transformers 中的 MRA 模型", step two: global top-k).
#pragma once

#include "mra_internal.cuh"

namespace mra {

// Finds, in the global histogram gh[0..nbins) of one head (read through L2),
// the bucket that holds the need-th largest element counted from the top.
// Runs on all 256 threads of the block; writes the bucket and the count still
// needed inside it to *out_bin / *out_need (shared memory).
static __device__ __noinline__ void find_bucket_256(const unsigned int *gh, int nbins, unsigned int need,
                                unsigned int *s_tmp /* >= 256 */, int *out_bin,
                                unsigned int *out_need) {
    const int t = threadIdx.x;
    const int per = nbins / 256;
    if (t == 0) {  // defined result even if no bucket qualifies (cannot happen when need <= total)
        *out_bin = 0;
        *out_need = 1;
    }
    unsigned int local = 0;
    for (int i = 0; i < per; ++i) local += __ldcg(gh + t * per + i);
    s_tmp[t] = local;
    __syncthreads();
    // inclusive suffix sum over threads (Hillis-Steele, 8 steps)
    for (int off = 1; off < 256; off <<= 1) {
        unsigned int add = (t + off < 256) ? s_tmp[t + off] : 0u;
        __syncthreads();
        s_tmp[t] += add;
        __syncthreads();
    }
    const unsigned int above = (t + 1 < 256) ? s_tmp[t + 1] : 0u;  // bins above my range
    if (above < need && need <= above + local) {
        unsigned int cum = above;
        for (int i = per - 1; i >= 0; --i) {
            unsigned int hb = __ldcg(gh + t * per + i);
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

}  // namespace mra
