// mra_group_plan.cu - work items of the tcgen05 attention kernel.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理", step three:
// the exact attention runs only on the selected 32x32 blocks.  The tcgen05
// kernel computes it on tiles of 128 query rows, i.e. four adjacent block rows
// of one head (M = 128, one query row per tensor-memory lane), over the union
// of the four rows' selected key blocks; each union entry carries which of
// the four rows selected it, so every other (row, key block) pair is masked
// out of the softmax and receives no weight.
//
// One CTA per (batch, head) turns the per-row work items and column lists of
// the selection (or of a caller's block list) into
//   ucols   the union entries of every group, key blocks ascending:
//           c | rows << 16 | partly-padded-key-block << 20,
//   gitems  work items: a group and a chunk of at most gchunk union entries
//           (a group with an empty union still gets one item, which writes its
//           low-resolution or zero output),
// and records the head's item count and the largest count over all heads.
// Key blocks without a valid token and block rows without a valid query are
// dropped from the unions: their terms are exactly zero.
#include "mra_internal.cuh"

namespace mra {
namespace {

constexpr int kPlanThreads = 512;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kMaxRows = kMaxN / kBlock;             // 2048 block rows
constexpr int kMaxGroups = kMaxRows / kGroupRows;    // 512 groups
static_assert(kMaxGroups <= kPlanThreads, "one thread per group in the scans");

// Exclusive prefix sum over the CTA; *total gets the sum.
__device__ int plan_exclusive_scan(int v, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < kPlanWarps ? warp_sums[lane] : 0;
        int z = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += y;
        }
        if (lane < kPlanWarps) warp_sums[lane] = z - w;
        if (lane == 31) warp_sums[32] = z;
    }
    __syncthreads();
    const int res = warp_sums[warp] + x - v;
    *total = warp_sums[32];
    __syncthreads();
    return res;
}

// Selection bitmaps of up to kSmemRows block rows per head live in shared
// memory (32 KB); longer maps use the workspace bitmap of the head (the
// low-resolution PV kernel, which reads the selection's bitmap there in full
// mode, has completed before this kernel starts).
constexpr int kSmemRows = 512;
constexpr int kSmemWords = kSmemRows * kSmemRows / 32;

__global__ void __launch_bounds__(kPlanThreads)
group_plan_kernel(const WorkItem *__restrict__ items, const int *__restrict__ head_items,
                  const int *__restrict__ cols, const int *__restrict__ cnt, int has_mask, int H, int nbr,
                  int cap, int k, int ngroups, int gchunk, int gcap, unsigned int *__restrict__ gbitmap,
                  int *__restrict__ ucols, GroupItem *__restrict__ gitems, int *__restrict__ head_gitems,
                  int *__restrict__ group_arrive, int *__restrict__ max_items, unsigned int *__restrict__ status) {
    pdl_wait();
    __shared__ unsigned int s_bits[kSmemWords];
    __shared__ int s_ucnt[kMaxGroups], s_nit[kMaxGroups], s_ustart[kMaxGroups], s_istart[kMaxGroups];
    __shared__ int warp_sums[33];
    const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b = bh / H;
    const int wpr = (nbr + 31) / 32;
    const int *cnt_b = cnt ? cnt + (size_t)b * nbr : nullptr;
    unsigned int *bits = nbr <= kSmemRows ? s_bits : gbitmap + (size_t)bh * nbr * wpr;
    for (int i = t; i < nbr * wpr; i += kPlanThreads) bits[i] = 0u;
    for (int g = t; g < ngroups; g += kPlanThreads) group_arrive[(size_t)bh * ngroups + g] = 0;
    __syncthreads();
    // every selected (row, key block) of the head into the row bitmaps: one
    // thread per work item of the selection, all loads independent; rows
    // without a valid query and key blocks without a valid token are dropped
    const int nitems = head_items[bh];
    for (int i = t; i < nitems; i += kPlanThreads) {
        const WorkItem it = items[(size_t)bh * cap + i];
        const int r = it.row - bh * nbr;
        if (r < 0 || r >= nbr || (cnt_b && cnt_b[r] == 0)) continue;
        for (int e = 0; e < it.ncols; ++e) {
            const int c = cols[it.col_start + e];
            if (c < 0 || c >= nbr || (cnt_b && cnt_b[c] == 0)) continue;
            atomicOr(&bits[r * wpr + (c >> 5)], 1u << (c & 31));
        }
    }
    __syncthreads();
    // union sizes and item counts: one warp per group, lanes over the words
    auto row_word = [&](int g, int j, int w) -> unsigned int {
        const int r = g * kGroupRows + j;
        return r < nbr ? bits[r * wpr + w] : 0u;
    };
    for (int g = warp; g < ngroups; g += kPlanWarps) {
        int u = 0;
        for (int w = lane; w < wpr; w += 32)
            u += __popc(row_word(g, 0, w) | row_word(g, 1, w) | row_word(g, 2, w) | row_word(g, 3, w));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
        if (lane == 0) {
            s_ucnt[g] = u;
            s_nit[g] = u > 0 ? (u + gchunk - 1) / gchunk : 1;
        }
    }
    __syncthreads();
    int utot = 0, ntot = 0;
    const int us = plan_exclusive_scan(t < ngroups ? s_ucnt[t] : 0, warp_sums, &utot);
    const int is = plan_exclusive_scan(t < ngroups ? s_nit[t] : 0, warp_sums, &ntot);
    if (t < ngroups) {
        s_ustart[t] = us;
        s_istart[t] = is;
    }
    __syncthreads();
    if (utot > k || ntot > gcap) {
        // cannot happen for a valid selection (each union entry is a selected
        // block); leaves the head without work rather than writing out of range
        if (t == 0) {
            head_gitems[bh] = 0;
            atomicOr(status, kDevCount);
        }
        return;
    }
    // union entries in ascending key-block order (lane = column within a
    // 32-column word), then the items of the group
    const unsigned int below = (1u << lane) - 1u;
    for (int g = warp; g < ngroups; g += kPlanWarps) {
        int o = bh * k + s_ustart[g];
        for (int w = 0; w < wpr; ++w) {
            const unsigned int a0 = row_word(g, 0, w), a1 = row_word(g, 1, w), a2 = row_word(g, 2, w),
                               a3 = row_word(g, 3, w);
            const unsigned int u = a0 | a1 | a2 | a3;
            if ((u >> lane) & 1u) {
                const int c = w * 32 + lane;
                const int rows = (int)(((a0 >> lane) & 1u) | (((a1 >> lane) & 1u) << 1) | (((a2 >> lane) & 1u) << 2) |
                                       (((a3 >> lane) & 1u) << 3));
                const bool part = has_mask && (cnt_b == nullptr || cnt_b[c] < kBlock);
                ucols[o + __popc(u & below)] = c | (rows << kUnionRowShift) | (part ? kUnionPartial : 0);
            }
            o += __popc(u);
        }
        const int U = s_ucnt[g], nit = s_nit[g];
        for (int i = lane; i < nit; i += 32) {
            GroupItem it;
            it.group = bh * ngroups + g;
            it.ustart = bh * k + s_ustart[g] + i * gchunk;
            it.ucount = max(0, min(gchunk, U - i * gchunk));
            it.chunk_info = i | (nit << 16);
            gitems[(size_t)bh * gcap + s_istart[g] + i] = it;
        }
    }
    if (t == 0) {
        head_gitems[bh] = ntot;
        atomicMax(max_items, ntot);
    }
}

}  // namespace

cudaError_t launch_group_plan(const Problem &p, const Workspace &w, const float *mask, bool have_counts,
                              cudaStream_t s) {
    // the valid-token counts come from the pool kernel; block lists skip the
    // pool, so with a mask every entry is treated as possibly padded there
    const int *cnt = (mask && have_counts) ? w.cnt : nullptr;
    return launch_dependent(group_plan_kernel, dim3((unsigned)p.BH), dim3(kPlanThreads), 0, s, w.items,
                            w.head_items, w.cols, cnt, mask ? 1 : 0, p.H, p.nbr, p.cap, p.k,
                            p.ngroups, p.gchunk, p.gcap, w.bitmap, w.ucols, w.gitems, w.head_gitems,
                            w.group_arrive,
                            w.work_next + 2, w.status);
}

}  // namespace mra
