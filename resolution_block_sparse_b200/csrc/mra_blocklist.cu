// mra_blocklist.cu - block-sparse attention on a caller-given block set, and
// the BigBird block pattern as one such set.
//
// The attention kernels take work items (block row, chunk of selected key
// blocks) and per-head column lists; the MRA path builds them from its
// top-k.  Here they come from a sorted list of flat block indices r*nbr + c
// per head, so the same kernels run any block-sparse pattern (sparse mode:
// softmax over the union of the given blocks, no low-resolution part).
//
// Page "Transformers 中的 BigBird：面向超长序列的稀疏注意力模型完全指南", the
// attention-mechanism section and the usage notes: a window of 3 blocks, 2
// global blocks (attend to and are attended by every block), at least one
// random block per query block, the sequence length a multiple of the block
// size, and full attention for sequences of at most (5 + 2r) blocks.
// Readings where the page is open: the global blocks are the first and the
// last block; the window is clipped at the ends; a block chosen twice counts
// once; the random blocks are drawn by the caller.
#include <algorithm>
#include <vector>

#include "mra.h"
#include "mra_internal.cuh"

namespace mra {
namespace {

constexpr int kListThreads = 1024;

// Exclusive prefix sum over the CTA (1024 threads); *total gets the sum.
__device__ int cta_exclusive_scan(int v, int *warp_sums, int *total) {
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
        int w = warp_sums[lane];
        int z = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += y;
        }
        warp_sums[lane] = z - w;   // exclusive over warps
        if (lane == 31) warp_sums[32] = z;
    }
    __syncthreads();
    const int res = warp_sums[warp] + x - v;
    *total = warp_sums[32];
    __syncthreads();
    return res;
}

// One CTA per (batch, head): clears the attention kernel's per-call counters
// (the head's row and item-group arrival counts; CTA 0 the work counter), validates the
// head's list (entries in [0, nbr^2), strictly increasing, -1 padding only at
// the end) while counting its entries per block row and writing the column
// list, then builds the work items (row starts = exclusive scan of the row
// counts, which is where each row's run begins in the sorted list) and the
// head's item count.  An invalid list flags MRA_DEV_COUNT and leaves the head
// with no work items.
__global__ void __launch_bounds__(kListThreads)
blocklist_items_kernel(const int32_t *__restrict__ lists, int cap_sel, int nbr, int k, int cap, int chunk,
                       int *__restrict__ cols, WorkItem *__restrict__ items, int *__restrict__ head_items,
                       int *__restrict__ row_arrive, int *__restrict__ slot_arrive, int *__restrict__ work_next,
                       unsigned int *__restrict__ status) {
    pdl_wait();
    __shared__ int warp_sums[33];
    __shared__ int s_cnt[kMaxN / kBlock];
    __shared__ int s_len, s_bad;
    const int bh = blockIdx.x, t = threadIdx.x;
    const int32_t *lst = lists + (size_t)bh * cap_sel;
    const long long nbr2 = (long long)nbr * nbr;
    for (int r = t; r < nbr; r += kListThreads) {
        row_arrive[(size_t)bh * nbr + r] = 0;
        s_cnt[r] = 0;
    }
    for (int i = t; i < cap; i += kListThreads) slot_arrive[(size_t)bh * cap + i] = 0;
    if (bh == 0 && t < 4) work_next[t] = 0;
    if (t == 0) {
        s_len = cap_sel;
        s_bad = 0;
    }
    __syncthreads();
    for (int i = t; i < cap_sel; i += kListThreads)
        if (lst[i] < 0) atomicMin(&s_len, i);
    __syncthreads();
    const int n = s_len;
    for (int i = t; i < cap_sel; i += kListThreads) {
        const int32_t x = lst[i];
        if (i < n) {
            if (x < nbr2 && (i + 1 >= n || x < lst[i + 1])) {
                const int r = x / nbr;
                atomicAdd(&s_cnt[r], 1);
                cols[(size_t)bh * k + i] = x - r * nbr;
            } else {
                s_bad = 1;
            }
        } else if (x >= 0) {
            s_bad = 1;
        }
    }
    __syncthreads();
    if (s_bad || n > k) {
        if (t == 0) {
            head_items[bh] = 0;
            atomicOr(status, kDevCount);
        }
        return;
    }
    // rows t*kRowsPer .. : counts, their exclusive scan (row starts), items
    constexpr int kRowsPer = (kMaxN / kBlock + kListThreads - 1) / kListThreads;   // 2
    int cnt[kRowsPer], nit[kRowsPer];
    int sel_local = 0, it_local = 0;
#pragma unroll
    for (int u = 0; u < kRowsPer; ++u) {
        const int r = t * kRowsPer + u;
        cnt[u] = r < nbr ? s_cnt[r] : 0;
        nit[u] = r < nbr ? (cnt[u] > 0 ? (cnt[u] + chunk - 1) / chunk : 1) : 0;
        sel_local += cnt[u];
        it_local += nit[u];
    }
    int sel_total, total;
    int sel_before = cta_exclusive_scan(sel_local, warp_sums, &sel_total);
    int it_before = cta_exclusive_scan(it_local, warp_sums, &total);
    if (total > cap) {
        if (t == 0) {
            head_items[bh] = 0;
            atomicOr(status, kDevCount);
        }
        return;
    }
#pragma unroll
    for (int u = 0; u < kRowsPer; ++u) {
        const int r = t * kRowsPer + u;
        if (r >= nbr) continue;
        for (int j = 0; j < nit[u]; ++j) {
            WorkItem w;
            w.row = bh * nbr + r;
            w.col_start = bh * k + sel_before + j * chunk;
            w.ncols = max(0, min(chunk, cnt[u] - j * chunk));
            w.chunk_info = j | (nit[u] << 16);
            items[(size_t)bh * cap + it_before + j] = w;
        }
        sel_before += cnt[u];
        it_before += nit[u];
    }
    if (t == 0) head_items[bh] = total;
}

}  // namespace

cudaError_t launch_blocklist_items(const Problem &p, const Workspace &w, const int32_t *lists, int cap_sel,
                                   cudaStream_t s) {
    return launch_dependent(blocklist_items_kernel, dim3((unsigned)p.BH), dim3(kListThreads), 0, s, lists, cap_sel,
                            p.nbr, p.k, p.cap, p.chunk, w.cols, w.items, w.head_items, w.row_arrive,
                            w.slot_arrive, w.work_next, w.status);
}

// The BigBird pattern of one head as sorted flat 32-token block indices.
int bigbird_block_list(int N, int block_size, int num_random, const int32_t *rand_blocks, int32_t *out,
                       int capacity, int *count) {
    if (N < kBlock || N % kBlock != 0 || block_size < kBlock || block_size % kBlock != 0 ||
        N % block_size != 0 || num_random < 1 || !rand_blocks || !out || !count)
        return MRA_ERR_INVALID_ARG;
    if (N > kMaxN) return MRA_ERR_UNSUPPORTED;
    const int nb = N / block_size, f = block_size / kBlock, nbr = N / kBlock;
    for (int i = 0; i < nb * num_random; ++i)
        if (rand_blocks[i] < 0 || rand_blocks[i] >= nb) return MRA_ERR_INVALID_ARG;
    const bool full = nb <= 5 + 2 * num_random;
    std::vector<unsigned char> coarse((size_t)nb * nb, 0);
    for (int i = 0; i < nb; ++i) {
        unsigned char *row = &coarse[(size_t)i * nb];
        if (full || i == 0 || i == nb - 1) {
            std::fill(row, row + nb, 1);
            continue;
        }
        row[0] = row[nb - 1] = 1;
        for (int j = std::max(0, i - 1); j <= std::min(nb - 1, i + 1); ++j) row[j] = 1;
        for (int u = 0; u < num_random; ++u) row[rand_blocks[(size_t)i * num_random + u]] = 1;
    }
    int n = 0;
    for (int r = 0; r < nbr; ++r)
        for (int c = 0; c < nbr; ++c) {
            if (!coarse[(size_t)(r / f) * nb + c / f]) continue;
            if (n >= capacity) return MRA_ERR_TOO_LARGE;
            out[n++] = r * nbr + c;
        }
    *count = n;
    return MRA_OK;
}

}  // namespace mra
