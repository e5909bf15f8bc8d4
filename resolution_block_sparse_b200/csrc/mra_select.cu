// mra_select.cu - global top-num_block selection and the CSR / work-list build.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理", step two: a
// global top-k over each (batch, head)'s low-resolution map, k = num_block,
// returning the selected block coordinates.  Equal keys go to the smaller flat
// index r*nbr + c.
//
// Radix select over the 35-bit keys: the first 11-bit digit is histogrammed by
// the low-resolution kernel, two 12-bit digits here.  After each pass the last
// CTA of a head (threadfence + arrival counter, no waiting) locates the bucket
// of the k-th key; after the third pass the threshold key T is exact and
// `need` says how many keys equal to T are taken (the smallest indices).
// Then, per block row, counts of keys above / equal to T, a per-head scan that
// assigns CSR offsets and attention work items (chunks of at most `chunk`
// columns), and the column lists in ascending column order.
#include "mra_internal.cuh"
#include "mra_select_common.cuh"

namespace mra {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
radix_pass_kernel(const unsigned long long *__restrict__ keys, long long nbr2, long long chunk,
                  int pass, int shift, int bits, unsigned int *__restrict__ hist,
                  unsigned int *__restrict__ arrive, SelState *__restrict__ state) {
    pdl_wait();
    __shared__ unsigned int h[kHistBins];
    __shared__ unsigned int s_tmp[256];
    __shared__ int s_last, s_bin;
    __shared__ unsigned int s_need;
    const int t = threadIdx.x;
    const int bh = blockIdx.y;
    const SelState st = state[bh];
    const int hi = shift + bits;
    const unsigned long long want = st.prefix >> hi;
    const unsigned int dmask = (1u << bits) - 1u;
    for (int i = t; i < (1 << bits); i += kThreads) h[i] = 0u;
    __syncthreads();
    const long long start = (long long)blockIdx.x * chunk;
    const long long end = min(start + chunk, nbr2);
    const unsigned long long *kb = keys + (size_t)bh * nbr2;
    constexpr int kUnroll = 4;
    for (long long i0 = start + (t & ~31) * kUnroll; i0 < end; i0 += (long long)kThreads * kUnroll) {
        unsigned long long kv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const long long i = i0 + u * 32 + (t & 31);
            kv[u] = i < end ? __ldcg(kb + i) : ~0ull;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const long long i = i0 + u * 32 + (t & 31);
            const bool act = i < end && (kv[u] >> hi) == want;
            warp_hist_add(h, (unsigned)(kv[u] >> shift) & dmask, act);
        }
    }
    __syncthreads();
    unsigned int *gh = hist + ((size_t)bh * 3 + pass) * kHistBins;
    for (int i = t; i < (1 << bits); i += kThreads)
        if (h[i]) atomicAdd(&gh[i], h[i]);
    __threadfence();
    __syncthreads();
    if (t == 0) s_last = (atomicAdd(&arrive[(size_t)bh * 4 + pass], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    find_bucket_256(gh, 1 << bits, st.need, s_tmp, &s_bin, &s_need);
    if (t == 0) {
        SelState ns;
        ns.prefix = st.prefix | ((unsigned long long)s_bin << shift);
        ns.need = s_need;
        ns.pad = 0;
        state[bh] = ns;
    }
}

// One warp per block row: number of keys above and equal to the threshold.
__global__ void __launch_bounds__(kThreads)
row_counts_kernel(const unsigned long long *__restrict__ keys, const SelState *__restrict__ state,
                  int nbr, long long nbr2, int rows, int *__restrict__ gt, int *__restrict__ eq) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int bh = row / nbr, r = row % nbr;
    const unsigned long long T = state[bh].prefix;
    const unsigned long long *kr = keys + (size_t)bh * nbr2 + (size_t)r * nbr;
    int g = 0, e = 0;
    for (int c = lane; c < nbr; c += 32) {
        const unsigned long long key = kr[c];
        g += key > T;
        e += key == T;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (lane == 0) {
        gt[row] = g;
        eq[row] = e;
    }
}

constexpr int kScanThreads = 1024;

// Exclusive scan of one int per thread over the block; returns the prefix and
// writes the block total to *total.
__device__ int block_exclusive_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < kScanThreads / 32) ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;  // inclusive prefix of warp totals
    }
    __syncthreads();
    const int before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    *total = s_warp[kScanThreads / 32 - 1];
    __syncthreads();
    return before;
}

// One CTA per (batch, head): CSR row offsets and the attention work list.
__global__ void __launch_bounds__(kScanThreads)
row_scan_kernel(const int *__restrict__ gt, const int *__restrict__ eq,
                const SelState *__restrict__ state, int nbr, int k, int cap, int chunk,
                int *__restrict__ row_start, int *__restrict__ take_eq, WorkItem *__restrict__ items,
                int *__restrict__ head_items, unsigned int *__restrict__ status) {
    pdl_wait();
    __shared__ int s_warp[32];
    const int bh = blockIdx.x;
    const int t = threadIdx.x;
    const int per = (nbr + kScanThreads - 1) / kScanThreads;   // rows per thread (<= 2)
    const int rbeg = min(t * per, nbr), rend = min(rbeg + per, nbr);
    const int base = bh * nbr;
    const unsigned int need = state[bh].need;

    int eq_local = 0;
    for (int r = rbeg; r < rend; ++r) eq_local += eq[base + r];
    int tot;
    int eq_before = block_exclusive_scan(eq_local, s_warp, &tot);

    int sel[2] = {0, 0}, tk[2] = {0, 0};
    int sel_local = 0;
    for (int r = rbeg, i = 0; r < rend; ++r, ++i) {
        const int e = eq[base + r];
        int take = (int)need - eq_before;
        take = take < 0 ? 0 : (take > e ? e : take);
        tk[i] = take;
        sel[i] = gt[base + r] + take;
        sel_local += sel[i];
        eq_before += e;
    }
    int sel_total;
    int sel_before = block_exclusive_scan(sel_local, s_warp, &sel_total);
    int it_local = 0;
    for (int r = rbeg, i = 0; r < rend; ++r, ++i) it_local += sel[i] > 0 ? (sel[i] + chunk - 1) / chunk : 1;
    int it_total;
    int it_before = block_exclusive_scan(it_local, s_warp, &it_total);

    for (int r = rbeg, i = 0; r < rend; ++r, ++i) {
        const int rs = bh * k + sel_before;
        row_start[base + r] = rs;
        take_eq[base + r] = tk[i];
        const int n = sel[i] > 0 ? (sel[i] + chunk - 1) / chunk : 1;
        for (int j = 0; j < n && it_before + j < cap; ++j) {
            WorkItem w;
            w.row = base + r;
            w.col_start = rs + j * chunk;
            w.ncols = min(chunk, sel[i] - j * chunk);
            if (w.ncols < 0) w.ncols = 0;
            w.chunk_info = j | (n << 16);
            items[(size_t)bh * cap + it_before + j] = w;
        }
        sel_before += sel[i];
        it_before += n;
    }
    if (t == 0) {
        // a head whose selection does not add up to k is skipped (never read
        // out of bounds) and flagged in the status word
        const bool ok = (sel_total == k && it_total <= cap);
        head_items[bh] = ok ? it_total : 0;
        if (!ok) atomicOr(status, kDevCount);
    }
}

// One warp per block row: the selected columns in ascending order, the
// exported flat indices, and (full mode) the row's selection bitmap.
__global__ void __launch_bounds__(kThreads)
cols_kernel(const unsigned long long *__restrict__ keys, const SelState *__restrict__ state,
            const int *__restrict__ row_start, const int *__restrict__ take_eq, int nbr,
            long long nbr2, int rows, int k, int *__restrict__ cols, int32_t *__restrict__ sel_out,
            unsigned int *__restrict__ bitmap, int wpr) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int bh = row / nbr, r = row % nbr;
    const unsigned long long T = state[bh].prefix;
    const unsigned long long *kr = keys + (size_t)bh * nbr2 + (size_t)r * nbr;
    const int rs = row_start[row];
    const int take = take_eq[row];
    const int limit = (bh + 1) * k;   // this head's slice of cols[] ends here
    const unsigned int lt_mask = (1u << lane) - 1u;
    int eq_seen = 0, sel_seen = 0;
    for (int c0 = 0; c0 < nbr; c0 += 32) {
        const int c = c0 + lane;
        unsigned long long key = 0;
        if (c < nbr) key = kr[c];
        const bool is_gt = (c < nbr) && key > T;
        const bool is_eq = (c < nbr) && key == T;
        const unsigned int eqb = __ballot_sync(0xffffffffu, is_eq);
        const int eq_rank = eq_seen + __popc(eqb & lt_mask);
        const bool sel = is_gt || (is_eq && eq_rank < take);
        const unsigned int sb = __ballot_sync(0xffffffffu, sel);
        if (sel && rs + sel_seen + __popc(sb & lt_mask) < limit) {
            const int pos = rs + sel_seen + __popc(sb & lt_mask);
            cols[pos] = c;
            if (sel_out) sel_out[pos] = r * nbr + c;
        }
        if (bitmap && lane == 0) bitmap[(size_t)row * wpr + (c0 >> 5)] = sb;
        eq_seen += __popc(eqb);
        sel_seen += __popc(sb);
    }
}

constexpr int kSmallThreads = 1024;

// Whole selection of one (batch, head) in one CTA, for maps of at most
// kSmallMaxKeys keys (nbr <= 128): the keys stay in shared memory for the
// two remaining radix passes, the per-row counts, the row scan, the work
// list and the column lists.
__global__ void __launch_bounds__(kSmallThreads)
select_small_kernel(const unsigned long long *__restrict__ keys, SelState *__restrict__ state,
                    int nbr, int k, int cap, int chunk, int *__restrict__ cols, int32_t *__restrict__ sel_out,
                    unsigned int *__restrict__ bitmap, int wpr, WorkItem *__restrict__ items,
                    int *__restrict__ head_items, unsigned int *__restrict__ status) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned long long sk[];   // [nbr * nbr]
    __shared__ unsigned int h[kHistBins];
    __shared__ unsigned int s_tmp[kSmallThreads];
    __shared__ int s_gt[kSmallMaxRows], s_eq[kSmallMaxRows], s_sel[kSmallMaxRows];
    __shared__ int s_start[kSmallMaxRows], s_take[kSmallMaxRows], s_item[kSmallMaxRows];
    __shared__ int s_bin, s_total_sel, s_total_items;
    __shared__ unsigned int s_need;
    const int bh = blockIdx.x;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int n = nbr * nbr;
    const unsigned long long *kb = keys + (size_t)bh * n;
    {
        // all (up to 16) loads of this thread in flight before the stores
        constexpr int kL = kSmallMaxKeys / kSmallThreads;
        unsigned long long v[kL];
#pragma unroll
        for (int u = 0; u < kL; ++u) {
            const int i = t + u * kSmallThreads;
            v[u] = i < n ? __ldcg(kb + i) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < kL; ++u) {
            const int i = t + u * kSmallThreads;
            if (i < n) sk[i] = v[u];
        }
    }
    const SelState st = state[bh];
    unsigned long long prefix = st.prefix;
    unsigned int need = st.need;
    __syncthreads();

    for (int pass = 1; pass <= 2; ++pass) {
        const int shift = (pass == 1) ? kHist2Bits : 0;
        const int bits = (pass == 1) ? kHist1Bits : kHist2Bits;
        const int hi = shift + bits;
        const unsigned long long want = prefix >> hi;
        const unsigned int dmask = (1u << bits) - 1u;
        for (int i = t; i < (1 << bits); i += kSmallThreads) h[i] = 0u;
        __syncthreads();
        for (int i0 = (t & ~31); i0 < n; i0 += kSmallThreads) {
            const int i = i0 + lane;
            const unsigned long long key = i < n ? sk[i] : ~0ull;
            warp_hist_add(h, (unsigned)(key >> shift) & dmask, i < n && (key >> hi) == want);
        }
        __syncthreads();
        find_bucket<kSmallThreads>([](int i) { return h[i]; }, 1 << bits, need, s_tmp, &s_bin,
                                   &s_need);
        prefix |= (unsigned long long)s_bin << shift;
        need = s_need;
        __syncthreads();
    }
    const unsigned long long T = prefix;
    if (t == 0) {
        SelState ns;
        ns.prefix = T;
        ns.need = need;
        ns.pad = 0;
        state[bh] = ns;
    }

    // keys above / equal to the threshold, per block row
    for (int r = warp; r < nbr; r += kSmallThreads / 32) {
        int g = 0, e = 0;
        for (int c = lane; c < nbr; c += 32) {
            const unsigned long long key = sk[r * nbr + c];
            g += key > T;
            e += key == T;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (lane == 0) {
            s_gt[r] = g;
            s_eq[r] = e;
        }
    }
    __syncthreads();
    // row scan on warp 0: rows 4*lane .. 4*lane+3
    if (warp == 0) {
        int eqv[4], sel[4], itm[4];
        int eq_local = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = 4 * lane + j;
            eqv[j] = r < nbr ? s_eq[r] : 0;
            eq_local += eqv[j];
        }
        int x = eq_local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        int eq_before = x - eq_local;
        int sel_local = 0, it_local = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = 4 * lane + j;
            int take = (int)need - eq_before;
            take = take < 0 ? 0 : (take > eqv[j] ? eqv[j] : take);
            sel[j] = r < nbr ? s_gt[r] + take : 0;
            itm[j] = r < nbr ? (sel[j] > 0 ? (sel[j] + chunk - 1) / chunk : 1) : 0;
            if (r < nbr) s_take[r] = take;
            eq_before += eqv[j];
            sel_local += sel[j];
            it_local += itm[j];
        }
        int xs = sel_local, xi = it_local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ys = __shfl_up_sync(0xffffffffu, xs, o);
            const int yi = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) {
                xs += ys;
                xi += yi;
            }
        }
        int sb = xs - sel_local, ib = xi - it_local;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = 4 * lane + j;
            if (r < nbr) {
                s_sel[r] = sel[j];
                s_start[r] = sb;
                s_item[r] = ib;
            }
            sb += sel[j];
            ib += itm[j];
        }
        if (lane == 31) {
            s_total_sel = xs;
            s_total_items = xi;
        }
    }
    __syncthreads();
    const bool ok = (s_total_sel == k && s_total_items <= cap);
    if (t == 0) {
        head_items[bh] = ok ? s_total_items : 0;
        if (!ok) atomicOr(status, kDevCount);
    }
    if (!ok) return;
    // work items: one thread per row
    for (int r = t; r < nbr; r += kSmallThreads) {
        const int sel = s_sel[r];
        const int nit = sel > 0 ? (sel + chunk - 1) / chunk : 1;
        const int rs = bh * k + s_start[r];
        for (int j = 0; j < nit; ++j) {
            WorkItem w;
            w.row = bh * nbr + r;
            w.col_start = rs + j * chunk;
            w.ncols = max(0, min(chunk, sel - j * chunk));
            w.chunk_info = j | (nit << 16);
            items[(size_t)bh * cap + s_item[r] + j] = w;
        }
    }
    // column lists: one warp per row, ascending columns
    const unsigned int lt_mask = (1u << lane) - 1u;
    for (int r = warp; r < nbr; r += kSmallThreads / 32) {
        const int rs = bh * k + s_start[r];
        const int take = s_take[r];
        int eq_seen = 0, sel_seen = 0;
        for (int c0 = 0; c0 < nbr; c0 += 32) {
            const int c = c0 + lane;
            const unsigned long long key = c < nbr ? sk[r * nbr + c] : 0ull;
            const bool is_gt = c < nbr && key > T;
            const bool is_eq = c < nbr && key == T;
            const unsigned int eqb = __ballot_sync(0xffffffffu, is_eq);
            const bool sel = is_gt || (is_eq && eq_seen + __popc(eqb & lt_mask) < take);
            const unsigned int sb = __ballot_sync(0xffffffffu, sel);
            if (sel) {
                const int pos = rs + sel_seen + __popc(sb & lt_mask);
                cols[pos] = c;
                if (sel_out) sel_out[pos] = r * nbr + c;
            }
            if (bitmap && lane == 0) bitmap[((size_t)bh * nbr + r) * wpr + (c0 >> 5)] = sb;
            eq_seen += __popc(eqb);
            sel_seen += __popc(sb);
        }
    }
}

}  // namespace

cudaError_t launch_radix_pass(const Problem &p, const Workspace &w, int pass, cudaStream_t s) {
    // pass 1: bits 12..23, pass 2: bits 0..11
    const int shift = (pass == 1) ? kHist2Bits : 0;
    const int bits = (pass == 1) ? kHist1Bits : kHist2Bits;
    dim3 grid(p.radix_ctas, p.BH);
    return launch_dependent(radix_pass_kernel, dim3(grid), dim3(kThreads), 0, s, w.keys, p.nbr2, p.radix_chunk, pass, shift, bits,
                                                w.hist, w.arrive, w.state);
}

cudaError_t launch_row_counts(const Problem &p, const Workspace &w, cudaStream_t s) {
    const int rows = p.BH * p.nbr;
    const int grid = (rows + kThreads / 32 - 1) / (kThreads / 32);
    return launch_dependent(row_counts_kernel, dim3(grid), dim3(kThreads), 0, s, w.keys, w.state, p.nbr, p.nbr2, rows, w.gt, w.eq);
}

cudaError_t launch_row_scan(const Problem &p, const Workspace &w, cudaStream_t s) {
    return launch_dependent(row_scan_kernel, dim3(p.BH), dim3(kScanThreads), 0, s, w.gt, w.eq, w.state, p.nbr, p.k, p.cap, p.chunk,
                                                  w.row_start, w.take_eq, w.items, w.head_items,
                                                  w.status);
}

cudaError_t launch_select_small(const Problem &p, const Workspace &w, int32_t *sel_out,
                                cudaStream_t s) {
    const size_t smem = sizeof(unsigned long long) * (size_t)p.nbr2;
    cudaError_t e = cudaFuncSetAttribute(select_small_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_dependent(select_small_kernel, dim3(p.BH), dim3(kSmallThreads), smem, s,
        w.keys, w.state, p.nbr, p.k, p.cap, p.chunk, w.cols, sel_out, p.mode == 0 ? w.bitmap : nullptr,
        w.words_per_row, w.items, w.head_items, w.status);
}

cudaError_t launch_cols(const Problem &p, const Workspace &w, int32_t *sel_out, cudaStream_t s) {
    const int rows = p.BH * p.nbr;
    const int grid = (rows + kThreads / 32 - 1) / (kThreads / 32);
    return launch_dependent(cols_kernel, dim3(grid), dim3(kThreads), 0, s, w.keys, w.state, w.row_start, w.take_eq, p.nbr, p.nbr2,
                                          rows, p.k, w.cols, sel_out, p.mode == 0 ? w.bitmap : nullptr,
                                          w.words_per_row);
}

}  // namespace mra
