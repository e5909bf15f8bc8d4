// mra_select.cu - global top-num_block selection and the CSR / work-list build
// for maps above 128 x 128 blocks.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理", step two: a
// global top-k over each (batch, head)'s low-resolution map, k = num_block,
// returning the selected block coordinates.  Equal keys go to the smaller flat
// index r*nbr + c.
//
// Radix select over the 35-bit keys (an 11-bit digit, then two of 12 bits).
// The keys kernel (mra_lowres.cu) histograms the first digit and locates the
// bucket of the k-th key.  Then:
//   select_scan      one pass over every key: keys whose first digit is above
//                    the bucket are selected for certain (they go straight
//                    into the selection bitmap), keys in the bucket (about
//                    2 K of a head's 262 K on the N=16384 workload) are
//                    compacted with their flat index into a candidate list;
//   select_finalize  one CTA per head: the two lower digits over the
//                    candidates give the exact threshold T and how many keys
//                    equal to T are taken; candidates above T join the
//                    bitmap, those equal to T go to a tie bitmap; per row the
//                    counts above and at T (the scan's certain counts plus the
//                    candidates'), then a scan over the rows that assigns CSR
//                    offsets, work items and the ties in row order;
//   select_cols      one warp per row: the column lists in ascending order
//                    and the final selection bitmap.
// The candidate list is sized for every key of a head, so it cannot overflow.
#include "mra_internal.cuh"
#include "mra_select_common.cuh"

namespace mra {
namespace {

constexpr int kScanWarps = 8;
constexpr int kShift0 = kHist1Bits + kHist2Bits;

// One warp per block row, in groups of kScanChunks 32-column chunks: all of a
// group's loads are issued before any is used, the group's keys stay in
// registers, and one atomic per group reserves its candidates' slots.
constexpr int kScanChunks = 16;

__global__ void __launch_bounds__(32 * kScanWarps)
select_scan_kernel(const unsigned long long *__restrict__ keys, const SelState *__restrict__ state, int nbr,
                   long long nbr2, int rows, int wpr, unsigned int *__restrict__ bitmap,
                   unsigned int *__restrict__ tiebits, int *__restrict__ above_cnt,
                   unsigned long long *__restrict__ cand_key, int *__restrict__ cand_idx,
                   int *__restrict__ ccount) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kScanWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int bh = row / nbr, r = row - bh * nbr;
    const unsigned long long b0 = state[bh].prefix >> kShift0;   // the bucket's first digit
    const unsigned long long *kr = keys + (size_t)bh * nbr2 + (size_t)r * nbr;
    unsigned long long *ck = cand_key + (size_t)bh * nbr2;
    int *ci = cand_idx + (size_t)bh * nbr2;
    const unsigned int lt_mask = (1u << lane) - 1u;
    int nabove = 0;
    for (int g0 = 0; g0 < nbr; g0 += 32 * kScanChunks) {
        unsigned long long kv[kScanChunks];
#pragma unroll
        for (int j = 0; j < kScanChunks; ++j) {
            const int c = g0 + 32 * j + lane;
            kv[j] = c < nbr ? __ldcg(kr + c) : 0ull;
        }
        unsigned int inb[kScanChunks];
        int ncand = 0;
#pragma unroll
        for (int j = 0; j < kScanChunks; ++j) {
            const int c0 = g0 + 32 * j;
            const int c = c0 + lane;
            const unsigned long long d0 = kv[j] >> kShift0;
            const unsigned int above = __ballot_sync(0xffffffffu, c < nbr && d0 > b0);
            inb[j] = __ballot_sync(0xffffffffu, c < nbr && d0 == b0);
            if (lane == 0 && c0 < nbr) {
                bitmap[(size_t)row * wpr + (c0 >> 5)] = above;
                tiebits[(size_t)row * wpr + (c0 >> 5)] = 0u;
            }
            ncand += __popc(inb[j]);
            nabove += __popc(above);
        }
        if (ncand == 0) continue;
        int base = 0;
        if (lane == 0) base = atomicAdd(&ccount[bh], ncand);
        base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
        for (int j = 0; j < kScanChunks; ++j) {
            if ((inb[j] >> lane) & 1u) {
                const int pos = base + __popc(inb[j] & lt_mask);
                ck[pos] = kv[j];
                ci[pos] = r * nbr + g0 + 32 * j + lane;
            }
            base += __popc(inb[j]);
        }
    }
    if (lane == 0) above_cnt[row] = nabove;
}

constexpr int kFinThreads = 1024;
constexpr int kFinWarps = kFinThreads / 32;
constexpr int kFinStage = 4096;   // candidates kept in shared memory (the rest are read from L2)

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
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;   // inclusive prefix of the warp totals
    }
    __syncthreads();
    const int before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    *total = s_warp[kFinWarps - 1];
    __syncthreads();
    return before;
}

// Exclusive prefix of v over the lanes of a warp; *total gets the warp's sum.
__device__ __forceinline__ int warp_exclusive(int v, int lane, int *total) {
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    *total = __shfl_sync(0xffffffffu, x, 31);
    return x - v;
}

// One CTA per (batch, head).
__global__ void __launch_bounds__(kFinThreads)
select_finalize_kernel(SelState *__restrict__ state, const unsigned long long *__restrict__ cand_key,
                       const int *__restrict__ cand_idx, const int *__restrict__ ccount,
                       const int *__restrict__ above_cnt, int nbr, long long nbr2, int wpr, int k, int cap,
                       int chunk, unsigned int *__restrict__ bitmap, unsigned int *__restrict__ tiebits,
                       int *__restrict__ row_start, int *__restrict__ row_take, WorkItem *__restrict__ items,
                       int *__restrict__ head_items, unsigned int *__restrict__ status) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned long long fin_smem[];
    unsigned long long *s_ck = fin_smem;                                           // [kFinStage] candidate keys
    int *s_ci = reinterpret_cast<int *>(s_ck + kFinStage);                          // [kFinStage] their indices
    unsigned int *h = reinterpret_cast<unsigned int *>(s_ci + kFinStage);          // [kHistBins]
    int *s_gt = reinterpret_cast<int *>(h + kHistBins);                             // [nbr] keys above T per row
    int *s_eq = s_gt + nbr;                                                         // [nbr] keys equal to T per row
    __shared__ unsigned int s_tmp[kFinThreads];
    __shared__ int s_warp[32];
    __shared__ int s_bin;
    __shared__ unsigned int s_need;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int bh = blockIdx.x;
    const int n = ccount[bh];
    const unsigned long long *gck = cand_key + (size_t)bh * nbr2;
    const int *gci = cand_idx + (size_t)bh * nbr2;
    unsigned long long prefix = state[bh].prefix;
    unsigned int need = state[bh].need;
    int sh = kShift0;
    // the row counts of the scan and the candidates, all loads issued at once
    for (int r = t; r < nbr; r += kFinThreads) {
        s_gt[r] = __ldcg(above_cnt + (size_t)bh * nbr + r);
        s_eq[r] = 0;
    }
    for (int i = t; i < min(n, kFinStage); i += kFinThreads) {
        s_ck[i] = __ldcg(gck + i);
        s_ci[i] = __ldcg(gci + i);
    }
    __syncthreads();
    auto cand_key_at = [&](int i) { return i < kFinStage ? s_ck[i] : __ldcg(gck + i); };
    auto cand_idx_at = [&](int i) { return i < kFinStage ? s_ci[i] : __ldcg(gci + i); };
    // the two lower digits over the candidates (every candidate matches the
    // first digit); a digit whose bucket is taken whole ends the search
    for (int pass = 1; pass <= 2; ++pass) {
        const int shift = pass == 1 ? kHist2Bits : 0;
        const int hi = shift + 12;
        const unsigned long long want = prefix >> hi;
        for (int i = t; i < kHistBins; i += kFinThreads) h[i] = 0u;
        __syncthreads();
        for (int i0 = warp * 32; i0 < n; i0 += kFinThreads) {
            const int i = i0 + lane;
            const unsigned long long key = i < n ? cand_key_at(i) : ~0ull;
            hist_add(h, (unsigned)(key >> shift) & 0xfffu, i < n && (key >> hi) == want);
        }
        __syncthreads();
        find_bucket_smem<kFinThreads, kHistBins>(h, need, s_tmp, &s_bin, &s_need);
        const int bin = s_bin;
        const unsigned int bneed = s_need;
        const bool whole = bneed == h[bin];
        prefix |= (unsigned long long)bin << shift;
        need = bneed;
        sh = shift;
        __syncthreads();   // h[bin] read everywhere before the next clear
        if (whole) break;
    }
    const unsigned long long Tsh = prefix >> sh;
    if (t == 0) {
        SelState ns;
        ns.prefix = prefix;
        ns.need = need;
        ns.pad = (unsigned)sh;
        state[bh] = ns;
    }
    // per row: the certain selections counted by the scan, then the
    // candidates above T (into the bitmap) and at T (into the tie bitmap,
    // cleared by the scan)
    unsigned int *bm = bitmap + (size_t)bh * nbr * wpr;
    unsigned int *tb = tiebits + (size_t)bh * nbr * wpr;
    for (int i = t; i < n; i += kFinThreads) {
        const unsigned long long kk = cand_key_at(i) >> sh;
        const int idx = cand_idx_at(i);
        const int r = idx / nbr, c = idx - r * nbr;
        if (kk > Tsh) {
            atomicOr(&bm[r * wpr + (c >> 5)], 1u << (c & 31));
            atomicAdd(&s_gt[r], 1);
        } else if (kk == Tsh) {
            atomicOr(&tb[r * wpr + (c >> 5)], 1u << (c & 31));
            atomicAdd(&s_eq[r], 1);
        }
    }
    __syncthreads();
    // rows in order: the ties go to the first rows until need is met; CSR
    // offsets and work items (chunks of at most `chunk` columns)
    const int per = (nbr + kFinThreads - 1) / kFinThreads;   // rows per thread (<= 2)
    const int rbeg = min(t * per, nbr), rend = min(rbeg + per, nbr);
    int eq_local = 0;
    for (int r = rbeg; r < rend; ++r) eq_local += s_eq[r];
    int tot;
    int eq_before = block_exclusive_scan(eq_local, s_warp, &tot);
    int sel[2] = {0, 0};
    int sel_local = 0, it_local = 0;
    for (int r = rbeg, i = 0; r < rend; ++r, ++i) {
        const int e = s_eq[r];
        int take = (int)need - eq_before;
        take = take < 0 ? 0 : (take > e ? e : take);
        row_take[(size_t)bh * nbr + r] = take;
        sel[i] = s_gt[r] + take;
        sel_local += sel[i];
        it_local += sel[i] > 0 ? (sel[i] + chunk - 1) / chunk : 1;
        eq_before += e;
    }
    int sel_total, it_total;
    int sel_before = block_exclusive_scan(sel_local, s_warp, &sel_total);
    int it_before = block_exclusive_scan(it_local, s_warp, &it_total);
    const bool ok = sel_total == k && it_total <= cap;
    if (t == 0) {
        // a head whose selection does not add up to k is skipped (never read
        // out of bounds) and flagged in the status word
        head_items[bh] = ok ? it_total : 0;
        if (!ok) atomicOr(status, kDevCount);
    }
    if (!ok) return;   // uniform over the CTA
    for (int r = rbeg, i = 0; r < rend; ++r, ++i) {
        const int rs = bh * k + sel_before;
        row_start[(size_t)bh * nbr + r] = rs;
        const int nit = sel[i] > 0 ? (sel[i] + chunk - 1) / chunk : 1;
        for (int j = 0; j < nit; ++j) {
            WorkItem w;
            w.row = bh * nbr + r;
            w.col_start = rs + j * chunk;
            w.ncols = max(0, min(chunk, sel[i] - j * chunk));
            w.chunk_info = j | (nit << 16);
            items[(size_t)bh * cap + it_before + j] = w;
        }
        sel_before += sel[i];
        it_before += nit;
    }
}

// Column lists: one warp per block row, lane per bitmap word, ascending
// columns; the row's first row_take ties (in column order) are taken, and the
// final selection bitmap is written back.
__global__ void __launch_bounds__(32 * kScanWarps)
select_cols_kernel(const int *__restrict__ row_start, const int *__restrict__ row_take,
                   const int *__restrict__ head_items, int nbr, int rows, int wpr,
                   unsigned int *__restrict__ bitmap, const unsigned int *__restrict__ tiebits,
                   int *__restrict__ cols, int32_t *__restrict__ sel_out) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kScanWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int bh = row / nbr, r = row - bh * nbr;
    if (head_items[bh] == 0) return;   // the head's selection failed its count check
    const int take = row_take[row];
    const int rs = row_start[row];
    int sel_seen = 0, tie_seen = 0;
    for (int w0 = 0; w0 < wpr; w0 += 32) {
        const int w = w0 + lane;
        const unsigned int a = w < wpr ? __ldcg(&bitmap[(size_t)row * wpr + w]) : 0u;
        const unsigned int tie = w < wpr ? __ldcg(&tiebits[(size_t)row * wpr + w]) : 0u;
        int tie_tot;
        const int tie_before = tie_seen + warp_exclusive(__popc(tie), lane, &tie_tot);
        int room = take - tie_before;
        room = room < 0 ? 0 : (room > __popc(tie) ? __popc(tie) : room);
        unsigned int chosen = 0u, x = tie;
        for (int j = 0; j < room; ++j) {
            chosen |= x & (0u - x);
            x &= x - 1u;
        }
        const unsigned int fin = a | chosen;
        if (w < wpr) bitmap[(size_t)row * wpr + w] = fin;
        int fin_tot;
        int pos = rs + sel_seen + warp_exclusive(__popc(fin), lane, &fin_tot);
        for (unsigned int y = fin; y; y &= y - 1u) {
            const int c = w * 32 + __ffs(y) - 1;
            cols[pos] = c;
            if (sel_out) sel_out[pos] = r * nbr + c;
            ++pos;
        }
        sel_seen += fin_tot;
        tie_seen += tie_tot;
    }
}

}  // namespace

cudaError_t launch_select_scan(const Problem &p, const Workspace &w, cudaStream_t s) {
    const int rows = p.BH * p.nbr;
    const int grid = (rows + kScanWarps - 1) / kScanWarps;
    return launch_dependent(select_scan_kernel, dim3(grid), dim3(32 * kScanWarps), 0, s,
                            (const unsigned long long *)w.keys, (const SelState *)w.state, p.nbr, p.nbr2, rows,
                            w.words_per_row, w.bitmap, w.tiebits, w.above_cnt, w.cand_key, w.cand_idx, w.ccount);
}

cudaError_t launch_select_finalize(const Problem &p, const Workspace &w, int32_t *sel_out, cudaStream_t s) {
    const size_t smem = (sizeof(unsigned long long) + sizeof(int)) * kFinStage +
                        sizeof(int) * ((size_t)kHistBins + 2 * (size_t)p.nbr);
    cudaError_t e = cudaFuncSetAttribute(select_finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_dependent(select_finalize_kernel, dim3(p.BH), dim3(kFinThreads), smem, s, w.state,
                         (const unsigned long long *)w.cand_key, (const int *)w.cand_idx, (const int *)w.ccount,
                         (const int *)w.above_cnt, p.nbr, p.nbr2, w.words_per_row, p.k, p.cap, p.chunk, w.bitmap,
                         w.tiebits, w.row_start, w.row_take, w.items, w.head_items, w.status);
    if (e != cudaSuccess) return e;
    const int rows = p.BH * p.nbr;
    const int grid = (rows + kScanWarps - 1) / kScanWarps;
    return launch_dependent(select_cols_kernel, dim3(grid), dim3(32 * kScanWarps), 0, s, (const int *)w.row_start,
                            (const int *)w.row_take, (const int *)w.head_items, p.nbr, rows, w.words_per_row,
                            w.bitmap, (const unsigned int *)w.tiebits, w.cols, sel_out);
}

}  // namespace mra
