// mra_lowres_select.cu - low-resolution logits, selection keys and the whole
// global top-k selection in ONE kernel, for maps of up to 128 x 128 blocks.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理":
//   step one - the small full matmul of the pooled Q and K (block-logit map),
//              empty blocks pushed down in their rows and columns;
//   step two - a global top-k over the map with the 5e3 prior biases,
//              returning the selected block coordinates.
//
// One thread-block cluster per (batch, head): each CTA computes 16 block rows
// of the map (fp32 FFMA, 2x4 register tiles), keeps their 35-bit keys in
// shared memory, and the cluster runs the three radix passes of the top-k
// together: every CTA adds its histogram of a pass into every CTA's copy of
// the cluster histogram through distributed shared memory, so after one
// cluster barrier each CTA locates the bucket of the k-th key on its own; a
// pass whose bucket is taken whole ends the search.  Cluster barriers
// (hardware barriers, no spinning) separate the steps.  The per-row counts
// (pushed to every CTA the same way), the scan that assigns CSR offsets and
// attention work items across the cluster, and the column lists follow in
// the same kernel.  The key encoding and the tie rule are those of the
// multi-kernel path (mra_lowres.cu, mra_select.cu).
#include <cooperative_groups.h>

#include "mra_internal.cuh"
#include "mra_select_common.cuh"

namespace cg = cooperative_groups;

namespace mra {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 16;                 // block rows per CTA
constexpr int kCT = 128;                  // columns of the map (at most)
constexpr int kCPT = kCT / 32;            // columns per lane in the per-row passes (4), strided by 32
constexpr int kMaxCta = 8;                // portable cluster size
constexpr int kHistBits12 = 12;           // the two lower digits
constexpr unsigned int kMask12 = (1u << kHistBits12) - 1u;
static_assert(kHist1Bits == kHistBits12 && kHist2Bits == kHistBits12, "lower digits are 12 bits");

// Row stride of the K-hat tile in shared memory: D + 4 floats keeps rows
// 16-byte aligned and puts the rows read by 8 consecutive lanes in distinct
// bank groups.
template <int D>
constexpr int ks_stride() { return D + 4; }

// Keys of the k-th key's first-digit bucket that rank 0 gathers to finish
// the selection on its own.
constexpr int kCand = 4096;

// Words of the region that holds the K-hat tile during the GEMM and, after
// it, the cluster histogram of the first digit (2048 words) followed by
// either the gathered keys (kCand 64-bit keys) or the cluster histograms of
// the two lower digits (2 x 4096 words).
constexpr int kSelWords = (1 << kHist0Bits) + 2 * kHistBins;
static_assert(2 * kCand <= 2 * kHistBins, "gathered keys share the lower-digit histograms' words");
template <int D>
__host__ __device__ constexpr int region_floats() {
    return ks_stride<D>() * kCT > kSelWords ? ks_stride<D>() * kCT : kSelWords;
}

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

struct ClusterShared {
    unsigned int lh[kHistBins];     // this CTA's histogram of the current pass
    unsigned int s_tot[kWarps];
    int bin;
    unsigned int bin_need;
    int cand_n;                     // rank 0: keys gathered so far
    int small_n;                    // rank 0: keys of a bucket of at most 32
    unsigned long long small[32];
    unsigned long long pub_prefix;  // threshold published by rank 0
    unsigned int pub_need;
    int pub_sh;
    int all_gt[kMaxCta * kRows], all_eq[kMaxCta * kRows];   // per-row counts of the whole head
    int row_take[kRows], row_start[kRows], row_item[kRows], row_sel[kRows];
    int total_sel, total_items;
    int flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads)
lowres_select_cluster_kernel(const float *__restrict__ qhat, const float *__restrict__ khat,
                             const int *__restrict__ cnt, int H, int nbr, float scale, int first_n,
                             int diag_n, int k, int cap, int chunk,
                             float *__restrict__ mlo, float *__restrict__ logit_out,
                             int *__restrict__ cols, int32_t *__restrict__ sel_out,
                             unsigned int *__restrict__ bitmap, int wpr, WorkItem *__restrict__ items,
                             int *__restrict__ head_items, SelState *__restrict__ state,
                             unsigned int *__restrict__ status) {
    pdl_wait();
    constexpr int KS = ks_stride<D>();
    constexpr int kF4 = D / 4;   // float4 per row of Q-hat / K-hat
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int ncta = (int)cluster.num_blocks();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *qs = reinterpret_cast<float *>(smem_raw);                     // [kRows][D]
    float *ks = qs + kRows * D;                                           // [kCT][KS]
    float *lt = ks + region_floats<D>();                                  // [kRows][nbr]
    unsigned long long *sk = reinterpret_cast<unsigned long long *>(lt + kRows * nbr);  // [kRows][nbr]
    int *cnts = reinterpret_cast<int *>(sk + kRows * nbr);                // [nbr]
    __shared__ ClusterShared cs;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int r0 = rank * kRows;
    const int rows_here = max(0, min(kRows, nbr - r0));
    const long long nbr2 = (long long)nbr * nbr;
    const float *qh = qhat + (size_t)bh * nbr * D;
    const float *kh = khat + (size_t)bh * nbr * D;

    for (int i = t; i < kHistBins; i += kThreads) cs.lh[i] = 0u;
    if (t == 0) {
        cs.flag = 0;
        cs.cand_n = 0;
    }
    // ------------------------------------------------------------ logits
    {
        constexpr int kQ = (kRows * kF4 + kThreads - 1) / kThreads;
        constexpr int kK = (kCT * kF4 + kThreads - 1) / kThreads;
        float4 qv[kQ], kv[kK];
        int cv[(kCT + kThreads - 1) / kThreads];
        // all loads first (coalesced rows), then the shared-memory stores
#pragma unroll
        for (int u = 0; u < kQ; ++u) {
            const int i = t + u * kThreads;
            const int r = i / kF4;
            qv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < kRows * kF4 && r < rows_here)
                qv[u] = reinterpret_cast<const float4 *>(qh + (size_t)(r0 + r) * D)[i % kF4];
        }
#pragma unroll
        for (int u = 0; u < kK; ++u) {
            const int i = t + u * kThreads;
            kv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < nbr * kF4) kv[u] = reinterpret_cast<const float4 *>(kh)[i];
        }
#pragma unroll
        for (int u = 0; u < (int)(sizeof(cv) / sizeof(int)); ++u) {
            const int c = t + u * kThreads;
            cv[u] = c < nbr ? cnt[(size_t)b * nbr + c] : 0;
        }
#pragma unroll
        for (int u = 0; u < kQ; ++u) {
            const int i = t + u * kThreads;
            if (i < kRows * kF4) reinterpret_cast<float4 *>(qs)[i] = qv[u];
        }
#pragma unroll
        for (int u = 0; u < kK; ++u) {
            const int i = t + u * kThreads;
            if (i < kCT * kF4) *reinterpret_cast<float4 *>(ks + (i / kF4) * KS + 4 * (i % kF4)) = kv[u];
        }
#pragma unroll
        for (int u = 0; u < (int)(sizeof(cv) / sizeof(int)); ++u) {
            const int c = t + u * kThreads;
            if (c < nbr) cnts[c] = cv[u];
        }
    }
    __syncthreads();
    {
        // thread tile: one column c of the map (its K-hat row in registers)
        // and kRPT rows (Q-hat read as loads that every lane of the warp
        // shares); the sum over d runs in the same order as a plain dot
        // product
        constexpr int kHalves = kThreads / kCT;
        constexpr int kRPT = kRows / kHalves;
        const int c = t % kCT, half = t / kCT;
        if (c < nbr) {
            float4 kr[kF4];
#pragma unroll
            for (int d4 = 0; d4 < kF4; ++d4) kr[d4] = *reinterpret_cast<const float4 *>(ks + c * KS + 4 * d4);
            float acc[kRPT];
#pragma unroll
            for (int i = 0; i < kRPT; ++i) acc[i] = 0.0f;
#pragma unroll
            for (int d4 = 0; d4 < kF4; ++d4) {
#pragma unroll
                for (int i = 0; i < kRPT; ++i) {
                    const float4 q4 = *reinterpret_cast<const float4 *>(qs + (kRPT * half + i) * D + 4 * d4);
                    acc[i] = fmaf(q4.x, kr[d4].x, acc[i]);
                    acc[i] = fmaf(q4.y, kr[d4].y, acc[i]);
                    acc[i] = fmaf(q4.z, kr[d4].z, acc[i]);
                    acc[i] = fmaf(q4.w, kr[d4].w, acc[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < kRPT; ++i) lt[(kRPT * half + i) * nbr + c] = acc[i] * scale;
        }
    }
    __syncthreads();
    // the K-hat tile is dead: it becomes the cluster histograms, cleared
    // before this CTA's arrival at the cluster barrier that every CTA waits on
    // before adding into another CTA's histograms
    unsigned int *hist0 = reinterpret_cast<unsigned int *>(ks);
    for (int i = t; i < kSelWords / 4; i += kThreads)
        reinterpret_cast<uint4 *>(hist0)[i] = make_uint4(0u, 0u, 0u, 0u);
    cluster_arrive();

    // ------------------------------------------------------------ row max, keys, pass-0 histogram
    // one warp per row; lane owns columns lane + 32*j
    {
        int flag = 0;
        for (int rr = warp; rr < kRows; rr += kWarps) {
            const bool row_ok = rr < rows_here;   // warp-uniform
            const int gr = r0 + rr;
            float lv[kCPT];
            float m = -INFINITY;
#pragma unroll
            for (int j = 0; j < kCPT; ++j) {
                const int c = lane + 32 * j;
                const bool ok = row_ok && c < nbr;
                lv[j] = ok ? lt[rr * nbr + c] : 0.0f;
                if (ok && cnts[c] > 0) m = fmaxf(m, lv[j]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (m == -INFINITY) m = 0.0f;
            if (row_ok && lane == 0) mlo[(size_t)bh * nbr + gr] = m;
            const int row_empty = row_ok && cnts[min(gr, nbr - 1)] <= 0;
#pragma unroll
            for (int j = 0; j < kCPT; ++j) {
                const int c = lane + 32 * j;
                const bool ok = row_ok && c < nbr;
                unsigned long long key = 0ull;
                if (ok) {
                    key = selection_key(lv[j], m, gr, c, first_n, diag_n, row_empty, cnts[c] <= 0, flag);
                    sk[rr * nbr + c] = key;
                    const size_t gi = (size_t)bh * nbr2 + (size_t)gr * nbr + c;
                    if (logit_out) logit_out[gi] = lv[j];
                }
                hist_add(cs.lh, (unsigned)(key >> (kHist1Bits + kHist2Bits)) & ((1u << kHist0Bits) - 1u), ok);
            }
        }
        if (flag) atomicOr(&cs.flag, 1);
    }
    __syncthreads();
    if (t == 0 && cs.flag) atomicOr(status, kDevKeyRange);
    cluster_wait();   // every CTA's histograms are clear

    // ------------------------------------------------------------ radix select
    // First digit: every CTA adds its histogram into every CTA's copy of the
    // cluster histogram, so after one cluster barrier each CTA locates the
    // bucket of the k-th key on its own (same sums, same result everywhere).
    // If the bucket is not taken whole, its keys (usually a few hundred) are
    // gathered into rank 0, which resolves the two lower digits alone and
    // publishes the threshold; a bucket too large to gather takes the lower
    // digits through cluster histograms like the first.  A digit whose bucket
    // is taken whole ends the search: the threshold is then compared at that
    // digit's bit.
    const int n_here = rows_here * nbr;
    const unsigned int lt_mask = (1u << lane) - 1u;
    auto push_hist = [&](unsigned int *hp, int nbins) {
        for (int i = t; i < nbins; i += kThreads) {
            const unsigned int v = cs.lh[i];
            if (v) {
                for (int j = 0; j < ncta; ++j) {
                    int dst = rank + j;
                    if (dst >= ncta) dst -= ncta;
                    atomicAdd(cluster.map_shared_rank(hp, dst) + i, v);
                }
                cs.lh[i] = 0u;
            }
        }
    };
    constexpr int kShift0 = kHist1Bits + kHist2Bits;
    push_hist(hist0, 1 << kHist0Bits);
    cluster.sync();   // the first digit's cluster histogram is complete in every CTA
    find_bucket_smem<kThreads, 1 << kHist0Bits>(hist0, (unsigned)k, cs.s_tot, &cs.bin, &cs.bin_need);
    unsigned long long prefix = (unsigned long long)cs.bin << kShift0;
    unsigned int need = cs.bin_need;
    int sh = kShift0;
    const unsigned int in_bin0 = hist0[cs.bin];
    if (need != in_bin0) {
        if (in_bin0 <= (unsigned)kCand) {
            unsigned long long *cand = reinterpret_cast<unsigned long long *>(hist0 + (1 << kHist0Bits));
            unsigned long long *cand0 = cluster.map_shared_rank(cand, 0);
            int *cand_n0 = cluster.map_shared_rank(&cs.cand_n, 0);
            const unsigned long long want0 = prefix >> kShift0;
            // one remote atomic per warp reserves the warp's slots
            int nmine = 0;
            for (int e0 = warp * 32; e0 < n_here; e0 += kThreads) {
                const int e = e0 + lane;
                nmine += __popc(__ballot_sync(0xffffffffu, e < n_here && (sk[min(e, n_here - 1)] >> kShift0) == want0));
            }
            if (nmine) {
                int base = 0;
                if (lane == 0) base = atomicAdd(cand_n0, nmine);
                base = __shfl_sync(0xffffffffu, base, 0);
                for (int e0 = warp * 32; e0 < n_here; e0 += kThreads) {
                    const int e = e0 + lane;
                    const unsigned long long key = e < n_here ? sk[e] : 0ull;
                    const bool m = e < n_here && (key >> kShift0) == want0;
                    const unsigned int bal = __ballot_sync(0xffffffffu, m);
                    if (m) cand0[base + __popc(bal & lt_mask)] = key;
                    base += __popc(bal);
                }
            }
            cluster.sync();   // rank 0 holds the bucket's keys
            if (rank == 0) {
                const int n = (int)in_bin0;
                for (int pass = 1; pass < 3; ++pass) {
                    const int shift = pass == 1 ? kHist2Bits : 0;
                    const int hi = shift + kHistBits12;
                    const unsigned long long want = prefix >> hi;
                    for (int e0 = warp * 32; e0 < n; e0 += kThreads) {
                        const int e = e0 + lane;
                        const unsigned long long key = e < n ? cand[e] : ~0ull;
                        hist_add(cs.lh, (unsigned)(key >> shift) & kMask12, e < n && (key >> hi) == want);
                    }
                    __syncthreads();
                    find_bucket_smem<kThreads, kHistBins>(cs.lh, need, cs.s_tot, &cs.bin, &cs.bin_need);
                    const int bin = cs.bin;
                    const unsigned int bin_need = cs.bin_need;
                    const unsigned int in_bin = cs.lh[bin];
                    prefix |= (unsigned long long)bin << shift;
                    need = bin_need;
                    sh = shift;
                    __syncthreads();   // lh[bin] read everywhere
                    for (int i = t; i < kHistBins; i += kThreads) cs.lh[i] = 0u;
                    if (bin_need == in_bin) break;   // bucket taken whole
                    if (pass == 1 && in_bin <= 32u) {
                        // at most 32 keys share the top 23 bits: warp 0 finds the
                        // need-th largest of them by counting, at full precision
                        if (t == 0) cs.small_n = 0;
                        __syncthreads();
                        const unsigned long long want1 = prefix >> kHist2Bits;
                        for (int e0 = warp * 32; e0 < n; e0 += kThreads) {
                            const int e = e0 + lane;
                            const unsigned long long key = e < n ? cand[e] : 0ull;
                            const bool m = e < n && (key >> kHist2Bits) == want1;
                            const unsigned int bal = __ballot_sync(0xffffffffu, m);
                            int base = 0;
                            if (bal && lane == 0) base = atomicAdd(&cs.small_n, __popc(bal));
                            base = __shfl_sync(0xffffffffu, base, 0);
                            if (m) cs.small[base + __popc(bal & lt_mask)] = key;
                        }
                        __syncthreads();
                        if (warp == 0) {
                            const bool valid = lane < (int)in_bin;
                            const unsigned long long mine = valid ? cs.small[lane] : 0ull;
                            int gt = 0, ge = 0;
                            for (int j = 0; j < (int)in_bin; ++j) {
                                const unsigned long long kj = __shfl_sync(0xffffffffu, mine, j);
                                gt += kj > mine;
                                ge += kj >= mine;
                            }
                            if (valid && gt < (int)need && (int)need <= ge) {
                                cs.pub_prefix = mine;   // equal keys write the same values
                                cs.pub_need = need - (unsigned)gt;
                            }
                        }
                        __syncthreads();
                        prefix = cs.pub_prefix;
                        need = cs.pub_need;
                        sh = 0;
                        break;
                    }
                    __syncthreads();   // lh cleared before the next pass adds
                }
                if (t < ncta) {
                    ClusterShared *dst = cluster.map_shared_rank(&cs, t);
                    dst->pub_prefix = prefix;
                    dst->pub_need = need;
                    dst->pub_sh = sh;
                }
            }
            cluster.sync();   // every CTA holds the threshold
            prefix = cs.pub_prefix;
            need = cs.pub_need;
            sh = cs.pub_sh;
        } else {
            for (int pass = 1; pass < 3; ++pass) {
                const int shift = pass == 1 ? kHist2Bits : 0;
                const int bits = pass == 1 ? kHist1Bits : kHist2Bits;
                const int hi = shift + bits;
                const unsigned long long want = prefix >> hi;
                const unsigned int dmask = (1u << bits) - 1u;
                for (int e0 = warp * 32; e0 < n_here; e0 += kThreads) {
                    const int e = e0 + lane;
                    const unsigned long long key = e < n_here ? sk[e] : ~0ull;
                    hist_add(cs.lh, (unsigned)(key >> shift) & dmask, e < n_here && (key >> hi) == want);
                }
                __syncthreads();
                unsigned int *hp = hist0 + (1 << kHist0Bits) + (pass - 1) * kHistBins;
                push_hist(hp, 1 << bits);
                cluster.sync();   // this digit's cluster histogram is complete in every CTA
                find_bucket_smem<kThreads, kHistBins>(hp, need, cs.s_tot, &cs.bin, &cs.bin_need);
                const int bin = cs.bin;
                const unsigned int bin_need = cs.bin_need;
                const bool whole = bin_need == hp[bin];
                prefix |= (unsigned long long)bin << shift;
                need = bin_need;
                sh = shift;
                if (whole) break;
            }
        }
    }
    const unsigned long long Tsh = prefix >> sh;
    if (rank == 0 && t == 0) {
        SelState st;
        st.prefix = prefix;
        st.need = need;
        st.pad = (unsigned)sh;
        state[bh] = st;
    }

    // ------------------------------------------------------------ per-row counts and scans
    // each row's (above, at) threshold counts go to every CTA of the cluster
    for (int rr = warp; rr < kRows; rr += kWarps) {
        int g = 0, e = 0;
        if (rr < rows_here)
#pragma unroll
            for (int j = 0; j < kCPT; ++j) {
                const int c = lane + 32 * j;
                if (c < nbr) {
                    const unsigned long long kk = sk[rr * nbr + c] >> sh;
                    g += kk > Tsh;
                    e += kk == Tsh;
                }
            }
        g = __reduce_add_sync(0xffffffffu, g);
        e = __reduce_add_sync(0xffffffffu, e);
        if (rr < rows_here && lane < ncta) {
            cluster.map_shared_rank(cs.all_gt, lane)[r0 + rr] = g;
            cluster.map_shared_rank(cs.all_eq, lane)[r0 + rr] = e;
        }
    }
    cluster.sync();   // every row's counts are in every CTA; no remote access after this
    // every CTA scans all rows of the head (warp 0, four rows per lane) and
    // keeps what concerns its own rows
    if (warp == 0) {
        constexpr int kPer = (kMaxCta * kRows) / 32;
        int eqv[kPer], gtv[kPer];
        int eq_local = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int r = kPer * lane + j;
            eqv[j] = r < nbr ? cs.all_eq[r] : 0;
            gtv[j] = r < nbr ? cs.all_gt[r] : 0;
            eq_local += eqv[j];
        }
        int x = eq_local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        int eq_before = x - eq_local;
        int sel[kPer], itm[kPer], tk[kPer];
        int sel_local = 0, it_local = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int r = kPer * lane + j;
            int take = (int)need - eq_before;
            take = take < 0 ? 0 : (take > eqv[j] ? eqv[j] : take);
            tk[j] = take;
            sel[j] = r < nbr ? gtv[j] + take : 0;
            itm[j] = r < nbr ? (sel[j] > 0 ? (sel[j] + chunk - 1) / chunk : 1) : 0;
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
        for (int j = 0; j < kPer; ++j) {
            const int r = kPer * lane + j;
            if (r >= r0 && r < r0 + rows_here) {
                cs.row_take[r - r0] = tk[j];
                cs.row_sel[r - r0] = sel[j];
                cs.row_start[r - r0] = sb;
                cs.row_item[r - r0] = ib;
            }
            sb += sel[j];
            ib += itm[j];
        }
        if (lane == 31) {
            cs.total_sel = xs;
            cs.total_items = xi;
        }
    }
    __syncthreads();
    const bool ok = cs.total_sel == k && cs.total_items <= cap;
    if (rank == 0 && t == 0) {
        head_items[bh] = ok ? cs.total_items : 0;
        if (!ok) atomicOr(status, kDevCount);
    }
    if (!ok) return;
    // work items: one thread per local row
    for (int r = t; r < rows_here; r += kThreads) {
        const int sel = cs.row_sel[r];
        const int nit = sel > 0 ? (sel + chunk - 1) / chunk : 1;
        const int rs = bh * k + cs.row_start[r];
        for (int j = 0; j < nit; ++j) {
            WorkItem w;
            w.row = bh * nbr + r0 + r;
            w.col_start = rs + j * chunk;
            w.ncols = max(0, min(chunk, sel - j * chunk));
            w.chunk_info = j | (nit << 16);
            items[(size_t)bh * cap + cs.row_item[r] + j] = w;
        }
    }
    // column lists: one warp per local row, ascending columns
    for (int r = warp; r < rows_here; r += kWarps) {
        const int rs = bh * k + cs.row_start[r];
        const int take = cs.row_take[r];
        const int gr = r0 + r;
        int eq_seen = 0, sel_seen = 0;
        for (int c0 = 0; c0 < nbr; c0 += 32) {
            const int c = c0 + lane;
            const unsigned long long kk = c < nbr ? (sk[r * nbr + c] >> sh) : 0ull;
            const bool is_gt = c < nbr && kk > Tsh;
            const bool is_eq = c < nbr && kk == Tsh;
            const unsigned int eqb = __ballot_sync(0xffffffffu, is_eq);
            const bool sel = is_gt || (is_eq && eq_seen + __popc(eqb & lt_mask) < take);
            const unsigned int sb = __ballot_sync(0xffffffffu, sel);
            if (sel) {
                const int pos = rs + sel_seen + __popc(sb & lt_mask);
                cols[pos] = c;
                if (sel_out) sel_out[pos] = gr * nbr + c;
            }
            if (bitmap && lane == 0) bitmap[((size_t)bh * nbr + gr) * wpr + (c0 >> 5)] = sb;
            eq_seen += __popc(eqb);
            sel_seen += __popc(sb);
        }
    }
}

template <int D>
cudaError_t launch_typed(const Problem &p, const Workspace &w, float *logit_out, int32_t *sel_out,
                         cudaStream_t s) {
    const int ncta = (p.nbr + kRows - 1) / kRows;
    const size_t smem = sizeof(float) * ((size_t)kRows * D + (size_t)region_floats<D>() + (size_t)kRows * p.nbr) +
                        sizeof(unsigned long long) * (size_t)kRows * p.nbr + sizeof(int) * (size_t)p.nbr;
    auto kern = lowres_select_cluster_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ncta, p.BH, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ncta;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see launch_dependent
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const float scale = 1.0f / sqrtf((float)p.D);
    const float *qhat = w.pooled;
    const float *khat = w.pooled + (size_t)p.BH * p.nbr * p.D;
    // full mode keeps the logit map for the low-resolution part
    float *lmap = logit_out ? logit_out : (p.mode == 0 ? w.lo_logits : nullptr);
    e = cudaLaunchKernelEx(&cfg, kern, qhat, khat, (const int *)w.cnt, p.H, p.nbr, scale, p.first_n,
                           p.diag_n, p.k, p.cap, p.chunk, w.mlo, lmap, w.cols, sel_out,
                           p.mode == 0 ? w.bitmap : (unsigned int *)nullptr, w.words_per_row, w.items,
                           w.head_items, w.state, w.status);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

bool lowres_select_fused_supported(const Problem &p) {
    return p.nbr <= kMaxCta * kRows && p.nbr <= kCT;
}

cudaError_t launch_lowres_select_fused(const Problem &p, const Workspace &w, float *logit_out,
                                       int32_t *sel_out, cudaStream_t s) {
    return p.D == 64 ? launch_typed<64>(p, w, logit_out, sel_out, s)
                     : launch_typed<32>(p, w, logit_out, sel_out, s);
}

}  // namespace mra
