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
// together: local histograms are added into the rank-0 CTA's histogram of
// the pass through distributed shared memory, rank 0 locates the bucket of
// the k-th key and publishes it, and a pass whose bucket is taken whole ends
// the search.  Cluster barriers (hardware barriers, no spinning) separate the
// steps.  The per-row counts, the scan that
// assigns CSR offsets and attention work items across the cluster, and the
// column lists follow in the same kernel.  The key encoding and the tie rule
// are those of the multi-kernel path (mra_lowres.cu, mra_select.cu).
#include <cooperative_groups.h>

#include "mra_internal.cuh"
#include "mra_select_common.cuh"

namespace cg = cooperative_groups;

namespace mra {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 16;                 // block rows per CTA
constexpr int kRG = 8, kCG = 32;          // row groups x column groups
constexpr int kMR = kRows / kRG;          // rows per thread tile (2)
constexpr int kCT = 4 * kCG;              // columns per tile (128)
constexpr int kMaxCta = 8;                // portable cluster size

// Floats of the region that holds the transposed K-hat tile during the GEMM
// and the histograms of the first two radix passes afterwards.
template <int D>
constexpr int region_floats() { return D * kCT > 2 * kHistBins ? D * kCT : 2 * kHistBins; }

__device__ __forceinline__ int band_of(int r, int c, int g) {
    if (g <= 0) return 0;
    const int lo = -(g / 2);
    const int hi = (g + 1) / 2 - 1;
    const int off = c - r;
    return (off >= lo && off <= hi) ? 1 : 0;
}

struct ClusterShared {
    unsigned int hist2[kHistBins];  // rank 0: cluster histogram of the third pass
    unsigned int lh[kHistBins];     // this CTA's histogram
    unsigned int s_tmp[kThreads];
    int bin;
    unsigned int bin_need;
    unsigned long long pub_prefix;   // rank 0: result of the pass
    unsigned int pub_need;
    int pub_done;
    int all_gt[kMaxCta * kRows], all_eq[kMaxCta * kRows];   // rank 0: per-row counts of the head
    int row_take[kRows], row_start[kRows], row_item[kRows], row_sel[kRows];
    int total_sel, total_items;
    int flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads)
lowres_select_cluster_kernel(const float *__restrict__ qhat, const float *__restrict__ khat,
                             const int *__restrict__ cnt, int H, int nbr, float scale, int first_n,
                             int diag_n, int k, int cap, int chunk,
                             unsigned long long *__restrict__ keys_out,
                             float *__restrict__ mlo, float *__restrict__ logit_out,
                             int *__restrict__ cols, int32_t *__restrict__ sel_out,
                             unsigned int *__restrict__ bitmap, int wpr, WorkItem *__restrict__ items,
                             int *__restrict__ head_items, SelState *__restrict__ state,
                             unsigned int *__restrict__ status) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *qs = reinterpret_cast<float *>(smem_raw);                     // [kRows][D]
    float *kT = qs + kRows * D;                                           // [D][kCT]
    float *lt = kT + region_floats<D>();                                  // [kRows][nbr]
    unsigned long long *sk = reinterpret_cast<unsigned long long *>(lt + kRows * nbr);  // [kRows][nbr]
    int *cnts = reinterpret_cast<int *>(sk + kRows * nbr);                // [nbr]
    __shared__ ClusterShared cs;
    __shared__ float rmax[kRows];
    ClusterShared *cs0 = cluster.map_shared_rank(&cs, 0);

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int r0 = rank * kRows;
    const int rows_here = max(0, min(kRows, nbr - r0));
    const long long nbr2 = (long long)nbr * nbr;
    const float *qh = qhat + (size_t)bh * nbr * D;
    const float *kh = khat + (size_t)bh * nbr * D;

    if (rank == 0)
        for (int i = t; i < kHistBins; i += kThreads) cs.hist2[i] = 0u;
    if (t == 0) cs.flag = 0;
    // ------------------------------------------------------------ logits
    {
        constexpr int kQ = (kRows * D / 4 + kThreads - 1) / kThreads;
        float4 v[kQ];
        int cv[(kMaxCta * kRows + kThreads - 1) / kThreads];
#pragma unroll
        for (int u = 0; u < kQ; ++u) {
            const int i = t + u * kThreads;
            const int r = (4 * i) / D;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < kRows * D / 4 && r < rows_here)
                v[u] = reinterpret_cast<const float4 *>(qh + (size_t)(r0 + r) * D)[(4 * i) % D / 4];
        }
#pragma unroll
        for (int u = 0; u < (int)(sizeof(cv) / sizeof(int)); ++u) {
            const int c = t + u * kThreads;
            cv[u] = c < nbr ? cnt[(size_t)b * nbr + c] : 0;
        }
#pragma unroll
        for (int u = 0; u < kQ; ++u) {
            const int i = t + u * kThreads;
            if (i < kRows * D / 4) reinterpret_cast<float4 *>(qs)[i] = v[u];
        }
#pragma unroll
        for (int u = 0; u < (int)(sizeof(cv) / sizeof(int)); ++u) {
            const int c = t + u * kThreads;
            if (c < nbr) cnts[c] = cv[u];
        }
    }
    const int rg = t / kCG, cg_ = t % kCG;
    for (int ct = 0; ct < nbr; ct += kCT) {
        __syncthreads();
        {
            constexpr int kL = kCT * D / 4 / kThreads;
            float4 v[kL];
#pragma unroll
            for (int u = 0; u < kL; ++u) {
                const int e = t + u * kThreads;
                const int c = e % kCT, d4 = e / kCT;
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ct + c < nbr) v[u] = reinterpret_cast<const float4 *>(kh + (size_t)(ct + c) * D)[d4];
            }
#pragma unroll
            for (int u = 0; u < kL; ++u) {
                const int e = t + u * kThreads;
                const int c = e % kCT, d4 = e / kCT;
                kT[(4 * d4 + 0) * kCT + c] = v[u].x;
                kT[(4 * d4 + 1) * kCT + c] = v[u].y;
                kT[(4 * d4 + 2) * kCT + c] = v[u].z;
                kT[(4 * d4 + 3) * kCT + c] = v[u].w;
            }
        }
        __syncthreads();
        float acc[kMR][4];
#pragma unroll
        for (int i = 0; i < kMR; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
            float4 qv[kMR];
#pragma unroll
            for (int i = 0; i < kMR; ++i) qv[i] = *reinterpret_cast<const float4 *>(qs + (kMR * rg + i) * D + d);
#pragma unroll
            for (int dd = 0; dd < 4; ++dd) {
                const float4 kv = *reinterpret_cast<const float4 *>(kT + (d + dd) * kCT + 4 * cg_);
#pragma unroll
                for (int i = 0; i < kMR; ++i) {
                    const float qd = dd == 0 ? qv[i].x : dd == 1 ? qv[i].y : dd == 2 ? qv[i].z : qv[i].w;
                    acc[i][0] = fmaf(qd, kv.x, acc[i][0]);
                    acc[i][1] = fmaf(qd, kv.y, acc[i][1]);
                    acc[i][2] = fmaf(qd, kv.z, acc[i][2]);
                    acc[i][3] = fmaf(qd, kv.w, acc[i][3]);
                }
            }
        }
        const int c0 = ct + 4 * cg_;
#pragma unroll
        for (int i = 0; i < kMR; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (c0 + j < nbr) lt[(kMR * rg + i) * nbr + c0 + j] = acc[i][j] * scale;
    }
    __syncthreads();
    // row max over valid columns (0 when none)
    for (int r = warp; r < kRows; r += kThreads / 32) {
        float m = -INFINITY;
        for (int c = lane; c < nbr; c += 32)
            if (cnts[c] > 0) m = fmaxf(m, lt[r * nbr + c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (m == -INFINITY) m = 0.0f;
        if (lane == 0) {
            rmax[r] = m;
            if (r < rows_here) mlo[(size_t)bh * nbr + r0 + r] = m;
        }
    }
    __syncthreads();
    // keys (shared + global), exported logits
    const int n_here = rows_here * nbr;
    int flag = 0;
    for (int e = t; e < n_here; e += kThreads) {
        const int r = e / nbr, c = e - r * nbr;
        const int gr = r0 + r;
        const float l = lt[e];
        float x = l - rmax[r];
        if (x == 0.0f) x = 0.0f;   // canonical +0
        if (!(fabsf(x) < 2500.0f)) flag = 1;
        int tier = 0;
        if (first_n > 0 && (gr < first_n || c < first_n)) ++tier;
        tier += band_of(gr, c, diag_n);
        if (cnts[gr] <= 0) tier -= 2;
        if (cnts[c] <= 0) tier -= 2;
        const unsigned long long key =
            ((unsigned long long)(tier + 4) << 32) | (unsigned long long)float_order_bits(x);
        sk[e] = key;
        keys_out[(size_t)bh * nbr2 + (size_t)gr * nbr + c] = key;
        if (logit_out) logit_out[(size_t)bh * nbr2 + (size_t)gr * nbr + c] = l;
    }
    if (flag) atomicOr(&cs.flag, 1);
    // the histograms of the first two passes reuse the K-hat tile (rank 0's
    // copy is cleared here, before any CTA adds into it)
    unsigned int *hist01 = reinterpret_cast<unsigned int *>(kT);
    if (rank == 0)
        for (int i = t; i < 2 * kHistBins; i += kThreads) hist01[i] = 0u;
    cluster.sync();   // histograms clear; every CTA of the cluster is running
    if (t == 0 && cs.flag) atomicOr(status, kDevKeyRange);

    // ------------------------------------------------------------ radix passes
    // Every CTA adds its histogram into rank 0's buffer of the pass; rank 0
    // locates the bucket of the k-th key in its own shared memory and
    // publishes it.  A pass whose bucket is taken whole ends the search early:
    // the threshold is then compared at that digit's bit.
    unsigned int *hist_local[3] = {hist01, hist01 + kHistBins, cs.hist2};
    unsigned long long prefix = 0ull;
    unsigned int need = (unsigned)k;
    int sh = 0;            // comparisons against the threshold use key >> sh
    bool done = false;
    for (int pass = 0; pass < 3 && !done; ++pass) {
        const int shift = pass == 0 ? (kHist1Bits + kHist2Bits) : (pass == 1 ? kHist2Bits : 0);
        const int bits = pass == 0 ? kHist0Bits : (pass == 1 ? kHist1Bits : kHist2Bits);
        const int hi = shift + bits;
        const unsigned long long want = prefix >> hi;
        const unsigned int dmask = (1u << bits) - 1u;
        for (int i = t; i < (1 << bits); i += kThreads) cs.lh[i] = 0u;
        __syncthreads();
        for (int e0 = (t & ~31); e0 < n_here; e0 += kThreads) {
            const int e = e0 + lane;
            const unsigned long long key = e < n_here ? sk[e] : ~0ull;
            warp_hist_add(cs.lh, (unsigned)(key >> shift) & dmask, e < n_here && (key >> hi) == want);
        }
        __syncthreads();
        unsigned int *hb = cluster.map_shared_rank(hist_local[pass], 0);
        for (int i = t; i < (1 << bits); i += kThreads)
            if (cs.lh[i]) atomicAdd(&hb[i], cs.lh[i]);
        cluster.sync();   // the cluster histogram of this pass is complete
        if (rank == 0) {
            unsigned int *h = hist_local[pass];
            find_bucket<kThreads>([h](int i) { return h[i]; }, 1 << bits, need, cs.s_tmp, &cs.bin,
                                  &cs.bin_need);
            if (t == 0) {
                const unsigned int in_bin = h[cs.bin];
                cs.pub_prefix = prefix | ((unsigned long long)cs.bin << shift);
                cs.pub_done = (cs.bin_need == in_bin) ? 1 : 0;
                cs.pub_need = cs.bin_need;
            }
        }
        cluster.sync();   // rank 0 published the bucket
        prefix = cs0->pub_prefix;
        need = cs0->pub_need;
        done = cs0->pub_done != 0;
        sh = shift;
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
    for (int r = warp; r < kRows; r += kThreads / 32) {
        int g = 0, e = 0;
        if (r < rows_here)
            for (int c = lane; c < nbr; c += 32) {
                const unsigned long long kk = sk[r * nbr + c] >> sh;
                g += kk > Tsh;
                e += kk == Tsh;
            }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (lane == 0 && r < rows_here) {
            cs0->all_gt[r0 + r] = g;
            cs0->all_eq[r0 + r] = e;
        }
    }
    cluster.sync();   // every row's counts are in rank 0
    // every CTA scans all rows of the head (warp 0, four rows per lane) and
    // keeps what concerns its own rows
    if (warp == 0) {
        constexpr int kPer = (kMaxCta * kRows) / 32;
        int eqv[kPer], gtv[kPer];
        int eq_local = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int r = kPer * lane + j;
            eqv[j] = r < nbr ? cs0->all_eq[r] : 0;
            gtv[j] = r < nbr ? cs0->all_gt[r] : 0;
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
    __shared__ int s_ok;
    if (t == 0) {
        s_ok = (cs.total_sel == k && cs.total_items <= cap);
        if (rank == 0) {
            head_items[bh] = s_ok ? cs.total_items : 0;
            if (!s_ok) atomicOr(status, kDevCount);
        }
    }
    __syncthreads();
    const int s_sel_before = 0, s_item_before = 0;
    if (s_ok) {
        // work items: one thread per local row
        for (int r = t; r < rows_here; r += kThreads) {
            const int sel = cs.row_sel[r];
            const int nit = sel > 0 ? (sel + chunk - 1) / chunk : 1;
            const int rs = bh * k + s_sel_before + cs.row_start[r];
            for (int j = 0; j < nit; ++j) {
                WorkItem w;
                w.row = bh * nbr + r0 + r;
                w.col_start = rs + j * chunk;
                w.ncols = max(0, min(chunk, sel - j * chunk));
                w.chunk_info = j | (nit << 16);
                items[(size_t)bh * cap + s_item_before + cs.row_item[r] + j] = w;
            }
        }
        // column lists: one warp per local row, ascending columns
        const unsigned int lt_mask = (1u << lane) - 1u;
        for (int r = warp; r < rows_here; r += kThreads / 32) {
            const int rs = bh * k + s_sel_before + cs.row_start[r];
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
    cluster.sync();   // no CTA leaves while another still reads its shared memory
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
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ncta;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float scale = 1.0f / sqrtf((float)p.D);
    const float *qhat = w.pooled;
    const float *khat = w.pooled + (size_t)p.BH * p.nbr * p.D;
    e = cudaLaunchKernelEx(&cfg, kern, qhat, khat, (const int *)w.cnt, p.H, p.nbr, scale, p.first_n,
                           p.diag_n, p.k, p.cap, p.chunk, w.keys, w.mlo, logit_out, w.cols, sel_out,
                           p.mode == 0 ? w.bitmap : (unsigned int *)nullptr, w.words_per_row, w.items,
                           w.head_items, w.state, w.status);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

bool lowres_select_fused_supported(const Problem &p) {
    return p.nbr <= kMaxCta * kRows;
}

cudaError_t launch_lowres_select_fused(const Problem &p, const Workspace &w, float *logit_out,
                                       int32_t *sel_out, cudaStream_t s) {
    return p.D == 64 ? launch_typed<64>(p, w, logit_out, sel_out, s)
                     : launch_typed<32>(p, w, logit_out, sel_out, s);
}

}  // namespace mra
