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
// together: local histograms are added into the rank-0 CTA's histogram
// through distributed shared memory, rank 0 locates the bucket of the k-th
// key, and every CTA reads the result back.  Cluster barriers separate the
// steps (hardware barriers, no spinning).  The per-row counts, the scan that
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

__device__ __forceinline__ int band_of(int r, int c, int g) {
    if (g <= 0) return 0;
    const int lo = -(g / 2);
    const int hi = (g + 1) / 2 - 1;
    const int off = c - r;
    return (off >= lo && off <= hi) ? 1 : 0;
}

struct ClusterShared {
    unsigned int hist[kHistBins];   // rank 0: the cluster histogram of the current pass
    unsigned int lh[kHistBins];     // this CTA's histogram
    unsigned int s_tmp[kThreads];
    unsigned long long prefix;      // rank 0: threshold bits fixed so far
    unsigned int need;
    int bin;
    unsigned int bin_need;
    int tot_eq[kMaxCta], tot_sel[kMaxCta], tot_items[kMaxCta];   // rank 0: per-CTA totals
    int row_gt[kRows], row_eq[kRows], row_sel[kRows], row_take[kRows], row_start[kRows], row_item[kRows];
    int flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads)
lowres_select_cluster_kernel(const float *__restrict__ qhat, const float *__restrict__ khat,
                             const int *__restrict__ cnt, int H, int nbr, float scale, int first_n,
                             int diag_n, int k, int cap, unsigned long long *__restrict__ keys_out,
                             float *__restrict__ mlo, float *__restrict__ logit_out,
                             int *__restrict__ cols, int32_t *__restrict__ sel_out,
                             unsigned int *__restrict__ bitmap, int wpr, WorkItem *__restrict__ items,
                             int *__restrict__ head_items, SelState *__restrict__ state,
                             unsigned int *__restrict__ status) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int ncta = (int)cluster.num_blocks();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *qs = reinterpret_cast<float *>(smem_raw);                     // [kRows][D]
    float *kT = qs + kRows * D;                                           // [D][kCT]
    float *lt = kT + D * kCT;                                             // [kRows][nbr]
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
        for (int i = t; i < kHistBins; i += kThreads) cs.hist[i] = 0u;
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
    cluster.sync();   // rank 0's histogram is clear; every CTA of the cluster is running
    if (t == 0 && cs.flag) atomicOr(status, kDevKeyRange);

    // ------------------------------------------------------------ radix passes
    unsigned long long prefix = 0ull;
    unsigned int need = (unsigned)k;
    for (int pass = 0; pass < 3; ++pass) {
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
        for (int i = t; i < (1 << bits); i += kThreads)
            if (cs.lh[i]) atomicAdd(&cs0->hist[i], cs.lh[i]);
        cluster.sync();   // the cluster histogram of this pass is complete
        if (rank == 0) {
            find_bucket<kThreads>([](int i) { return cs.hist[i]; }, 1 << bits, need, cs.s_tmp, &cs.bin,
                                  &cs.bin_need);
            if (t == 0) {
                cs.prefix = prefix | ((unsigned long long)cs.bin << shift);
                cs.need = cs.bin_need;
            }
            __syncthreads();
            for (int i = t; i < kHistBins; i += kThreads) cs.hist[i] = 0u;   // for the next pass
        }
        cluster.sync();   // rank 0 published the bucket
        prefix = cs0->prefix;
        need = cs0->need;
    }
    const unsigned long long T = prefix;
    if (rank == 0 && t == 0) {
        SelState st;
        st.prefix = T;
        st.need = need;
        st.pad = 0;
        state[bh] = st;
    }

    // ------------------------------------------------------------ per-row counts and scans
    for (int r = warp; r < kRows; r += kThreads / 32) {
        int g = 0, e = 0;
        if (r < rows_here)
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
            cs.row_gt[r] = g;
            cs.row_eq[r] = e;
        }
    }
    __syncthreads();
    if (t == 0) {
        int te = 0;
        for (int r = 0; r < kRows; ++r) te += cs.row_eq[r];
        cs0->tot_eq[rank] = te;
    }
    cluster.sync();
    if (t == 0) {
        int eq_before = 0;
        for (int i = 0; i < rank; ++i) eq_before += cs0->tot_eq[i];
        int ts = 0, ti = 0;
        for (int r = 0; r < rows_here; ++r) {
            int take = (int)need - eq_before;
            take = take < 0 ? 0 : (take > cs.row_eq[r] ? cs.row_eq[r] : take);
            const int sel = cs.row_gt[r] + take;
            cs.row_take[r] = take;
            cs.row_sel[r] = sel;
            cs.row_start[r] = ts;
            cs.row_item[r] = ti;
            ts += sel;
            ti += sel > 0 ? (sel + kChunk - 1) / kChunk : 1;
            eq_before += cs.row_eq[r];
        }
        cs0->tot_sel[rank] = ts;
        cs0->tot_items[rank] = ti;
    }
    cluster.sync();
    __shared__ int s_sel_before, s_item_before, s_ok;
    if (t == 0) {
        int sb = 0, ib = 0, st = 0, it = 0;
        for (int i = 0; i < ncta; ++i) {
            if (i < rank) {
                sb += cs0->tot_sel[i];
                ib += cs0->tot_items[i];
            }
            st += cs0->tot_sel[i];
            it += cs0->tot_items[i];
        }
        s_sel_before = sb;
        s_item_before = ib;
        s_ok = (st == k && it <= cap);
        if (rank == 0) {
            head_items[bh] = s_ok ? it : 0;
            if (!s_ok) atomicOr(status, kDevCount);
        }
    }
    __syncthreads();
    if (s_ok) {
        // work items: one thread per local row
        for (int r = t; r < rows_here; r += kThreads) {
            const int sel = cs.row_sel[r];
            const int nit = sel > 0 ? (sel + kChunk - 1) / kChunk : 1;
            const int rs = bh * k + s_sel_before + cs.row_start[r];
            for (int j = 0; j < nit; ++j) {
                WorkItem w;
                w.row = bh * nbr + r0 + r;
                w.col_start = rs + j * kChunk;
                w.ncols = max(0, min(kChunk, sel - j * kChunk));
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
                const unsigned long long key = c < nbr ? sk[r * nbr + c] : 0ull;
                const bool is_gt = c < nbr && key > T;
                const bool is_eq = c < nbr && key == T;
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
    const size_t smem = sizeof(float) * ((size_t)kRows * D + (size_t)D * kCT + (size_t)kRows * p.nbr) +
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
                           p.diag_n, p.k, p.cap, w.keys, w.mlo, logit_out, w.cols, sel_out,
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
