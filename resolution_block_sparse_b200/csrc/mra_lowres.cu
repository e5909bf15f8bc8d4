// mra_lowres.cu - low-resolution logits, selection keys, and the
// low-resolution correction of full mode.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理":
//   step one  - a small full matmul of the pooled Q and K gives the block-logit
//               map; blocks without valid tokens are pushed down in their rows
//               and columns;
//   step two  - a global top-k over that map, with a 5e3 bias on the first-n
//               row/column blocks and on the band around the main diagonal;
//   step four - in full mode the pooled V, weighted by the low-resolution
//               attention of the unselected blocks, is added with its own
//               maximum and normaliser.
//
// Selection key.  The top-k ranks, per (batch, head), the value
//   x + 5e3 * tier,  x = l - rowmax (fp32), tier = #priors - 2*[empty row] - 2*[empty col],
// which equals the page's additive biases (5e3 per prior, 1e4 per empty side).
// Instead of adding 5e3 in fp32 (which would quantise x to ~5e-4), the key is
// the exact lexicographic pair (tier, x) packed into 35 bits:
//   key = (tier + 4) << 32 | order_bits(x).
// For |x| < 2500 this order equals the order of the exact sum; a larger |x|
// raises MRA_DEV_KEY_RANGE in the device status word.
#include <cuda_bf16.h>

#include "mra_internal.cuh"
#include "mra_select_common.cuh"

namespace mra {

namespace {

__device__ __forceinline__ int in_band(int r, int c, int g) {
    if (g <= 0) return 0;
    const int lo = -(g / 2);
    const int hi = (g + 1) / 2 - 1;
    const int off = c - r;
    return (off >= lo && off <= hi) ? 1 : 0;
}

constexpr int kLowresThreads = 256;

// One CTA: R block rows of one (batch, head) against every block column, in
// tiles of kKeysCT columns.  Thread tile: R/8 rows x 2 consecutive columns,
// fp32 FFMA; the Q-hat rows and a transposed K-hat column tile sit in shared
// memory (a fixed 16 KB tile, so that short row strips leave room for several
// CTAs per SM).
constexpr int kKeysCT = 64;

template <int D, int R>
__global__ void __launch_bounds__(kLowresThreads)
lowres_keys_kernel(const float *__restrict__ qhat, const float *__restrict__ khat,
                   const int *__restrict__ cnt, int H, int nbr, long long nbr2, float scale,
                   int first_n, int diag_n, int k, unsigned long long *__restrict__ keys,
                   float *__restrict__ mlo, float *__restrict__ logit_out,
                   unsigned int *__restrict__ hist, unsigned int *__restrict__ arrive,
                   SelState *__restrict__ state, unsigned int *__restrict__ status) {
    pdl_wait();
    constexpr int CT = kKeysCT;
    constexpr int RPT = R / 8;                 // rows per thread (eight row groups)
    static_assert(R % 8 == 0 && kLowresThreads == 256, "thread tiling: 8 row groups x 32 column pairs");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *qs = reinterpret_cast<float *>(smem_raw);                  // [R][D]
    float *kT = qs + R * D;                                            // [D][CT]
    float *lt = kT + D * CT;                                           // [R][nbr]
    float *rmax = lt + (size_t)R * nbr;                                // [R]
    int *cnts = reinterpret_cast<int *>(rmax + R);                     // [nbr]
    unsigned int *h0 = reinterpret_cast<unsigned int *>(cnts + nbr);   // [2048]
    __shared__ unsigned int s_tmp[256];
    __shared__ int s_flag, s_last, s_bin;
    __shared__ unsigned int s_need;

    const int t = threadIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int r0 = blockIdx.x * R;
    const float *qh = qhat + (size_t)bh * nbr * D;
    const float *kh = khat + (size_t)bh * nbr * D;

    if (t == 0) s_flag = 0;
    for (int c = t; c < nbr; c += kLowresThreads) cnts[c] = cnt[(size_t)b * nbr + c];
    for (int i = t; i < (1 << kHist0Bits); i += kLowresThreads) h0[i] = 0u;
    {
        // all loads in flight before the first shared-memory store
        constexpr int kQ = (R * D / 4 + kLowresThreads - 1) / kLowresThreads;
        float4 v[kQ];
#pragma unroll
        for (int u = 0; u < kQ; ++u) {
            const int i = t + u * kLowresThreads;
            const int r = (4 * i) / D;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < R * D / 4 && r0 + r < nbr)
                v[u] = reinterpret_cast<const float4 *>(qh + (size_t)(r0 + r) * D)[(4 * i) % D / 4];
        }
#pragma unroll
        for (int u = 0; u < kQ; ++u) {
            const int i = t + u * kLowresThreads;
            if (i < R * D / 4) reinterpret_cast<float4 *>(qs)[i] = v[u];
        }
    }

    const int rg = t >> 5, cg = t & 31;   // rows RPT*rg .., columns 2*cg, 2*cg + 1 of the tile
    for (int ct = 0; ct < nbr; ct += CT) {
        __syncthreads();
        // transposed column tile: kT[d][c] = khat[ct + c][d]
        {
            constexpr int kL = CT * D / 4 / kLowresThreads;   // float4 loads per thread
            float4 v[kL];
#pragma unroll
            for (int u = 0; u < kL; ++u) {
                const int e = t + u * kLowresThreads;
                const int c = e % CT, d4 = e / CT;
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ct + c < nbr) v[u] = reinterpret_cast<const float4 *>(kh + (size_t)(ct + c) * D)[d4];
            }
#pragma unroll
            for (int u = 0; u < kL; ++u) {
                const int e = t + u * kLowresThreads;
                const int c = e % CT, d4 = e / CT;
                kT[(4 * d4 + 0) * CT + c] = v[u].x;
                kT[(4 * d4 + 1) * CT + c] = v[u].y;
                kT[(4 * d4 + 2) * CT + c] = v[u].z;
                kT[(4 * d4 + 3) * CT + c] = v[u].w;
            }
        }
        __syncthreads();
        float acc[RPT][2];
#pragma unroll
        for (int i = 0; i < RPT; ++i) acc[i][0] = acc[i][1] = 0.0f;
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
            float4 qv[RPT];
#pragma unroll
            for (int i = 0; i < RPT; ++i) qv[i] = *reinterpret_cast<const float4 *>(qs + (RPT * rg + i) * D + d);
#pragma unroll
            for (int dd = 0; dd < 4; ++dd) {
                const float2 kv = *reinterpret_cast<const float2 *>(kT + (d + dd) * CT + 2 * cg);
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const float qd = dd == 0 ? qv[i].x : dd == 1 ? qv[i].y : dd == 2 ? qv[i].z : qv[i].w;
                    acc[i][0] = fmaf(qd, kv.x, acc[i][0]);
                    acc[i][1] = fmaf(qd, kv.y, acc[i][1]);
                }
            }
        }
        const int c0 = ct + 2 * cg;
#pragma unroll
        for (int i = 0; i < RPT; ++i)
#pragma unroll
            for (int j = 0; j < 2; ++j)
                if (c0 + j < nbr) lt[(size_t)(RPT * rg + i) * nbr + c0 + j] = acc[i][j] * scale;
    }
    __syncthreads();

    // row max over valid columns (0 when the row has none)
    const int warp = t >> 5, lane = t & 31;
    for (int r = warp; r < R; r += kLowresThreads / 32) {
        float m = -INFINITY;
        for (int c = lane; c < nbr; c += 32)
            if (cnts[c] > 0) m = fmaxf(m, lt[(size_t)r * nbr + c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (m == -INFINITY) m = 0.0f;
        if (lane == 0) {
            rmax[r] = m;
            if (r0 + r < nbr) mlo[(size_t)bh * nbr + r0 + r] = m;
        }
    }
    __syncthreads();

    // keys, exported logits, first radix histogram (bits 24..34)
    const int rows_here = min(R, nbr - r0);
    const int n_here = rows_here * nbr;
    unsigned long long *kout = keys + (size_t)bh * nbr2 + (size_t)r0 * nbr;
    int flag = 0;
    // warp-uniform trip count so that the histogram update can aggregate lanes
    for (int e0 = (t & ~31); e0 < n_here; e0 += kLowresThreads) {
        const int e = e0 + lane;
        const bool act = e < n_here;
        unsigned long long key = 0;
        if (act) {
            const int r = e / nbr, c = e - r * nbr;
            const int gr = r0 + r;
            const float l = lt[e];
            float x = l - rmax[r];
            if (x == 0.0f) x = 0.0f;  // canonical +0
            if (!(fabsf(x) < 2500.0f)) flag = 1;
            int tier = 0;
            if (first_n > 0 && (gr < first_n || c < first_n)) ++tier;
            tier += in_band(gr, c, diag_n);
            if (cnts[gr] <= 0) tier -= 2;
            if (cnts[c] <= 0) tier -= 2;
            key = ((unsigned long long)(tier + 4) << 32) | (unsigned long long)float_order_bits(x);
            kout[e] = key;
            if (logit_out) logit_out[(size_t)bh * nbr2 + (size_t)gr * nbr + c] = l;
        }
        warp_hist_add(h0, (unsigned)(key >> 24), act);
    }
    if (flag) s_flag = 1;
    __syncthreads();
    if (t == 0 && s_flag) atomicOr(status, kDevKeyRange);
    unsigned int *gh = hist + (size_t)bh * 3 * kHistBins;
    for (int i = t; i < (1 << kHist0Bits); i += kLowresThreads)
        if (h0[i]) atomicAdd(&gh[i], h0[i]);

    // the last CTA of this head locates the bucket of the k-th key
    __threadfence();
    __syncthreads();
    if (t == 0) s_last = (atomicAdd(&arrive[(size_t)bh * 4 + 0], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    find_bucket_256(gh, 1 << kHist0Bits, (unsigned)k, s_tmp, &s_bin, &s_need);
    if (t == 0) {
        SelState st;
        st.prefix = (unsigned long long)s_bin << (kHist1Bits + kHist2Bits);
        st.need = s_need;
        st.pad = 0;
        state[bh] = st;
    }
}

// Low-resolution part of full mode for R block rows of one (batch, head):
//   w_rc = cnt_c * exp(l_rc - rowmax_r) for every unselected c with cnt_c > 0,
//   olo_r = sum_c w_rc * vhat_c,   llo_r = sum_c w_rc.
// block rows per CTA (every CTA reads the whole pooled V of its head, so
// fewer rows per CTA cost more loads than they win in occupancy)
template <int D>
constexpr int pv_rows() { return 32; }

template <int D>
__global__ void __launch_bounds__(kLowresThreads)
lowres_pv_kernel(const unsigned long long *__restrict__ keys, const unsigned int *__restrict__ bitmap,
                 int wpr, const int *__restrict__ cnt, const float *__restrict__ vhat, int H,
                 int nbr, long long nbr2, float *__restrict__ olo, float *__restrict__ llo) {
    pdl_wait();
    constexpr int R = pv_rows<D>();
    constexpr int kCt = 32;
    constexpr int kVL = kCt * D / 4 / kLowresThreads;      // float4 loads of the V-hat tile
    constexpr int kWL = R * kCt / kLowresThreads;          // weights per thread and tile
    __shared__ __align__(16) float vs[kCt][D];
    __shared__ float ws[R][kCt + 1];
    const int t = threadIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int r0 = blockIdx.x * R;
    const float *vh = vhat + (size_t)bh * nbr * D;
    // thread tile: kRpt rows x 4 head dims
    constexpr int kDG = D / 4;                    // dim groups
    constexpr int kRG = kLowresThreads / kDG;     // row groups
    constexpr int kRpt = R / kRG;                 // rows per thread
    static_assert(kRpt >= 1 && kRG * kRpt == R, "tile shape");
    const int dg = t % kDG, rg = t / kDG;
    float4 acc[kRpt];
    float lsum[kRpt];
#pragma unroll
    for (int i = 0; i < kRpt; ++i) {
        acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        lsum[i] = 0.0f;
    }

    // the global loads of tile ct + kCt are issued before the products of
    // tile ct, so that their latency overlaps the arithmetic
    float4 vv[kVL];
    unsigned long long kv[kWL];
    unsigned int bw[kWL];
    int cc[kWL];
    auto load_tile = [&](int ct) {
#pragma unroll
        for (int u = 0; u < kVL; ++u) {
            const int i = t + u * kLowresThreads;
            const int c = (4 * i) / D;
            vv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (ct + c < nbr) vv[u] = reinterpret_cast<const float4 *>(vh + (size_t)(ct + c) * D)[(4 * i) % D / 4];
        }
#pragma unroll
        for (int u = 0; u < kWL; ++u) {
            const int e = t + u * kLowresThreads;
            const int r = e / kCt, c = e % kCt;
            const int gr = r0 + r, gc = ct + c;
            kv[u] = 0ull;
            bw[u] = 0xffffffffu;
            cc[u] = 0;
            if (gr < nbr && gc < nbr) {
                cc[u] = cnt[(size_t)b * nbr + gc];
                bw[u] = bitmap[((size_t)bh * nbr + gr) * wpr + (gc >> 5)];
                kv[u] = keys[(size_t)bh * nbr2 + (size_t)gr * nbr + gc];
            }
        }
    };
    load_tile(0);
    for (int ct = 0; ct < nbr; ct += kCt) {
        __syncthreads();   // previous tile fully consumed
#pragma unroll
        for (int u = 0; u < kVL; ++u) {
            const int i = t + u * kLowresThreads;
            reinterpret_cast<float4 *>(&vs[0][0])[i] = vv[u];
        }
#pragma unroll
        for (int u = 0; u < kWL; ++u) {
            const int e = t + u * kLowresThreads;
            const int r = e / kCt, c = e % kCt;
            const int gc = ct + c;
            float wv = 0.0f;
            if (cc[u] > 0 && !((bw[u] >> (gc & 31)) & 1u)) {
                const float x = float_from_order_bits((unsigned int)(kv[u] & 0xffffffffull));
                wv = (float)cc[u] * expf(x);
            }
            ws[r][c] = wv;
        }
        if (ct + kCt < nbr) load_tile(ct + kCt);
        __syncthreads();
#pragma unroll 8
        for (int c = 0; c < kCt; ++c) {
            const float4 v4 = *reinterpret_cast<const float4 *>(&vs[c][4 * dg]);
#pragma unroll
            for (int i = 0; i < kRpt; ++i) {
                const float wv = ws[rg * kRpt + i][c];
                acc[i].x = fmaf(wv, v4.x, acc[i].x);
                acc[i].y = fmaf(wv, v4.y, acc[i].y);
                acc[i].z = fmaf(wv, v4.z, acc[i].z);
                acc[i].w = fmaf(wv, v4.w, acc[i].w);
                lsum[i] += wv;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kRpt; ++i) {
        const int gr = r0 + rg * kRpt + i;
        if (gr < nbr) {
            *reinterpret_cast<float4 *>(olo + ((size_t)bh * nbr + gr) * D + 4 * dg) = acc[i];
            if (dg == 0) llo[(size_t)bh * nbr + gr] = lsum[i];
        }
    }
}

template <int D, int R>
cudaError_t launch_keys_rt(const Problem &p, const Workspace &w, float *logit_out, cudaStream_t s) {
    constexpr int CT = kKeysCT;
    const size_t smem = sizeof(float) * ((size_t)R * D + (size_t)D * CT + (size_t)R * p.nbr + R) +
                        sizeof(int) * (size_t)p.nbr + sizeof(unsigned int) * (1u << kHist0Bits);
    cudaError_t e = cudaFuncSetAttribute(lowres_keys_kernel<D, R>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.nbr + R - 1) / R, p.BH);
    const float scale = 1.0f / sqrtf((float)p.D);
    const float *qhat = w.pooled;
    const float *khat = w.pooled + (size_t)p.BH * p.nbr * p.D;
    return launch_dependent(lowres_keys_kernel<D, R>, dim3(grid), dim3(kLowresThreads), smem, s, 
        qhat, khat, w.cnt, p.H, p.nbr, p.nbr2, scale, p.first_n, p.diag_n, p.k, w.keys, w.mlo,
        logit_out, w.hist, w.arrive, w.state, w.status);
}

template <int D>
cudaError_t launch_keys_typed(const Problem &p, const Workspace &w, float *logit_out,
                              cudaStream_t s) {
    if (p.r_tile == 32) return launch_keys_rt<D, 32>(p, w, logit_out, s);
    if (p.r_tile == 16) return launch_keys_rt<D, 16>(p, w, logit_out, s);
    return launch_keys_rt<D, 8>(p, w, logit_out, s);
}

}  // namespace

cudaError_t launch_lowres_keys(const Problem &p, const Workspace &w, float *logit_out,
                               cudaStream_t s) {
    return p.D == 64 ? launch_keys_typed<64>(p, w, logit_out, s)
                     : launch_keys_typed<32>(p, w, logit_out, s);
}

cudaError_t launch_lowres_pv(const Problem &p, const Workspace &w, cudaStream_t s) {
    const float *vhat = w.pooled + (size_t)2 * p.BH * p.nbr * p.D;
    if (p.D == 64)
        return launch_dependent(lowres_pv_kernel<64>, dim3((p.nbr + pv_rows<64>() - 1) / pv_rows<64>(), p.BH),
                                dim3(kLowresThreads), 0, s, w.keys, w.bitmap, w.words_per_row, w.cnt, vhat, p.H,
                                p.nbr, p.nbr2, w.olo, w.llo);
    return launch_dependent(lowres_pv_kernel<32>, dim3((p.nbr + pv_rows<32>() - 1) / pv_rows<32>(), p.BH),
                            dim3(kLowresThreads), 0, s, w.keys, w.bitmap, w.words_per_row, w.cnt, vhat, p.H,
                            p.nbr, p.nbr2, w.olo, w.llo);
}

}  // namespace mra
