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

#include <algorithm>

#include "mra_internal.cuh"
#include "mra_select_common.cuh"

namespace mra {

namespace {

constexpr int kLowresThreads = 256;

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"((unsigned)__cvta_generic_to_shared(dst)),
                 "l"(src));
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"((unsigned)__cvta_generic_to_shared(dst)),
                 "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Logit map of maps above 128 x 128 blocks on 128 x 128 tiles:
// l_rc = scale * qhat_r . khat_c in fp32 (FFMA, d ascending), written to
// L [BH][nbr][nbr], and the maximum over the tile's valid columns (cnt > 0) of
// each row to pmax [BH][nbr][ntiles] (-inf when none).  CTAs walk the tiles
// with a stride of the grid, two CTAs per SM, so that one CTA's cp.async
// loads of Q-hat and K-hat rows overlap the other's products.  Thread (tx, ty)
// of 16 x 16 holds rows ty + 16 i and columns tx + 16 j (8 x 8 register tile:
// 256 FMAs per 16 shared-memory loads of 16 bytes); a warp's column loads are
// 16 consecutive rows of a padded [128][D + 4] tile and its row loads
// broadcast.
constexpr int kLgT = 128;
constexpr int kLgR = kLgT / 16;   // rows (and columns) per thread

template <int D>
struct LgSmem {
    float q[kLgT][D + 4];
    float k[kLgT][D + 4];
};

template <int D>
__global__ void __launch_bounds__(kLowresThreads, 2)
lowres_logits_kernel(const float *__restrict__ qhat, const float *__restrict__ khat,
                     const int *__restrict__ cnt, int H, int nbr, float scale, float *__restrict__ L,
                     float *__restrict__ pmax, int total_tiles) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char lg_smem[];
    LgSmem<D> &sh = *reinterpret_cast<LgSmem<D> *>(lg_smem);
    const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
    const int nt = (nbr + kLgT - 1) / kLgT;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
        const int bh = tile / (nt * nt), rem = tile - bh * nt * nt;
        const int ct = rem % nt;
        const int row0 = (rem / nt) * kLgT, col0 = ct * kLgT;
        {
            const float *qh = qhat + (size_t)bh * nbr * D;
            const float *kh = khat + (size_t)bh * nbr * D;
            for (int i = t; i < kLgT * D / 4; i += kLowresThreads) {
                const int r = i / (D / 4), d4 = i % (D / 4);
                if (row0 + r < nbr) cp_async16(&sh.q[r][4 * d4], qh + (size_t)(row0 + r) * D + 4 * d4);
                else *reinterpret_cast<float4 *>(&sh.q[r][4 * d4]) = make_float4(0.f, 0.f, 0.f, 0.f);
                if (col0 + r < nbr) cp_async16(&sh.k[r][4 * d4], kh + (size_t)(col0 + r) * D + 4 * d4);
                else *reinterpret_cast<float4 *>(&sh.k[r][4 * d4]) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            cp_async_commit();
            cp_async_wait<0>();
        }
        __syncthreads();   // this tile landed and is visible
        float acc[kLgR][kLgR];
#pragma unroll
        for (int i = 0; i < kLgR; ++i)
#pragma unroll
            for (int j = 0; j < kLgR; ++j) acc[i][j] = 0.0f;
#pragma unroll 1
        for (int d = 0; d < D; d += 4) {
            float4 kc[kLgR];
#pragma unroll
            for (int j = 0; j < kLgR; ++j) kc[j] = *reinterpret_cast<const float4 *>(&sh.k[tx + 16 * j][d]);
#pragma unroll
            for (int i = 0; i < kLgR; ++i) {
                const float4 qr = *reinterpret_cast<const float4 *>(&sh.q[ty + 16 * i][d]);
#pragma unroll
                for (int j = 0; j < kLgR; ++j) {
                    acc[i][j] = fmaf(qr.x, kc[j].x, acc[i][j]);
                    acc[i][j] = fmaf(qr.y, kc[j].y, acc[i][j]);
                    acc[i][j] = fmaf(qr.z, kc[j].z, acc[i][j]);
                    acc[i][j] = fmaf(qr.w, kc[j].w, acc[i][j]);
                }
            }
        }
        __syncthreads();   // every thread is done with the tiles before the next are staged
        const int *crow = cnt + (size_t)(bh / H) * nbr;
#pragma unroll
        for (int i = 0; i < kLgR; ++i) {
            const int r = row0 + ty + 16 * i;
            float m = -INFINITY;
#pragma unroll
            for (int j = 0; j < kLgR; ++j) {
                const int c = col0 + tx + 16 * j;
                const float l = acc[i][j] * scale;
                if (r < nbr && c < nbr) L[((size_t)bh * nbr + r) * nbr + c] = l;
                if (c < nbr && __ldg(crow + c) > 0) m = fmaxf(m, l);
            }
            // maximum over the 16 lanes of this row (a half warp)
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (tx == 0 && r < nbr) pmax[((size_t)bh * nbr + r) * nt + ct] = m;
        }
    }
}

// Selection keys of R block rows of one (batch, head) from the logit map: the
// row maximum over valid columns from the tile maxima (0 when the row has
// none), x = l - rowmax, the key (tier, order bits of x), and the first radix
// histogram; the last CTA of the head locates the bucket of the k-th key.
template <int R>
__global__ void __launch_bounds__(kLowresThreads)
lowres_keys_kernel(const float *__restrict__ L, const float *__restrict__ pmax,
                   const int *__restrict__ cnt, int H, int nbr, long long nbr2,
                   int first_n, int diag_n, int k, unsigned long long *__restrict__ keys,
                   float *__restrict__ mlo, unsigned int *__restrict__ hist, unsigned int *__restrict__ arrive,
                   SelState *__restrict__ state, unsigned int *__restrict__ status) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    int *cnts = reinterpret_cast<int *>(smem_raw);                     // [nbr]
    unsigned int *h0 = reinterpret_cast<unsigned int *>(cnts + nbr);   // [2048]
    __shared__ float rmax[R];
    __shared__ unsigned int s_tmp[256];
    __shared__ int s_flag, s_last, s_bin;
    __shared__ unsigned int s_need;

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int r0 = blockIdx.x * R;
    if (t == 0) s_flag = 0;
    for (int c = t; c < nbr; c += kLowresThreads) cnts[c] = cnt[(size_t)b * nbr + c];
    for (int i = t; i < (1 << kHist0Bits); i += kLowresThreads) h0[i] = 0u;
    const int ntiles = (nbr + kLgT - 1) / kLgT;
    for (int r = warp; r < R; r += kLowresThreads / 32) {
        float m = -INFINITY;
        if (r0 + r < nbr)
            for (int j = lane; j < ntiles; j += 32) m = fmaxf(m, pmax[((size_t)bh * nbr + r0 + r) * ntiles + j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (m == -INFINITY) m = 0.0f;
        if (lane == 0) {
            rmax[r] = m;
            if (r0 + r < nbr) mlo[(size_t)bh * nbr + r0 + r] = m;
        }
    }
    __syncthreads();

    // keys and the first radix histogram (bits 24..34): one warp per row, the
    // row's terms hoisted, kU loads of the row in flight per lane
    const int rows_here = min(R, nbr - r0);
    int flag = 0;
    constexpr int kU = 4;
    for (int r = warp; r < rows_here; r += kLowresThreads / 32) {
        const int gr = r0 + r;
        const float m = rmax[r];
        const float *lrow = L + ((size_t)bh * nbr + gr) * nbr;
        unsigned long long *krow = keys + (size_t)bh * nbr2 + (size_t)gr * nbr;
        const bool row_empty = cnts[gr] <= 0;
        for (int c0 = 0; c0 < nbr; c0 += 32 * kU) {
            float lv[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int c = c0 + 32 * u + lane;
                lv[u] = c < nbr ? lrow[c] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int c = c0 + 32 * u + lane;
                const bool act = c < nbr;
                const unsigned long long key =
                    act ? selection_key(lv[u], m, gr, c, first_n, diag_n, row_empty, cnts[c] <= 0, flag) : 0ull;
                if (act) krow[c] = key;
                hist_add(h0, (unsigned)(key >> 24), act);
            }
        }
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

// Low-resolution part of full mode for kPvR block rows of one (batch, head):
//   w_rc = cnt_c * exp(l_rc - rowmax_r) for every unselected c with cnt_c > 0,
//   olo_r = sum_c w_rc * vhat_c,   llo_r = sum_c w_rc,
// over tiles of kPvC columns.  Each tile's logits, V-hat rows, counts and
// selection words arrive by cp.async into one of two buffers while the
// previous tile is multiplied; the weights are formed once per tile (stored
// [c][r]), then a register-tiled product: thread (tx, ty) of 16 x 16 holds
// rows 2 ty, 2 ty + 1 and dims D/16 * tx ...
constexpr int kPvR = 32, kPvC = 64;

template <int D>
struct PvSmem {
    float v[2][kPvC][D + 4];
    float l[2][kPvR][kPvC + 4];
    float wt[kPvC][kPvR + 4];
    unsigned int selw[2][kPvR][2];
    int cntc[2][kPvC];
    float m[kPvR];
};

template <int D>
__global__ void __launch_bounds__(kLowresThreads)
lowres_pv_kernel(const float *__restrict__ L, const float *__restrict__ mlo, const unsigned int *__restrict__ bitmap,
                 int wpr, const int *__restrict__ cnt, const float *__restrict__ vhat, int H, int nbr,
                 float *__restrict__ olo, float *__restrict__ llo) {
    pdl_wait();
    constexpr int DW = D / 16;
    extern __shared__ __align__(16) unsigned char pv_smem[];
    PvSmem<D> &sh = *reinterpret_cast<PvSmem<D> *>(pv_smem);
    const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int r0 = blockIdx.x * kPvR;
    const float *vh = vhat + (size_t)bh * nbr * D;
    const float *lh = L + (size_t)bh * nbr * nbr;
    const bool l16 = (nbr & 3) == 0;   // logit rows 16-byte aligned
    // issues the copies of the tile at column c0 into buffer bf; out-of-range
    // entries are written as zeros (counts 0: no weight)
    auto stage = [&](int c0, int bf) {
        for (int i = t; i < kPvC * D / 4; i += kLowresThreads) {
            const int c = i / (D / 4), d4 = i % (D / 4);
            if (c0 + c < nbr) cp_async16(&sh.v[bf][c][4 * d4], vh + (size_t)(c0 + c) * D + 4 * d4);
            else *reinterpret_cast<float4 *>(&sh.v[bf][c][4 * d4]) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (l16) {
            for (int i = t; i < kPvR * kPvC / 4; i += kLowresThreads) {
                const int r = i / (kPvC / 4), c4 = 4 * (i % (kPvC / 4));
                if (r0 + r < nbr && c0 + c4 < nbr)
                    cp_async16(&sh.l[bf][r][c4], lh + (size_t)(r0 + r) * nbr + c0 + c4);
            }
        } else {
            for (int i = t; i < kPvR * kPvC; i += kLowresThreads) {
                const int r = i / kPvC, c = i % kPvC;
                if (r0 + r < nbr && c0 + c < nbr) cp_async4(&sh.l[bf][r][c], lh + (size_t)(r0 + r) * nbr + c0 + c);
            }
        }
        if (t < kPvC) {
            if (c0 + t < nbr) cp_async4(&sh.cntc[bf][t], cnt + (size_t)b * nbr + c0 + t);
            else sh.cntc[bf][t] = 0;
        } else if (t < kPvC + 2 * kPvR) {
            const int r = (t - kPvC) >> 1, wsel = (t - kPvC) & 1;
            const int w = (c0 >> 5) + wsel;   // c0 is a multiple of 64
            if (r0 + r < nbr && w < wpr) cp_async4(&sh.selw[bf][r][wsel], bitmap + ((size_t)bh * nbr + r0 + r) * wpr + w);
            else sh.selw[bf][r][wsel] = ~0u;
        }
    };
    if (t < kPvR) sh.m[t] = r0 + t < nbr ? mlo[(size_t)bh * nbr + r0 + t] : 0.0f;
    float acc[2][DW], ls[2] = {0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int e = 0; e < DW; ++e) acc[i][e] = 0.0f;
    const int ntiles = (nbr + kPvC - 1) / kPvC;
    stage(0, 0);
    cp_async_commit();
    for (int it = 0; it < ntiles; ++it) {
        const int bf = it & 1, c0 = it * kPvC;
        if (it + 1 < ntiles) stage(c0 + kPvC, bf ^ 1);   // that buffer was last read before the barrier below
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();   // tile it landed (every thread's copies) and is visible
        // weights: thread t forms (r, c) = (e % 32, e / 32) for e = t + 256 u
#pragma unroll
        for (int u = 0; u < kPvR * kPvC / kLowresThreads; ++u) {
            const int e = t + u * kLowresThreads;
            const int r = e % kPvR, c = e / kPvR;
            float w = 0.0f;
            const int cc = sh.cntc[bf][c];
            if (cc > 0 && !((sh.selw[bf][r][c >> 5] >> (c & 31)) & 1u))
                w = (float)cc * expf(sh.l[bf][r][c] - sh.m[r]);
            sh.wt[c][r] = w;
        }
        __syncthreads();
#pragma unroll 8
        for (int c = 0; c < kPvC; ++c) {
            const float2 w2 = *reinterpret_cast<const float2 *>(&sh.wt[c][2 * ty]);
            float vv[DW];
            if constexpr (DW == 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(&sh.v[bf][c][4 * tx]);
                vv[0] = v4.x; vv[1] = v4.y; vv[2] = v4.z; vv[3] = v4.w;
            } else {
                const float2 v2 = *reinterpret_cast<const float2 *>(&sh.v[bf][c][2 * tx]);
                vv[0] = v2.x; vv[1] = v2.y;
            }
#pragma unroll
            for (int e = 0; e < DW; ++e) {
                acc[0][e] = fmaf(w2.x, vv[e], acc[0][e]);
                acc[1][e] = fmaf(w2.y, vv[e], acc[1][e]);
            }
            ls[0] += w2.x;
            ls[1] += w2.y;
        }
        __syncthreads();   // wt and this tile's buffers are free
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int gr = r0 + 2 * ty + i;
        if (gr >= nbr) continue;
        float *dst = olo + ((size_t)bh * nbr + gr) * D + DW * tx;
#pragma unroll
        for (int e = 0; e < DW; ++e) dst[e] = acc[i][e];
        if (tx == 0) llo[(size_t)bh * nbr + gr] = ls[i];
    }
}

// The same low-resolution part on the tensor cores for bf16 problems:
// O_lo = W V-hat as mma.sync m16n8k8 with tf32 operands (the fp32 bits of W
// and V-hat are passed as they are; the tensor core reads their top 19 bits,
// 2^-10 relative, far inside the bf16 output's rounding) and fp32
// accumulation; the weights use the special-function unit's 2^x (about 2 ulp)
// and the normaliser llo sums the fp32 weights.  A CTA covers
// kPtR = 32 block rows with four warps: warp w takes rows 16 (w & 1) ..
// + 15 and head dims (w >> 1) D/2 .. + D/2 - 1, forming the weights of its A
// fragments itself (cnt_c exp(l - rowmax) for unselected valid blocks) from
// the logit tile; 64-column tiles of the logits and V-hat arrive by
// double-buffered cp.async.  The column tiles of a row block split over
// gridDim.z CTAs (so that a small number of heads still fills the SMs); with
// more than one split each writes fp32 partials of O and of the normaliser
// at opart / lpart [split][row], which lowres_pv_merge adds in split order.
constexpr int kPtR = 32, kPtC = 64, kPtThreads = 128;
constexpr int kPtMaxSplits = 4;

template <int D>
struct PtSmem {
    float l[2][kPtR][kPtC + 4];        // rows: 8 g + tq spread over the banks
    float v[2][kPtC][D + 8];           // rows 4 apart in distinct banks
    int cntc[2][kPtC];
    unsigned int selw[2][kPtR][2];
};

constexpr float kLog2eLo = 1.4426950408889634f;
// 2^x on the special-function unit (ex2.approx.ftz, about 2 ulp)
__device__ __forceinline__ float sfu_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const unsigned int (&a)[4], unsigned int b0, unsigned int b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kPtThreads)
lowres_pv_tf32_kernel(const float *__restrict__ L, const float *__restrict__ mlo,
                      const unsigned int *__restrict__ bitmap, int wpr, const int *__restrict__ cnt,
                      const float *__restrict__ vhat, int H, int nbr, float *__restrict__ olo,
                      float *__restrict__ llo, float *__restrict__ opart, float *__restrict__ lpart) {
    pdl_wait();
    constexpr int NT = D / 16;   // n-tiles of 8 dims per warp
    extern __shared__ __align__(16) unsigned char pt_smem[];
    PtSmem<D> &sh = *reinterpret_cast<PtSmem<D> *>(pt_smem);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const int bh = blockIdx.y, b = bh / H;
    const int r0 = blockIdx.x * kPtR;
    const int wr = 16 * (warp & 1), wd = (warp >> 1) * (D / 2);
    const float *vh = vhat + (size_t)bh * nbr * D;
    const float *lh = L + (size_t)bh * nbr * nbr;
    const bool l16 = (nbr & 3) == 0;
    auto stage = [&](int c0, int bf) {
        for (int i = t; i < kPtC * D / 4; i += kPtThreads) {
            const int c = i / (D / 4), d4 = i % (D / 4);
            if (c0 + c < nbr) cp_async16(&sh.v[bf][c][4 * d4], vh + (size_t)(c0 + c) * D + 4 * d4);
            else *reinterpret_cast<float4 *>(&sh.v[bf][c][4 * d4]) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (l16) {
            for (int i = t; i < kPtR * kPtC / 4; i += kPtThreads) {
                const int r = i / (kPtC / 4), c4 = 4 * (i % (kPtC / 4));
                if (r0 + r < nbr && c0 + c4 < nbr)
                    cp_async16(&sh.l[bf][r][c4], lh + (size_t)(r0 + r) * nbr + c0 + c4);
                else
                    *reinterpret_cast<float4 *>(&sh.l[bf][r][c4]) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else {
            for (int i = t; i < kPtR * kPtC; i += kPtThreads) {
                const int r = i / kPtC, c = i % kPtC;
                if (r0 + r < nbr && c0 + c < nbr) cp_async4(&sh.l[bf][r][c], lh + (size_t)(r0 + r) * nbr + c0 + c);
                else sh.l[bf][r][c] = 0.0f;
            }
        }
        if (t < kPtC) {
            if (c0 + t < nbr) cp_async4(&sh.cntc[bf][t], cnt + (size_t)b * nbr + c0 + t);
            else sh.cntc[bf][t] = 0;
        } else if (t < kPtC + 2 * kPtR) {
            const int r = (t - kPtC) >> 1, ws = (t - kPtC) & 1;
            const int w = (c0 >> 5) + ws;   // c0 is a multiple of 64
            if (r0 + r < nbr && w < wpr) cp_async4(&sh.selw[bf][r][ws], bitmap + ((size_t)bh * nbr + r0 + r) * wpr + w);
            else sh.selw[bf][r][ws] = ~0u;
        }
    };
    // this thread's two rows: wr + g and wr + g + 8 of the CTA
    const int ra = r0 + wr + g, rb = ra + 8;
    // exp(l - m) = 2^(l log2e - m log2e)
    const float ma = (ra < nbr ? mlo[(size_t)bh * nbr + ra] : 0.0f) * kLog2eLo;
    const float mb = (rb < nbr ? mlo[(size_t)bh * nbr + rb] : 0.0f) * kLog2eLo;
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
    float la = 0.0f, lb = 0.0f;
    const int ntiles_all = (nbr + kPtC - 1) / kPtC;
    const int split = blockIdx.z, nsplit = gridDim.z;
    const int t_begin = split * ntiles_all / nsplit, t_end = (split + 1) * ntiles_all / nsplit;
    const int ntiles = t_end - t_begin;
    if (ntiles > 0) stage(t_begin * kPtC, 0);
    cp_async_commit();
    for (int it = 0; it < ntiles; ++it) {
        const int bf = it & 1;
        if (it + 1 < ntiles) stage((t_begin + it + 1) * kPtC, bf ^ 1);   // that buffer was last read before the barrier below
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();   // tile it landed and is visible
        const unsigned long long sa = (unsigned long long)sh.selw[bf][wr + g][0] |
                                      ((unsigned long long)sh.selw[bf][wr + g][1] << 32);
        const unsigned long long sb = (unsigned long long)sh.selw[bf][wr + g + 8][0] |
                                      ((unsigned long long)sh.selw[bf][wr + g + 8][1] << 32);
#pragma unroll 2
        for (int ks = 0; ks < kPtC / 8; ++ks) {
            const int c = 8 * ks + tq;
            const int cc0 = sh.cntc[bf][c], cc1 = sh.cntc[bf][c + 4];
            float w[4];
            w[0] = (cc0 > 0 && !((sa >> c) & 1ull)) ? (float)cc0 * sfu_exp2(fmaf(sh.l[bf][wr + g][c], kLog2eLo, -ma)) : 0.0f;
            w[1] = (cc0 > 0 && !((sb >> c) & 1ull)) ? (float)cc0 * sfu_exp2(fmaf(sh.l[bf][wr + g + 8][c], kLog2eLo, -mb)) : 0.0f;
            w[2] = (cc1 > 0 && !((sa >> (c + 4)) & 1ull)) ? (float)cc1 * sfu_exp2(fmaf(sh.l[bf][wr + g][c + 4], kLog2eLo, -ma)) : 0.0f;
            w[3] = (cc1 > 0 && !((sb >> (c + 4)) & 1ull)) ? (float)cc1 * sfu_exp2(fmaf(sh.l[bf][wr + g + 8][c + 4], kLog2eLo, -mb)) : 0.0f;
            la += w[0] + w[2];
            lb += w[1] + w[3];
            const unsigned int af[4] = {__float_as_uint(w[0]), __float_as_uint(w[1]), __float_as_uint(w[2]),
                                        __float_as_uint(w[3])};
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const unsigned int b0 = __float_as_uint(sh.v[bf][c][wd + 8 * n + g]);
                const unsigned int b1 = __float_as_uint(sh.v[bf][c + 4][wd + 8 * n + g]);
                mma_tf32(acc[n], af, b0, b1);
            }
        }
        __syncthreads();   // this tile's buffers are free
    }
    // row sums over the four lanes of a row
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
        la += __shfl_xor_sync(0xffffffffu, la, o);
        lb += __shfl_xor_sync(0xffffffffu, lb, o);
    }
    const size_t plane = (size_t)gridDim.y * nbr;   // rows of all heads
    float *od = nsplit == 1 ? olo : opart + (size_t)split * plane * D;
    float *ld = nsplit == 1 ? llo : lpart + (size_t)split * plane;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int d = wd + 8 * n + 2 * tq;
        if (ra < nbr) *reinterpret_cast<float2 *>(od + ((size_t)bh * nbr + ra) * D + d) = make_float2(acc[n][0], acc[n][1]);
        if (rb < nbr) *reinterpret_cast<float2 *>(od + ((size_t)bh * nbr + rb) * D + d) = make_float2(acc[n][2], acc[n][3]);
    }
    if (tq == 0 && (warp >> 1) == 0) {
        if (ra < nbr) ld[(size_t)bh * nbr + ra] = la;
        if (rb < nbr) ld[(size_t)bh * nbr + rb] = lb;
    }
}

// Sums the split partials of the low-resolution part in split order: one
// thread per four elements of O (and per row of the normaliser).
template <int D>
__global__ void __launch_bounds__(256)
lowres_pv_merge_kernel(const float *__restrict__ opart, const float *__restrict__ lpart, int nsplit, int rows,
                       float *__restrict__ olo, float *__restrict__ llo) {
    pdl_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;   // float4 index
    const int n4 = rows * (D / 4);
    if (i < n4) {
        float4 a = reinterpret_cast<const float4 *>(opart)[i];
        for (int sp = 1; sp < nsplit; ++sp) {
            const float4 b = reinterpret_cast<const float4 *>(opart + (size_t)sp * rows * D)[i];
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        reinterpret_cast<float4 *>(olo)[i] = a;
    }
    if (i < rows) {
        float l = lpart[i];
        for (int sp = 1; sp < nsplit; ++sp) l += lpart[(size_t)sp * rows + i];
        llo[i] = l;
    }
}

template <int R>
cudaError_t launch_keys_rt(const Problem &p, const Workspace &w, const float *L, cudaStream_t s) {
    const size_t smem = sizeof(int) * (size_t)p.nbr + sizeof(unsigned int) * (1u << kHist0Bits);
    cudaError_t e = cudaFuncSetAttribute(lowres_keys_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    return launch_dependent(lowres_keys_kernel<R>, dim3((p.nbr + R - 1) / R, p.BH), dim3(kLowresThreads), smem, s,
                            L, (const float *)w.lo_pmax, (const int *)w.cnt, p.H, p.nbr, p.nbr2, p.first_n,
                            p.diag_n, p.k, w.keys, w.mlo, w.hist, w.arrive, w.state, w.status);
}

template <int D>
cudaError_t launch_logits_typed(const Problem &p, const Workspace &w, float *L, cudaStream_t s) {
    const long long nt = (p.nbr + kLgT - 1) / kLgT;
    const long long total = nt * nt * p.BH;
    const float scale = 1.0f / sqrtf((float)p.D);
    const float *qhat = w.pooled;
    const float *khat = w.pooled + (size_t)p.BH * p.nbr * p.D;
    const size_t smem = sizeof(LgSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(lowres_logits_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = std::min<long long>(total, 2LL * device_sm_count());
    return launch_dependent(lowres_logits_kernel<D>, dim3((unsigned)grid), dim3(kLowresThreads), smem, s, qhat, khat,
                            (const int *)w.cnt, p.H, p.nbr, scale, L, w.lo_pmax, (int)total);
}

}  // namespace

float *lowres_logit_map(const Workspace &w, float *logit_out) { return logit_out ? logit_out : w.lo_logits; }

cudaError_t launch_lowres_keys(const Problem &p, const Workspace &w, float *logit_out, cudaStream_t s) {
    float *L = lowres_logit_map(w, logit_out);
    cudaError_t e = p.D == 64 ? launch_logits_typed<64>(p, w, L, s) : launch_logits_typed<32>(p, w, L, s);
    if (e != cudaSuccess) return e;
    if (p.r_tile == 32) return launch_keys_rt<32>(p, w, L, s);
    if (p.r_tile == 16) return launch_keys_rt<16>(p, w, L, s);
    return launch_keys_rt<8>(p, w, L, s);
}

// Column splits of the tensor-core low-resolution kernel: enough CTAs for
// about four per SM, at most kPtMaxSplits and one 64-column tile per split.
int lowres_pv_splits(const Problem &p) {
    if (p.dtype != 0) return 1;
    const long long ctas = (long long)((p.nbr + kPtR - 1) / kPtR) * p.BH;
    const long long want = (4LL * device_sm_count() + ctas - 1) / ctas;
    const int ntiles = (p.nbr + kPtC - 1) / kPtC;
    return (int)std::max<long long>(1, std::min<long long>({want, (long long)kPtMaxSplits, (long long)ntiles}));
}

cudaError_t launch_lowres_pv(const Problem &p, const Workspace &w, const float *logit_out, cudaStream_t s) {
    const float *L = logit_out ? logit_out : w.lo_logits;
    const float *vhat = w.pooled + (size_t)2 * p.BH * p.nbr * p.D;
    const dim3 grid((unsigned)((p.nbr + kPvR - 1) / kPvR), (unsigned)p.BH);
    auto run = [&](auto kern, size_t smem) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_dependent(kern, grid, dim3(kLowresThreads), smem, s, L, (const float *)w.mlo,
                                (const unsigned int *)w.bitmap, w.words_per_row, (const int *)w.cnt, vhat, p.H,
                                p.nbr, w.olo, w.llo);
    };
    if (p.dtype == 0) {   // bf16 problems: tf32 tensor-core products
        const int nsplit = lowres_pv_splits(p);
        const dim3 tgrid((unsigned)((p.nbr + kPtR - 1) / kPtR), (unsigned)p.BH, (unsigned)nsplit);
        auto run_tc = [&](auto kern, size_t smem) -> cudaError_t {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            return launch_dependent(kern, tgrid, dim3(kPtThreads), smem, s, L, (const float *)w.mlo,
                                    (const unsigned int *)w.bitmap, w.words_per_row, (const int *)w.cnt, vhat, p.H,
                                    p.nbr, w.olo, w.llo, w.lo_opart, w.lo_lpart);
        };
        cudaError_t e = p.D == 64 ? run_tc(lowres_pv_tf32_kernel<64>, sizeof(PtSmem<64>))
                                  : run_tc(lowres_pv_tf32_kernel<32>, sizeof(PtSmem<32>));
        if (e != cudaSuccess || nsplit == 1) return e;
        const int rows = p.BH * p.nbr;
        const int mgrid = (rows * (p.D / 4) + 255) / 256;
        return p.D == 64 ? launch_dependent(lowres_pv_merge_kernel<64>, dim3(mgrid), dim3(256), 0, s,
                                            (const float *)w.lo_opart, (const float *)w.lo_lpart, nsplit, rows, w.olo,
                                            w.llo)
                         : launch_dependent(lowres_pv_merge_kernel<32>, dim3(mgrid), dim3(256), 0, s,
                                            (const float *)w.lo_opart, (const float *)w.lo_lpart, nsplit, rows, w.olo,
                                            w.llo);
    }
    return p.D == 64 ? run(lowres_pv_kernel<64>, sizeof(PvSmem<64>)) : run(lowres_pv_kernel<32>, sizeof(PvSmem<32>));
}

}  // namespace mra
