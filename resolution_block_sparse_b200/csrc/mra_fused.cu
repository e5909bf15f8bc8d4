// mra_fused.cu - the whole MRA-2 forward pass of one (batch, head) in one CTA,
// for sequences of at most 16 blocks (512 tokens).
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理", steps one to
// four, as in the multi-kernel path: block means of the valid tokens, the
// low-resolution logits and their row maxima, the selection keys with the
// first-n and diagonal priors, the global top num_block, exact attention on
// the selected blocks and, in full mode, the low-resolution terms of the
// unselected blocks under the shared maximum.
//
// At these sizes the multi-kernel path spends its time in launches and in
// the hand-offs between kernels, not in arithmetic: here the head's Q, K and
// V (at most 192 KB) stay in shared memory from the first step to the last,
// every intermediate lives in shared memory, the top-k is a rank count over
// at most 256 keys, and one launch does the whole pass.  Each CTA works on its
// own head, so no CTA ever waits for another.
#include <cuda_bf16.h>

#include "mra.h"
#include "mra_internal.cuh"
#include "mra_mma.cuh"

namespace mra {
namespace {

using namespace mma;

constexpr int kFMaxRows = 16;                 // block rows (nbr) handled here
constexpr int kFMaxKeys = kFMaxRows * kFMaxRows;
constexpr size_t kFSmemMax = 227 * 1024;      // dynamic + static shared memory per CTA
constexpr float kFLog2e = 1.4426950408889634f;

struct FusedArgs {
    const void *q, *k, *v;
    const float *mask;
    void *out;
    int32_t *sel_out;
    float *logit_out, *pooled_out;
    int H, N, nbr, BH, kk, full, first_n, diag_n;
    float scale, scale_log2;
    long long ob;
    int oh, orow;
    unsigned int *status;
};

// per-head intermediates (static shared memory, about 22 KB)
struct FusedSmem {
    float qh[kFMaxRows][64], kh[kFMaxRows][64], vh[kFMaxRows][64], olo[kFMaxRows][64];
    float lg[kFMaxKeys];
    unsigned long long keys[kFMaxKeys];
    float mlo[kFMaxRows], llo[kFMaxRows], cntf[kFMaxRows];
    unsigned char sel[kFMaxKeys];
    unsigned char cols[kFMaxRows][kFMaxRows];
    int ncol[kFMaxRows];
    int flag;
};

// element (t, d) of a head tensor in shared memory: bf16 tensors are stored
// as swizzled [32][D] tiles (the layout the tensor-core fragments read),
// fp32 tensors row-major
template <typename T, int D>
__device__ __forceinline__ float elem(const T *s, int t, int d) {
    if constexpr (sizeof(T) == 2) {
        const __nv_bfloat16 *p = reinterpret_cast<const __nv_bfloat16 *>(s) + (size_t)(t >> 5) * 32 * D +
                                 swz<D>(t & 31, d >> 3) + (d & 7);
        return __bfloat162float(*p);
    } else {
        return reinterpret_cast<const float *>(s)[(size_t)t * D + d];
    }
}

template <typename T, int D, int NT>
__device__ void load_head(T *dst, const T *src, int N, int tid) {
    if constexpr (sizeof(T) == 2) {
        for (int tile = 0; tile < N / 32; ++tile)
            load_tile_async<D, NT>(reinterpret_cast<__nv_bfloat16 *>(dst) + (size_t)tile * 32 * D,
                                          reinterpret_cast<const __nv_bfloat16 *>(src) + (size_t)tile * 32 * D,
                                          tid);
    } else {
        const int n16 = N * D / 4;
        for (int e = tid; e < n16; e += NT) cp_async16(dst + (size_t)e * 4, src + (size_t)e * 4);
    }
}

// exact attention of the 16 query rows r0 .. r0+15 over the selected blocks
// of their block row (bf16 tensor cores), combined with the low-resolution
// part; one warp
template <int D>
__device__ void attend_slab_bf16(const FusedArgs &a, const FusedSmem &fs, const __nv_bfloat16 *sQ,
                                 const __nv_bfloat16 *sK, const __nv_bfloat16 *sV, const float *smask,
                                 int bh, int br, int half) {
    constexpr int kTile = 32 * D;
    const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const __nv_bfloat16 *qt = sQ + (size_t)br * kTile;
    unsigned qf[D / 16][4];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const int row = half * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = 2 * ks + (lane >> 4);
        ldsm_x4(qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], smem_u32(qt + swz<D>(row, ch)));
    }
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;
    const int ncol = fs.ncol[br];
    for (int j = 0; j < ncol; ++j) {
        const int c = fs.cols[br][j];
        const __nv_bfloat16 *kt = sK + (size_t)c * kTile;
        const __nv_bfloat16 *vt = sV + (size_t)c * kTile;
        float s[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ks += 2) {
                const int key = nt * 8 + (lane & 7);
                const int ch = 2 * ks + (lane >> 3);
                unsigned b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, smem_u32(kt + swz<D>(key, ch)));
                mma16816(s[nt], qf[ks], b0, b1);
                mma16816(s[nt], qf[ks + 1], b2, b3);
            }
        }
        if (smask) {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int kc = c * 32 + nt * 8 + tq * 2;
                if (!(smask[kc] > 0.0f)) s[nt][0] = s[nt][2] = -INFINITY;
                if (!(smask[kc + 1] > 0.0f)) s[nt][1] = s[nt][3] = -INFINITY;
            }
        }
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]));
            mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]));
        }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
        }
        const float mn_a = fmaxf(m_a, mx_a * a.scale_log2), mn_b = fmaxf(m_b, mx_b * a.scale_log2);
        if (mn_a != m_a || mn_b != m_b) {
            const float al_a = (m_a == -INFINITY) ? 0.0f : fast_exp2(m_a - mn_a);
            const float al_b = (m_b == -INFINITY) ? 0.0f : fast_exp2(m_b - mn_b);
            l_a *= al_a;
            l_b *= al_b;
#pragma unroll
            for (int nd = 0; nd < D / 8; ++nd) {
                o[nd][0] *= al_a;
                o[nd][1] *= al_a;
                o[nd][2] *= al_b;
                o[nd][3] *= al_b;
            }
            m_a = mn_a;
            m_b = mn_b;
        }
        const float ref_a = (m_a == -INFINITY) ? 0.0f : m_a;
        const float ref_b = (m_b == -INFINITY) ? 0.0f : m_b;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            s[nt][0] = fast_exp2(fmaf(s[nt][0], a.scale_log2, -ref_a));
            s[nt][1] = fast_exp2(fmaf(s[nt][1], a.scale_log2, -ref_a));
            s[nt][2] = fast_exp2(fmaf(s[nt][2], a.scale_log2, -ref_b));
            s[nt][3] = fast_exp2(fmaf(s[nt][3], a.scale_log2, -ref_b));
            l_a += s[nt][0] + s[nt][1];
            l_b += s[nt][2] + s[nt][3];
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            unsigned pf[4];
            pf[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
            pf[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
            pf[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            pf[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int nd2 = 0; nd2 < D / 16; ++nd2) {
                const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int ch = 2 * nd2 + (lane >> 4);
                unsigned b0, b1, b2, b3;
                ldsm_x4_t(b0, b1, b2, b3, smem_u32(vt + swz<D>(key, ch)));
                mma16816(o[2 * nd2], pf, b0, b1);
                mma16816(o[2 * nd2 + 1], pf, b2, b3);
            }
        }
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
    }
    // combine with the low-resolution part under the shared maximum
    const bool lo = a.full && fs.llo[br] > 0.0f;
    const float m_lo2 = a.full ? fs.mlo[br] * kFLog2e : 0.0f;
    const float l_lo = a.full ? fs.llo[br] : 0.0f;
    const int ta = br * 32 + half * 16 + g, tb = ta + 8;
    auto factors = [&](float m, float l, int t, float &fa, float &fb) {
        fa = fb = 0.0f;
        const bool hi = l > 0.0f;
        float M = hi ? m : -INFINITY;
        if (lo) M = fmaxf(M, m_lo2);
        if (M == -INFINITY || (smask && !(smask[t] > 0.0f))) return;
        const float al = hi ? fast_exp2(m - M) : 0.0f;
        const float be = lo ? fast_exp2(m_lo2 - M) : 0.0f;
        const float den = al * l + be * l_lo;
        if (den > 0.0f) {
            fa = al / den;
            fb = be / den;
        }
    };
    float fa_a, fb_a, fa_b, fb_b;
    factors(m_a, l_a, ta, fa_a, fb_a);
    factors(m_b, l_b, tb, fa_b, fb_b);
    const int b = bh / a.H;
    __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(a.out) + (size_t)b * a.ob + (size_t)(bh - b * a.H) * a.oh;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        const int d = nd * 8 + tq * 2;
        const float ol0 = lo ? fs.olo[br][d] : 0.0f, ol1 = lo ? fs.olo[br][d + 1] : 0.0f;
        *reinterpret_cast<__nv_bfloat162 *>(ob + (size_t)ta * a.orow + d) =
            __floats2bfloat162_rn(fmaf(o[nd][0], fa_a, ol0 * fb_a), fmaf(o[nd][1], fa_a, ol1 * fb_a));
        *reinterpret_cast<__nv_bfloat162 *>(ob + (size_t)tb * a.orow + d) =
            __floats2bfloat162_rn(fmaf(o[nd][2], fa_b, ol0 * fb_b), fmaf(o[nd][3], fa_b, ol1 * fb_b));
    }
}

// the same for one fp32 query row (one thread, FFMA, accurate exp2)
template <int D>
__device__ void attend_row_f32(const FusedArgs &a, const FusedSmem &fs, const float *sQ, const float *sK,
                               const float *sV, const float *smask, int bh, int t) {
    const int br = t >> 5;
    float o[D], qr[D];   // the query row in registers: rows of a warp share a bank
#pragma unroll
    for (int d = 0; d < D; ++d) {
        o[d] = 0.0f;
        qr[d] = sQ[(size_t)t * D + d];
    }
    float m = -INFINITY, l = 0.0f;
    const int ncol = fs.ncol[br];
    for (int j = 0; j < ncol; ++j) {
        const int c = fs.cols[br][j];
        for (int kj = c * 32; kj < c * 32 + 32; ++kj) {
            if (smask && !(smask[kj] > 0.0f)) continue;
            const float *kr = sK + (size_t)kj * D;
            float s = 0.0f;
#pragma unroll
            for (int d = 0; d < D; ++d) s = fmaf(qr[d], kr[d], s);
            const float s2 = s * a.scale_log2;
            const float *vr = sV + (size_t)kj * D;
            if (s2 > m) {
                const float al = (m == -INFINITY) ? 0.0f : exp2f(m - s2);
                l = l * al + 1.0f;
#pragma unroll
                for (int d = 0; d < D; ++d) o[d] = fmaf(o[d], al, vr[d]);
                m = s2;
            } else {
                const float p = exp2f(s2 - m);
                l += p;
#pragma unroll
                for (int d = 0; d < D; ++d) o[d] = fmaf(p, vr[d], o[d]);
            }
        }
    }
    const bool lo = a.full && fs.llo[br] > 0.0f;
    const float m_lo2 = a.full ? fs.mlo[br] * kFLog2e : 0.0f;
    const float l_lo = a.full ? fs.llo[br] : 0.0f;
    float fa = 0.0f, fb = 0.0f;
    {
        const bool hi = l > 0.0f;
        float M = hi ? m : -INFINITY;
        if (lo) M = fmaxf(M, m_lo2);
        if (M != -INFINITY && !(smask && !(smask[t] > 0.0f))) {
            const float al = hi ? exp2f(m - M) : 0.0f;
            const float be = lo ? exp2f(m_lo2 - M) : 0.0f;
            const float den = al * l + be * l_lo;
            if (den > 0.0f) {
                fa = al / den;
                fb = be / den;
            }
        }
    }
    const int b = bh / a.H;
    float *orow = static_cast<float *>(a.out) + (size_t)b * a.ob + (size_t)(bh - b * a.H) * a.oh +
                  (size_t)t * a.orow;
#pragma unroll
    for (int d = 0; d < D; ++d) orow[d] = fmaf(o[d], fa, (lo ? fs.olo[br][d] : 0.0f) * fb);
}

// NT threads: 512 for bf16 (16 warps share the head's 32 query slabs), 256
// for fp32 (one thread per query row, many registers)
template <typename T, int D, int NT>
__global__ void __launch_bounds__(NT)
fused_small_kernel(FusedArgs a) {
    extern __shared__ __align__(128) unsigned char fdyn[];
    __shared__ FusedSmem fs;
    pdl_wait();
    const int bh = blockIdx.x, tid = threadIdx.x;
    const int N = a.N, nbr = a.nbr, nk = nbr * nbr;
    const int b = bh / a.H;
    const size_t tb = (size_t)N * D * sizeof(T);
    T *sQ = reinterpret_cast<T *>(fdyn);
    T *sK = reinterpret_cast<T *>(fdyn + tb);
    T *sV = reinterpret_cast<T *>(fdyn + 2 * tb);
    float *smask = a.mask ? reinterpret_cast<float *>(fdyn + 3 * tb) : nullptr;
    const size_t head_off = (size_t)bh * N * D;

    // ------------------------------------------------ the head into shared memory
    load_head<T, D, NT>(sQ, static_cast<const T *>(a.q) + head_off, N, tid);
    load_head<T, D, NT>(sK, static_cast<const T *>(a.k) + head_off, N, tid);
    load_head<T, D, NT>(sV, static_cast<const T *>(a.v) + head_off, N, tid);
    cp_async_commit();
    if (smask)
        for (int t = tid; t < N; t += NT) smask[t] = a.mask[(size_t)b * N + t];
    if (tid == 0) fs.flag = 0;
    cp_async_wait<0>();
    __syncthreads();

    // ------------------------------------------------ step one: block means, counts
    for (int p = tid; p < nbr * D; p += NT) {
        const int br = p / D, d = p - br * D;
        float c = 0.0f, sq = 0.0f, sk = 0.0f, sv = 0.0f;
        for (int r = 0; r < 32; ++r) {
            const int t = br * 32 + r;
            const float m = smask ? smask[t] : 1.0f;
            c += m;
            sq = fmaf(m, elem<T, D>(sQ, t, d), sq);
            sk = fmaf(m, elem<T, D>(sK, t, d), sk);
            if (a.full) sv = fmaf(m, elem<T, D>(sV, t, d), sv);
        }
        fs.qh[br][d] = c > 0.0f ? sq / c : 0.0f;
        fs.kh[br][d] = c > 0.0f ? sk / c : 0.0f;
        fs.vh[br][d] = (a.full && c > 0.0f) ? sv / c : 0.0f;
        if (d == 0) fs.cntf[br] = c;
    }
    __syncthreads();
    if (a.pooled_out) {
        const size_t plane = (size_t)a.BH * nbr * D;
        for (int p = tid; p < nbr * D; p += NT) {
            const int br = p / D, d = p - br * D;
            const size_t i = ((size_t)bh * nbr + br) * D + d;
            a.pooled_out[i] = fs.qh[br][d];
            a.pooled_out[plane + i] = fs.kh[br][d];
            a.pooled_out[2 * plane + i] = fs.vh[br][d];
        }
    }
    // ------------------------------------------------ low-resolution logits
    if (tid < nk) {
        const int r = tid / nbr, c = tid - r * nbr;
        float s = 0.0f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) s = fmaf(fs.qh[r][d], fs.kh[c][d], s);
        fs.lg[tid] = s * a.scale;
        if (a.logit_out) a.logit_out[(size_t)bh * nk + tid] = s * a.scale;
    }
    __syncthreads();
    // ------------------------------------------------ step two: row max, keys
    if (tid < nk) {
        const int r = tid / nbr, c = tid - r * nbr;
        float m = -INFINITY;
        for (int cc = 0; cc < nbr; ++cc)
            if (fs.cntf[cc] > 0.0f) m = fmaxf(m, fs.lg[r * nbr + cc]);
        if (m == -INFINITY) m = 0.0f;
        if (c == 0) fs.mlo[r] = m;
        int range_err = 0;
        fs.keys[tid] = selection_key(fs.lg[tid], m, r, c, a.first_n, a.diag_n, !(fs.cntf[r] > 0.0f),
                                     !(fs.cntf[c] > 0.0f), range_err);
        if (range_err) fs.flag = 1;
    }
    __syncthreads();
    // ------------------------------------------------ global top-k: rank count, ties to the smaller index
    if (tid < nk) {
        const unsigned long long key = fs.keys[tid];
        int rank = 0;
        for (int j = 0; j < nk; ++j) {
            const unsigned long long kj = fs.keys[j];
            rank += (kj > key || (kj == key && j < tid)) ? 1 : 0;
        }
        fs.sel[tid] = rank < a.kk ? 1 : 0;
    }
    __syncthreads();
    if (a.sel_out && tid < nk && fs.sel[tid]) {
        int pos = 0;
        for (int j = 0; j < tid; ++j) pos += fs.sel[j];
        a.sel_out[(size_t)bh * a.kk + pos] = tid;
    }
    if (tid < nbr) {
        int n = 0;
        for (int c = 0; c < nbr; ++c)
            if (fs.sel[tid * nbr + c]) fs.cols[tid][n++] = (unsigned char)c;
        fs.ncol[tid] = n;
    }
    if (tid == 0 && fs.flag) atomicOr(a.status, kDevKeyRange);
    // ------------------------------------------------ step four (full mode): low-resolution terms
    if (a.full) {
        for (int p = tid; p < nbr * D; p += NT) {
            const int r = p / D, d = p - r * D;
            float acc = 0.0f, lsum = 0.0f;
            for (int c = 0; c < nbr; ++c) {
                const float cn = fs.cntf[c];
                if (!(cn > 0.0f) || fs.sel[r * nbr + c]) continue;
                const float w = cn * expf(fs.lg[r * nbr + c] - fs.mlo[r]);
                acc = fmaf(w, fs.vh[c][d], acc);
                lsum += w;
            }
            fs.olo[r][d] = acc;
            if (d == 0) fs.llo[r] = lsum;
        }
    }
    __syncthreads();
    // ------------------------------------------------ step three: exact attention on the selected blocks
    if constexpr (sizeof(T) == 2) {
        const int warp = tid >> 5;
        for (int slab = warp; slab < 2 * nbr; slab += NT / 32)
            attend_slab_bf16<D>(a, fs, reinterpret_cast<const __nv_bfloat16 *>(sQ),
                                reinterpret_cast<const __nv_bfloat16 *>(sK),
                                reinterpret_cast<const __nv_bfloat16 *>(sV), smask, bh, slab >> 1, slab & 1);
    } else {
        for (int t = tid; t < N; t += NT)
            attend_row_f32<D>(a, fs, reinterpret_cast<const float *>(sQ), reinterpret_cast<const float *>(sK),
                              reinterpret_cast<const float *>(sV), smask, bh, t);
    }
}

size_t fused_dyn_smem(const Problem &p) {
    const size_t esz = p.dtype == 0 ? 2 : 4;
    return 3 * (size_t)p.N * p.D * esz + sizeof(float) * (size_t)p.N;
}

template <typename T, int D>
cudaError_t launch_fused_typed(const Problem &p, const FusedArgs &a, cudaStream_t s) {
    constexpr int NT = sizeof(T) == 2 ? 512 : 256;
    const size_t smem = fused_dyn_smem(p);
    auto kern = fused_small_kernel<T, D, NT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_dependent(kern, dim3((unsigned)p.BH), dim3(NT), smem, s, a);
}

}  // namespace

bool fused_small_supported(const Problem &p) {
    if (p.nbr > kFMaxRows) return false;
    return fused_dyn_smem(p) + sizeof(FusedSmem) <= kFSmemMax;
}

bool fused_small_preferred(const Problem &p) {
    // one CTA per head holds its whole pass: faster than the multi-kernel
    // path once there are enough heads to occupy most SMs, and for bf16,
    // whose attention runs on the tensor cores
    return p.dtype == 0 && p.BH >= 64;
}

cudaError_t launch_fused_small(const Problem &p, const Workspace &w, const void *q, const void *k, const void *v,
                               const float *mask, void *out, int32_t *sel_out, float *logit_out, float *pooled_out,
                               const OutLayout *ol, cudaStream_t s) {
    FusedArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.mask = mask;
    a.out = out;
    a.sel_out = sel_out;
    a.logit_out = logit_out;
    a.pooled_out = pooled_out;
    a.H = p.H;
    a.N = p.N;
    a.nbr = p.nbr;
    a.BH = p.BH;
    a.kk = p.k;
    a.full = p.mode == 0 ? 1 : 0;
    a.first_n = p.first_n;
    a.diag_n = p.diag_n;
    a.scale = 1.0f / sqrtf((float)p.D);
    a.scale_log2 = kFLog2e / sqrtf((float)p.D);
    if (ol) {
        a.ob = ol->ob;
        a.oh = ol->oh;
        a.orow = ol->orow;
    } else {
        a.ob = (long long)p.H * p.N * p.D;
        a.oh = p.N * p.D;
        a.orow = p.D;
    }
    a.status = w.status;
    if (p.dtype == 0)
        return p.D == 64 ? launch_fused_typed<__nv_bfloat16, 64>(p, a, s) : launch_fused_typed<__nv_bfloat16, 32>(p, a, s);
    return p.D == 64 ? launch_fused_typed<float, 64>(p, a, s) : launch_fused_typed<float, 32>(p, a, s);
}

}  // namespace mra
