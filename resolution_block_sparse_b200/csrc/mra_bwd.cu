// mra_bwd.cu - backward pass: gradients of the forward output with respect to
// Q, K and V, with the selected blocks held fixed.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理":
//   step three - the sampled-dense products are autograd functions whose
//                backward reuses the forward's kernels through transposed
//                block indices, so the model trains end to end;
//   step four  - in sparse mode the low-resolution branch only picks blocks
//                (no gradient); in full mode its output is part of the result
//                and the gradient flows through the block means of Q, K, V.
//
// With p the softmax weights of a query row i (high- and low-resolution terms
// under one normaliser), lse2_i the base-2 log-sum-exp and delta_i = dO_i.O_i,
// both exported by the forward kernels:
//   high resolution, selected block (r, c), query i in r, key j in c:
//     p_ij = 2^(s_ij log2e - lse2_i),  ds_ij = p_ij (dO_i.v_j - delta_i)
//     dQ_i += ds_ij k_j / sqrt(D),  dK_j += ds_ij q_i / sqrt(D),  dV_j += p_ij dO_i
//   low resolution (full mode), unselected block c with cnt_c > 0, row block b:
//     W_bc = cnt_c 2^(l_bc log2e - R_b),  A_b = sum_i 2^(R_b - lse2_i) dO_i,
//     B_b = sum_i 2^(R_b - lse2_i) delta_i  (R_b: the smallest lse2 of b)
//     dl_bc = W_bc (vhat_c.A_b - B_b),  dvhat_c += W_bc A_b,
//     dqhat_b += dl_bc khat_c / sqrt(D),  dkhat_c += dl_bc qhat_b / sqrt(D)
//   and every valid token of a block takes its block mean's gradient / cnt.
//
// Kernels: bwd_item (one CTA per forward work item: dQ of its rows in
// registers, dK and dV of its key blocks added with vector fp32 atomics, the
// transposed index traversal being the atomics' addresses), and in full mode,
// launched before bwd_item, lowres_bwd_prep (A, B, R per row block; clears
// the block-mean gradient planes), lowres_bwd_tile (one CTA per 64 x 64 tile
// of (row block, key block) pairs: dl in shared memory, dqhat, dkhat and
// dvhat partial sums from 4 x 4 register tiles added with fp32 atomics) and
// lowres_bwd_scatter (block means to tokens; writes dQ, dK, dV, which the
// item kernel then adds to). All arithmetic is fp32 (FFMA).
#include <cuda_bf16.h>

#include <algorithm>

#include "mra_internal.cuh"
#include "mra_mma.cuh"

namespace mra {
namespace {

constexpr float kLog2eB = 1.4426950408889634f;
constexpr int kBwdThreads = 128;   // four threads per query row

template <typename T>
__device__ __forceinline__ float ldf(const T *p, size_t i);
template <>
__device__ __forceinline__ float ldf<float>(const float *p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

__device__ __forceinline__ void atomic_add4(float *p, float4 v) {
    atomicAdd(reinterpret_cast<float4 *>(p), v);
}

struct BwdArgs {
    const void *q, *k, *v, *dout;
    const float *mask;
    const WorkItem *items;
    const int *head_items;
    const int *cols;
    int cap, H, N, nbr;
    float scale, scale_log2;
    const float *lse2, *delta;
    float *dq, *dk, *dv;
};

// One work item (block row r, up to `chunk` selected key blocks).
template <typename T, int D>
__global__ void __launch_bounds__(kBwdThreads)
bwd_item_kernel(const BwdArgs a) {
    pdl_wait();
    constexpr int kDp = D / 4;
    __shared__ __align__(16) float sQ[32][D];
    __shared__ __align__(16) float sG[32][D];   // dO of the row block
    __shared__ __align__(16) float sK[32][D];
    __shared__ __align__(16) float sV[32][D];
    __shared__ float sP[32][33], sS[32][33];     // p and ds, [query][key]
    __shared__ float sKm[32];

    const int slot = blockIdx.x;
    const int bh = slot / a.cap, local = slot % a.cap;
    if (local >= a.head_items[bh]) return;
    const WorkItem it = a.items[slot];
    if (it.ncols <= 0) return;
    const int r = it.row % a.nbr;
    const int b = bh / a.H;
    const size_t head = (size_t)bh * a.N;
    const T *qg = static_cast<const T *>(a.q) + head * D;
    const T *kg = static_cast<const T *>(a.k) + head * D;
    const T *vg = static_cast<const T *>(a.v) + head * D;
    const T *gg = static_cast<const T *>(a.dout) + head * D;
    const float *mrow = a.mask ? a.mask + (size_t)b * a.N : nullptr;
    const int tid = threadIdx.x, qrow = tid >> 2, part = tid & 3, d0 = part * kDp;
    const size_t qi = (size_t)r * 32 + qrow;

    for (int e = tid; e < 32 * D; e += kBwdThreads) {
        sQ[e / D][e % D] = ldf(qg, (size_t)r * 32 * D + e);
        sG[e / D][e % D] = ldf(gg, (size_t)r * 32 * D + e);
    }
    const float lse2 = a.lse2[head + qi];   // +inf: the row's output is a constant
    const float dlt = a.delta[head + qi];
    float dq[kDp];
#pragma unroll
    for (int i = 0; i < kDp; ++i) dq[i] = 0.0f;

    for (int j = 0; j < it.ncols; ++j) {
        const int c = a.cols[it.col_start + j];
        __syncthreads();   // previous tile consumed (and sQ / sG written)
        for (int e = tid; e < 32 * D; e += kBwdThreads) {
            sK[e / D][e % D] = ldf(kg, (size_t)c * 32 * D + e);
            sV[e / D][e % D] = ldf(vg, (size_t)c * 32 * D + e);
        }
        if (tid < 32) sKm[tid] = mrow ? mrow[c * 32 + tid] : 1.0f;
        __syncthreads();
        for (int kj = 0; kj < 32; ++kj) {
            float s = 0.0f, dp = 0.0f;
#pragma unroll
            for (int i = 0; i < kDp; ++i) {
                s = fmaf(sQ[qrow][d0 + i], sK[kj][d0 + i], s);
                dp = fmaf(sG[qrow][d0 + i], sV[kj][d0 + i], dp);
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            dp += __shfl_xor_sync(0xffffffffu, dp, 2);
            const float p = (sKm[kj] > 0.0f) ? exp2f(fmaf(s, a.scale_log2, -lse2)) : 0.0f;
            const float ds = p * (dp - dlt);
            if (part == 0) {
                sP[qrow][kj] = p;
                sS[qrow][kj] = ds;
            }
            const float w = ds * a.scale;
#pragma unroll
            for (int i = 0; i < kDp; ++i) dq[i] = fmaf(w, sK[kj][d0 + i], dq[i]);
        }
        __syncthreads();
        // key kj = tid / 4 of block c: dK and dV over the 32 query rows
        {
            const int kj = tid >> 2;
            float dk[kDp], dv[kDp];
#pragma unroll
            for (int i = 0; i < kDp; ++i) dk[i] = dv[i] = 0.0f;
            for (int qr = 0; qr < 32; ++qr) {
                const float ds = sS[qr][kj] * a.scale, p = sP[qr][kj];
#pragma unroll
                for (int i = 0; i < kDp; ++i) {
                    dk[i] = fmaf(ds, sQ[qr][d0 + i], dk[i]);
                    dv[i] = fmaf(p, sG[qr][d0 + i], dv[i]);
                }
            }
            float *dkr = a.dk + (head + (size_t)c * 32 + kj) * D + d0;
            float *dvr = a.dv + (head + (size_t)c * 32 + kj) * D + d0;
#pragma unroll
            for (int i = 0; i < kDp; i += 4) {
                atomic_add4(dkr + i, make_float4(dk[i], dk[i + 1], dk[i + 2], dk[i + 3]));
                atomic_add4(dvr + i, make_float4(dv[i], dv[i + 1], dv[i + 2], dv[i + 3]));
            }
        }
    }
    float *dqr = a.dq + (head + qi) * D + d0;
#pragma unroll
    for (int i = 0; i < kDp; i += 4) atomic_add4(dqr + i, make_float4(dq[i], dq[i + 1], dq[i + 2], dq[i + 3]));
}

// The same work item on the tensor cores (bf16 inputs, warp-level
// mma.sync m16n8k16, fp32 accumulation), two warps of 16 query rows:
//   S = Q K^T and dP = dO V^T from ldmatrix fragments (as in the forward),
//   P and dS in fp32 registers, dQ += dS K with dS packed to bf16 in
//   registers, then (from bf16 copies of P and dS in shared memory, read
//   transposed by ldmatrix.trans) dK = dS^T Q and dV = P^T dO with each warp
//   owning 16 of the block's keys.  dK, dV and finally dQ are staged in
//   shared memory and added to global memory with float4 atomics.
constexpr int kMmaThreads = 64;
constexpr int kPS = 40;   // row stride (bf16) of the P and dS tiles: 80 bytes, conflict-free ldmatrix

template <int D>
struct BwdMmaSmem {
    static constexpr int kTile = 32 * D;
    __nv_bfloat16 q[kTile], g[kTile];     // Q and dO of the row block, swizzled
    __nv_bfloat16 kv[2][2][kTile];        // K/V double buffer, swizzled
    __nv_bfloat16 p[32 * kPS], ds[32 * kPS];   // [query][key]
    float stage[32][D + 4];               // fp32 staging of a 32 x D gradient tile
    float km[2][32];
    int cols[kChunk];
};

template <int D>
__device__ __forceinline__ void add_stage_atomic(float (*stage)[D + 4], float *gbase, int tid) {
    // gbase: row 0 of the 32 x D gradient tile in global memory
    for (int e = tid; e < 32 * D / 4; e += kMmaThreads) {
        const int row = e / (D / 4), c4 = (e % (D / 4)) * 4;
        atomic_add4(gbase + (size_t)row * D + c4, *reinterpret_cast<const float4 *>(&stage[row][c4]));
    }
}

template <int D>
__global__ void __launch_bounds__(kMmaThreads)
bwd_item_mma_kernel(const BwdArgs a) {
    using namespace mma;
    pdl_wait();
    constexpr int kTile = 32 * D;
    __shared__ __align__(128) BwdMmaSmem<D> sh;
    const int slot = blockIdx.x;
    const int bh = slot / a.cap, local = slot % a.cap;
    if (local >= a.head_items[bh]) return;
    const WorkItem it = a.items[slot];
    if (it.ncols <= 0) return;
    const int r = it.row % a.nbr;
    const int b = bh / a.H;
    const size_t head = (size_t)bh * a.N;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q) + head * D;
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(a.k) + head * D;
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(a.v) + head * D;
    const __nv_bfloat16 *gg = static_cast<const __nv_bfloat16 *>(a.dout) + head * D;
    const float *mrow = a.mask ? a.mask + (size_t)b * a.N : nullptr;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int ra = warp * 16 + g, rb = ra + 8;   // this thread's query rows (C fragments)

    load_tile_async<D, kMmaThreads>(sh.q, qg + (size_t)r * kTile, tid);
    load_tile_async<D, kMmaThreads>(sh.g, gg + (size_t)r * kTile, tid);
    const int ncols = it.ncols;
    for (int j = tid; j < ncols; j += kMmaThreads) sh.cols[j] = a.cols[it.col_start + j];
    __syncthreads();
    {
        const int c0 = sh.cols[0];
        load_tile_async<D, kMmaThreads>(sh.kv[0][0], kg + (size_t)c0 * kTile, tid);
        load_tile_async<D, kMmaThreads>(sh.kv[0][1], vg + (size_t)c0 * kTile, tid);
        if (tid < 32) sh.km[0][tid] = mrow ? mrow[c0 * 32 + tid] : 1.0f;
    }
    cp_async_commit();
    const float lse_a = a.lse2[head + (size_t)r * 32 + ra], lse_b = a.lse2[head + (size_t)r * 32 + rb];
    const float dl_a = a.delta[head + (size_t)r * 32 + ra], dl_b = a.delta[head + (size_t)r * 32 + rb];

    float dq[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.0f;
    unsigned qf[D / 16][4], gf[D / 16][4];

    for (int j = 0; j < ncols; ++j) {
        const int buf = j & 1;
        if (j + 1 < ncols) {
            const int c1 = sh.cols[j + 1];
            load_tile_async<D, kMmaThreads>(sh.kv[buf ^ 1][0], kg + (size_t)c1 * kTile, tid);
            load_tile_async<D, kMmaThreads>(sh.kv[buf ^ 1][1], vg + (size_t)c1 * kTile, tid);
            if (tid < 32) sh.km[buf ^ 1][tid] = mrow ? mrow[c1 * 32 + tid] : 1.0f;
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (j == 0) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int ch = 2 * ks + (lane >> 4);
                ldsm_x4(qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], smem_u32(sh.q + swz<D>(row, ch)));
                ldsm_x4(gf[ks][0], gf[ks][1], gf[ks][2], gf[ks][3], smem_u32(sh.g + swz<D>(row, ch)));
            }
        }
        const int c = sh.cols[j];
        const __nv_bfloat16 *sK = sh.kv[buf][0];
        const __nv_bfloat16 *sV = sh.kv[buf][1];
        // S = Q K^T and dP = dO V^T for this warp's 16 rows x 32 keys
        float sc[4][4], dp[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[nt][e] = dp[nt][e] = 0.0f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ks += 2) {
                const int key = nt * 8 + (lane & 7);
                const int ch = 2 * ks + (lane >> 3);
                unsigned b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, smem_u32(sK + swz<D>(key, ch)));
                mma16816(sc[nt], qf[ks], b0, b1);
                mma16816(sc[nt], qf[ks + 1], b2, b3);
                ldsm_x4(b0, b1, b2, b3, smem_u32(sV + swz<D>(key, ch)));
                mma16816(dp[nt], gf[ks], b0, b1);
                mma16816(dp[nt], gf[ks + 1], b2, b3);
            }
        }
        // P = 2^(s scale log2e - lse2), dS = P (dP - delta); both to shared memory (bf16)
        unsigned pk[4][2], dk_[4][2];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int kc = nt * 8 + tq * 2;
            const bool v0 = sh.km[buf][kc] > 0.0f, v1 = sh.km[buf][kc + 1] > 0.0f;
            const float p0 = v0 ? fast_exp2(fmaf(sc[nt][0], a.scale_log2, -lse_a)) : 0.0f;
            const float p1 = v1 ? fast_exp2(fmaf(sc[nt][1], a.scale_log2, -lse_a)) : 0.0f;
            const float p2 = v0 ? fast_exp2(fmaf(sc[nt][2], a.scale_log2, -lse_b)) : 0.0f;
            const float p3 = v1 ? fast_exp2(fmaf(sc[nt][3], a.scale_log2, -lse_b)) : 0.0f;
            const float d0v = p0 * (dp[nt][0] - dl_a), d1v = p1 * (dp[nt][1] - dl_a);
            const float d2v = p2 * (dp[nt][2] - dl_b), d3v = p3 * (dp[nt][3] - dl_b);
            pk[nt][0] = pack_bf16(p0, p1);
            pk[nt][1] = pack_bf16(p2, p3);
            dk_[nt][0] = pack_bf16(d0v, d1v);
            dk_[nt][1] = pack_bf16(d2v, d3v);
            *reinterpret_cast<unsigned *>(&sh.p[ra * kPS + kc]) = pk[nt][0];
            *reinterpret_cast<unsigned *>(&sh.p[rb * kPS + kc]) = pk[nt][1];
            *reinterpret_cast<unsigned *>(&sh.ds[ra * kPS + kc]) = dk_[nt][0];
            *reinterpret_cast<unsigned *>(&sh.ds[rb * kPS + kc]) = dk_[nt][1];
        }
        // dQ += dS K  (A = dS from registers, B = K read transposed, k = key)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            unsigned af[4] = {dk_[2 * kk][0], dk_[2 * kk][1], dk_[2 * kk + 1][0], dk_[2 * kk + 1][1]};
#pragma unroll
            for (int nd2 = 0; nd2 < D / 16; ++nd2) {
                const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int ch = 2 * nd2 + (lane >> 4);
                unsigned b0, b1, b2, b3;
                ldsm_x4_t(b0, b1, b2, b3, smem_u32(sK + swz<D>(key, ch)));
                mma16816(dq[2 * nd2], af, b0, b1);
                mma16816(dq[2 * nd2 + 1], af, b2, b3);
            }
        }
        __syncthreads();   // P and dS of both warps in shared memory
        // dK = dS^T Q, then dV = P^T dO: this warp's keys 16 warp .. +15
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            const __nv_bfloat16 *src = which == 0 ? sh.ds : sh.p;
            const __nv_bfloat16 *rhs = which == 0 ? sh.q : sh.g;
            float acc[D / 8][4];
#pragma unroll
            for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
#pragma unroll
            for (int kq = 0; kq < 2; ++kq) {
                // A (16 keys x 16 queries) = src^T: matrix i of the x4 load
                // takes rows q = 16 kq + (i / 2) 8 + lane % 8 at key offset (i % 2) 8
                unsigned af[4];
                {
                    const int i = lane >> 3;
                    const int qr = 16 * kq + (i >> 1) * 8 + (lane & 7);
                    const int key = warp * 16 + (i & 1) * 8;
                    ldsm_x4_t(af[0], af[1], af[2], af[3], smem_u32(src + qr * kPS + key));
                }
#pragma unroll
                for (int nd2 = 0; nd2 < D / 16; ++nd2) {
                    const int qrow = kq * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int ch = 2 * nd2 + (lane >> 4);
                    unsigned b0, b1, b2, b3;
                    ldsm_x4_t(b0, b1, b2, b3, smem_u32(rhs + swz<D>(qrow, ch)));
                    mma16816(acc[2 * nd2], af, b0, b1);
                    mma16816(acc[2 * nd2 + 1], af, b2, b3);
                }
            }
            const float f = which == 0 ? a.scale : 1.0f;
            const int ka = warp * 16 + g, kb = ka + 8;
#pragma unroll
            for (int nd = 0; nd < D / 8; ++nd) {
                const int d = nd * 8 + tq * 2;
                *reinterpret_cast<float2 *>(&sh.stage[ka][d]) = make_float2(acc[nd][0] * f, acc[nd][1] * f);
                *reinterpret_cast<float2 *>(&sh.stage[kb][d]) = make_float2(acc[nd][2] * f, acc[nd][3] * f);
            }
            __syncthreads();
            add_stage_atomic<D>(sh.stage, (which == 0 ? a.dk : a.dv) + (head + (size_t)c * 32) * D, tid);
            __syncthreads();
        }
    }
    // dQ of the item's rows
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        const int d = nd * 8 + tq * 2;
        *reinterpret_cast<float2 *>(&sh.stage[ra][d]) = make_float2(dq[nd][0] * a.scale, dq[nd][1] * a.scale);
        *reinterpret_cast<float2 *>(&sh.stage[rb][d]) = make_float2(dq[nd][2] * a.scale, dq[nd][3] * a.scale);
    }
    __syncthreads();
    add_stage_atomic<D>(sh.stage, a.dq + (head + (size_t)r * 32) * D, tid);
}

// ------------------------------------------------------------------ low resolution (full mode)

struct LoArgs {
    const void *dout;
    const float *lse2, *delta;
    const float *qhat, *khat, *vhat;   // [BH][nbr][D]
    const int *cnt;                    // [B][nbr]
    const unsigned int *bitmap;        // selected blocks, [BH*nbr][wpr]
    int wpr, H, N, nbr;
    float scale;
    float *ab;                         // [BH*nbr][D + 4]: A (D), B, R, valid
    float *dxh;                        // [3][BH][nbr][D]: dqhat, dkhat, dvhat
};

// A_b, B_b, R_b of one row block per warp (lane i holds query i of the
// block for the weights, dims lane + 32 e for A), and the block's rows of
// the three block-mean gradient planes set to zero.
constexpr int kPrepWarps = 8;

template <typename T, int D>
__global__ void __launch_bounds__(32 * kPrepWarps)
lowres_bwd_prep_kernel(const LoArgs a, int nrb) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int rb = blockIdx.x * kPrepWarps + (threadIdx.x >> 5);   // bh * nbr + b
    if (rb >= nrb) return;
    const int bh = rb / a.nbr, b = rb % a.nbr;
    const size_t q0 = (size_t)bh * a.N + (size_t)b * 32;
    const float l = a.lse2[q0 + lane];
    const float dl = a.delta[q0 + lane];
    float m = l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fminf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float wl = (l == INFINITY) ? 0.0f : exp2f(m - l);
    float bsum = wl * dl;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bsum += __shfl_xor_sync(0xffffffffu, bsum, o);
    constexpr int E = D / 32;
    const T *g = static_cast<const T *>(a.dout) + q0 * D;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.0f;
#pragma unroll 8
    for (int i = 0; i < 32; ++i) {
        const float wi = __shfl_sync(0xffffffffu, wl, i);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(wi, ldf(g, (size_t)i * D + lane + 32 * e), acc[e]);
    }
    float *out = a.ab + (size_t)rb * (D + 4);
    const size_t plane = (size_t)nrb * D;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int d = lane + 32 * e;
        out[d] = acc[e];
        a.dxh[(size_t)rb * D + d] = 0.0f;
        a.dxh[plane + (size_t)rb * D + d] = 0.0f;
        a.dxh[2 * plane + (size_t)rb * D + d] = 0.0f;
    }
    if (lane == 0) {
        out[D] = bsum;
        out[D + 1] = m;
        out[D + 2] = (m == INFINITY) ? 0.0f : 1.0f;   // the row block has a query with terms
    }
}

// The low-resolution gradient on 64 x 64 tiles of (row block b, key block c)
// pairs, one CTA per tile.  The CTA stages Q-hat and A of its 64 row blocks
// and K-hat and V-hat of its 64 key blocks in shared memory and forms
//   lg_bc = qhat_b . khat_c,  va_bc = vhat_c . A_b
//   W_bc  = cnt_c 2^(lg_bc scale log2e - R_b)  for an unselected pair with a
//           valid column and a row block that has a query with terms, else 0
//   dl_bc = W_bc (va_bc - B_b)
// once, then the tile's shares of the three sums
//   dqhat_b = scale sum_c dl_bc khat_c,  dkhat_c = scale sum_b dl_bc qhat_b,
//   dvhat_c = sum_b W_bc A_b
// which it adds into the block-mean gradient planes (zeroed by the prep
// kernel) with vector atomics.  Every product is an outer product of 4 x 4
// register tiles: thread (tx, ty) of 16 x 16 holds rows ty + 16 i and
// columns tx + 16 j of the tile, so a warp's row loads are 16 consecutive
// rows of a padded [64][D + 4] array (two wavefronts) and its column loads
// broadcast.  fp32 FFMA throughout.
constexpr int kLoT = 64;                 // blocks per tile side
constexpr int kLoThreads = 256;
constexpr int kLoP = kLoT + 4;           // padded row of the tile's pair arrays

template <int D>
struct LoTileSmem {
    float q[kLoT][D + 4];        // Q-hat of the tile's row blocks
    float a[kLoT][D + 4];        // A of the row blocks
    float k[kLoT][D + 4];        // K-hat of the key blocks
    union {
        float v[kLoT][D + 4];    // V-hat of the key blocks, then
        float wt[kLoT][kLoP];    // W [c][b] once the weights are formed
    };
    float dl[kLoT][kLoP];        // dl [b][c]
    float dlt[kLoT][kLoP];       // dl [c][b]
    float rb[kLoT], rbb[kLoT], rvalid[kLoT];   // R, B and validity of the row blocks
    float cntc[kLoT];                           // column counts (0 past nbr)
    unsigned long long sel[kLoT];               // selected bits of each row over the tile's columns
};

// 64 rows of [nbr][stride] starting at row0 into dst by cp.async (zeros
// past nbr); the caller commits and waits.
template <int D>
__device__ __forceinline__ void lo_stage(float (*dst)[D + 4], const float *src, int row0, int nbr, size_t stride,
                                         int t) {
#pragma unroll
    for (int i = t; i < kLoT * D / 4; i += kLoThreads) {
        const int r = i / (D / 4), d4 = i % (D / 4);
        if (row0 + r < nbr)
            mma::cp_async16(&dst[r][4 * d4], src + (size_t)(row0 + r) * stride + 4 * d4);
        else
            *reinterpret_cast<float4 *>(&dst[r][4 * d4]) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// acc[i][*] += sum over u of x[ri][u] * y[u][d0..d0+DW), ri = ty + 16 i; x is
// a [64][kLoP] pair array, y a [64][D + 4] operand; DW = D / 16 dims.
template <int D>
__device__ __forceinline__ void lo_accumulate(float (&acc)[4][D / 16], const float (*x)[kLoP],
                                              const float (*y)[D + 4], int ty, int d0) {
    constexpr int DW = D / 16;
#pragma unroll 2
    for (int u = 0; u < kLoT; u += 4) {
        float4 xr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xr[i] = *reinterpret_cast<const float4 *>(&x[ty + 16 * i][u]);
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
            float yv[DW];
            if constexpr (DW == 4) {
                const float4 y4 = *reinterpret_cast<const float4 *>(&y[u + uu][d0]);
                yv[0] = y4.x; yv[1] = y4.y; yv[2] = y4.z; yv[3] = y4.w;
            } else {
                const float2 y2 = *reinterpret_cast<const float2 *>(&y[u + uu][d0]);
                yv[0] = y2.x; yv[1] = y2.y;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float xv = uu == 0 ? xr[i].x : (uu == 1 ? xr[i].y : (uu == 2 ? xr[i].z : xr[i].w));
#pragma unroll
                for (int e = 0; e < DW; ++e) acc[i][e] = fmaf(xv, yv[e], acc[i][e]);
            }
        }
    }
}

// Adds scale * acc[i] to rows row0 + ty + 16 i (those below nbr) of the
// plane [nbr][D] at dst.
template <int D>
__device__ __forceinline__ void lo_flush(float *dst, const float (&acc)[4][D / 16], int row0, int nbr, int ty,
                                         int d0, float scale) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty + 16 * i;
        if (r >= nbr) continue;
        float *p = dst + (size_t)r * D + d0;
        if constexpr (D / 16 == 4) {
            atomic_add4(p, make_float4(acc[i][0] * scale, acc[i][1] * scale, acc[i][2] * scale, acc[i][3] * scale));
        } else {
            atomicAdd(reinterpret_cast<float2 *>(p), make_float2(acc[i][0] * scale, acc[i][1] * scale));
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kLoThreads, 2)
lowres_bwd_tile_kernel(const LoArgs a, int BH) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char lo_smem[];
    LoTileSmem<D> &sh = *reinterpret_cast<LoTileSmem<D> *>(lo_smem);
    const int col0 = blockIdx.x * kLoT, row0 = blockIdx.y * kLoT, bh = blockIdx.z;
    const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
    const size_t head = (size_t)bh * a.nbr * D;
    lo_stage<D>(sh.q, a.qhat + head, row0, a.nbr, D, t);
    lo_stage<D>(sh.a, a.ab + (size_t)bh * a.nbr * (D + 4), row0, a.nbr, D + 4, t);
    lo_stage<D>(sh.k, a.khat + head, col0, a.nbr, D, t);
    lo_stage<D>(sh.v, a.vhat + head, col0, a.nbr, D, t);
    mma::cp_async_commit();
    if (t < kLoT) {
        const int r = row0 + t;
        const bool ok = r < a.nbr;
        const float *ab = a.ab + ((size_t)bh * a.nbr + (ok ? r : 0)) * (D + 4);
        sh.rbb[t] = ok ? ab[D] : 0.0f;
        sh.rb[t] = ok ? ab[D + 1] : 0.0f;
        sh.rvalid[t] = ok ? ab[D + 2] : 0.0f;
        unsigned long long bits = ~0ull;
        if (ok) {
            const unsigned int *row = a.bitmap + ((size_t)bh * a.nbr + r) * a.wpr;
            const int w0 = col0 >> 5;   // col0 is a multiple of 64
            bits = (unsigned long long)row[w0];
            bits |= (unsigned long long)(w0 + 1 < a.wpr ? row[w0 + 1] : ~0u) << 32;
        }
        sh.sel[t] = bits;
    } else if (t < 2 * kLoT) {
        const int c = col0 + t - kLoT;
        sh.cntc[t - kLoT] = c < a.nbr ? (float)a.cnt[(size_t)(bh / a.H) * a.nbr + c] : 0.0f;
    }
    mma::cp_async_wait<0>();
    __syncthreads();

    // the weights: lg and va of rows ty + 16 i and columns tx + 16 j
    float lg[4][4], va[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) lg[i][j] = va[i][j] = 0.0f;
#pragma unroll 2
    for (int d = 0; d < D; d += 4) {
        float4 kc[4], vc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            kc[j] = *reinterpret_cast<const float4 *>(&sh.k[tx + 16 * j][d]);
            vc[j] = *reinterpret_cast<const float4 *>(&sh.v[tx + 16 * j][d]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 qr = *reinterpret_cast<const float4 *>(&sh.q[ty + 16 * i][d]);
            const float4 ar = *reinterpret_cast<const float4 *>(&sh.a[ty + 16 * i][d]);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                lg[i][j] = fmaf(qr.x, kc[j].x, fmaf(qr.y, kc[j].y, fmaf(qr.z, kc[j].z, fmaf(qr.w, kc[j].w, lg[i][j]))));
                va[i][j] = fmaf(ar.x, vc[j].x, fmaf(ar.y, vc[j].y, fmaf(ar.z, vc[j].z, fmaf(ar.w, vc[j].w, va[i][j]))));
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 16 * i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = tx + 16 * j;
            float W = 0.0f;
            if (sh.rvalid[r] != 0.0f && sh.cntc[c] > 0.0f && !((sh.sel[r] >> c) & 1ull))
                W = sh.cntc[c] * exp2f(fmaf(lg[i][j] * a.scale, kLog2eB, -sh.rb[r]));
            const float dl = W * (va[i][j] - sh.rbb[r]);
            sh.dl[r][c] = dl;
            sh.dlt[c][r] = dl;
            lg[i][j] = W;   // kept for the transposed store below
        }
    }
    __syncthreads();   // every thread is done reading V-hat
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) sh.wt[tx + 16 * j][ty + 16 * i] = lg[i][j];
    __syncthreads();

    constexpr int DW = D / 16;
    const int d0 = DW * tx;
    const size_t plane = (size_t)BH * a.nbr * D;
    float acc[4][DW];
    // dqhat of the row blocks: dl [b][c] times K-hat [c][d]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < DW; ++e) acc[i][e] = 0.0f;
    lo_accumulate<D>(acc, sh.dl, sh.k, ty, d0);
    lo_flush<D>(a.dxh + head, acc, row0, a.nbr, ty, d0, a.scale);
    // dkhat of the key blocks: dl [c][b] times Q-hat [b][d]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < DW; ++e) acc[i][e] = 0.0f;
    lo_accumulate<D>(acc, sh.dlt, sh.q, ty, d0);
    lo_flush<D>(a.dxh + plane + head, acc, col0, a.nbr, ty, d0, a.scale);
    // dvhat of the key blocks: W [c][b] times A [b][d]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < DW; ++e) acc[i][e] = 0.0f;
    lo_accumulate<D>(acc, sh.wt, sh.a, ty, d0);
    lo_flush<D>(a.dxh + 2 * plane + head, acc, col0, a.nbr, ty, d0, 1.0f);
}

// Writes every token's low-resolution gradient: its block mean's gradient
// divided by the count for a valid token of a non-empty block, zero for the
// rest.  This is the first write of dq, dk and dv in a full-mode backward;
// the per-item kernel adds the selected blocks' terms after it.
template <int D>
__global__ void __launch_bounds__(256)
lowres_bwd_scatter_kernel(const float *__restrict__ dxh, const int *__restrict__ cnt,
                          const float *__restrict__ mask, int H, int N, int nbr, int BH, float *dq, float *dk,
                          float *dv) {
    pdl_wait();
    const size_t n4 = (size_t)BH * N * D / 4;
    const size_t plane = (size_t)BH * nbr * D;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += (size_t)gridDim.x * blockDim.x) {
        const size_t i = 4 * e;
        const size_t tok = i / D;                   // bh * N + t
        const int d = (int)(i % D);
        const int bh = (int)(tok / N), t = (int)(tok % N);
        const int b = t / 32;
        const int cb = cnt[(size_t)(bh / H) * nbr + b];
        float4 xq = make_float4(0.f, 0.f, 0.f, 0.f), xk = xq, xv = xq;
        if (cb > 0 && (!mask || mask[(size_t)(bh / H) * N + t] > 0.0f)) {
            const float inv = 1.0f / (float)cb;
            const size_t src = ((size_t)bh * nbr + b) * D + d;
            const float4 hq = *reinterpret_cast<const float4 *>(dxh + src);
            const float4 hk = *reinterpret_cast<const float4 *>(dxh + plane + src);
            const float4 hv = *reinterpret_cast<const float4 *>(dxh + 2 * plane + src);
            xq = make_float4(hq.x * inv, hq.y * inv, hq.z * inv, hq.w * inv);
            xk = make_float4(hk.x * inv, hk.y * inv, hk.z * inv, hk.w * inv);
            xv = make_float4(hv.x * inv, hv.y * inv, hv.z * inv, hv.w * inv);
        }
        *reinterpret_cast<float4 *>(dq + i) = xq;
        *reinterpret_cast<float4 *>(dk + i) = xk;
        *reinterpret_cast<float4 *>(dv + i) = xv;
    }
}

template <typename T, int D>
cudaError_t launch_typed(const Problem &p, const Workspace &w, const void *q, const void *k, const void *v,
                         const float *mask, const void *dout, float *dq, float *dk, float *dv, cudaStream_t s) {
    BwdArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.dout = dout;
    a.mask = mask;
    a.items = w.items;
    a.head_items = w.head_items;
    a.cols = w.cols;
    a.cap = p.cap;
    a.H = p.H;
    a.N = p.N;
    a.nbr = p.nbr;
    a.scale = 1.0f / sqrtf((float)D);
    a.scale_log2 = a.scale * kLog2eB;
    a.lse2 = w.lse2;
    a.delta = w.delta;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    if constexpr (sizeof(T) == 2)
        return launch_dependent(bwd_item_mma_kernel<D>, dim3((unsigned)(p.BH * p.cap)), dim3(kMmaThreads), 0, s, a);
    else
        return launch_dependent(bwd_item_kernel<T, D>, dim3((unsigned)(p.BH * p.cap)), dim3(kBwdThreads), 0, s, a);
}

template <typename T, int D>
cudaError_t launch_lowres_typed(const Problem &p, const Workspace &w, const float *mask, const void *dout,
                                float *dq, float *dk, float *dv, cudaStream_t s) {
    LoArgs l;
    l.dout = dout;
    l.lse2 = w.lse2;
    l.delta = w.delta;
    l.qhat = w.pooled;
    l.khat = w.pooled + (size_t)p.BH * p.nbr * D;
    l.vhat = w.pooled + (size_t)2 * p.BH * p.nbr * D;
    l.cnt = w.cnt;
    l.bitmap = w.bitmap;
    l.wpr = w.words_per_row;
    l.H = p.H;
    l.N = p.N;
    l.nbr = p.nbr;
    l.scale = 1.0f / sqrtf((float)D);
    l.ab = w.lo_ab;
    l.dxh = w.lo_dxh;
    const int nrb = p.BH * p.nbr;
    cudaError_t e = launch_dependent(lowres_bwd_prep_kernel<T, D>, dim3((unsigned)((nrb + kPrepWarps - 1) / kPrepWarps)),
                                     dim3(32 * kPrepWarps), 0, s, l, nrb);
    if (e != cudaSuccess) return e;
    const size_t lo_smem = sizeof(LoTileSmem<D>);
    e = cudaFuncSetAttribute(lowres_bwd_tile_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lo_smem);
    if (e != cudaSuccess) return e;
    const unsigned nt = (unsigned)((p.nbr + kLoT - 1) / kLoT);
    e = launch_dependent(lowres_bwd_tile_kernel<D>, dim3(nt, nt, (unsigned)p.BH), dim3(kLoThreads), lo_smem, s, l,
                         p.BH);
    if (e != cudaSuccess) return e;
    const size_t n4 = (size_t)p.BH * p.N * D / 4;
    const unsigned grid = (unsigned)std::min<size_t>((n4 + 255) / 256, (size_t)device_sm_count() * 16);
    return launch_dependent(lowres_bwd_scatter_kernel<D>, dim3(grid), dim3(256), 0, s, w.lo_dxh, w.cnt, mask, p.H,
                            p.N, p.nbr, p.BH, dq, dk, dv);
}

}  // namespace

cudaError_t launch_backward_items(const Problem &p, const Workspace &w, const void *q, const void *k,
                                  const void *v, const float *mask, const void *dout, float *dq, float *dk,
                                  float *dv, cudaStream_t s) {
    if (p.dtype == 0)
        return p.D == 64 ? launch_typed<__nv_bfloat16, 64>(p, w, q, k, v, mask, dout, dq, dk, dv, s)
                         : launch_typed<__nv_bfloat16, 32>(p, w, q, k, v, mask, dout, dq, dk, dv, s);
    return p.D == 64 ? launch_typed<float, 64>(p, w, q, k, v, mask, dout, dq, dk, dv, s)
                     : launch_typed<float, 32>(p, w, q, k, v, mask, dout, dq, dk, dv, s);
}

cudaError_t launch_backward_lowres(const Problem &p, const Workspace &w, const float *mask, const void *dout,
                                   float *dq, float *dk, float *dv, cudaStream_t s) {
    if (p.dtype == 0)
        return p.D == 64 ? launch_lowres_typed<__nv_bfloat16, 64>(p, w, mask, dout, dq, dk, dv, s)
                         : launch_lowres_typed<__nv_bfloat16, 32>(p, w, mask, dout, dq, dk, dv, s);
    return p.D == 64 ? launch_lowres_typed<float, 64>(p, w, mask, dout, dq, dk, dv, s)
                     : launch_lowres_typed<float, 32>(p, w, mask, dout, dq, dk, dv, s);
}

}  // namespace mra
