// mra_attn.cu - exact softmax attention on the selected 32x32 blocks, merged
// with the low-resolution part (full mode).
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理":
//   step three - Q.K^T only on the selected blocks (sampled dense matmul), the
//                row max for a stable softmax, exp(.) times V, and the row sum
//                of the weights as normaliser; no dense N x N matrix is formed;
//   step four  - full mode adds the low-resolution output and normaliser after
//                bringing both parts to a shared maximum; sparse mode divides
//                the high-resolution output by its own normaliser.
//
// Work item = (batch*head, block row r, up to `chunk` selected columns).  The
// row max and sum are kept online (flash style) over the item's columns.  An
// item that covers its whole row writes the final output; the items of a longer
// row write (max, sum, output) partials and the last one to finish (arrival
// counter, no waiting) merges them.  Padded queries (mask 0) output 0.
//
// bf16 kernel: two warps, each owning 16 query rows, mma.sync m16n8k16 with
// fp32 accumulation; Q and K/V blocks in a ring of XOR-swizzled shared-memory
// buffers, loaded by TMA (one 4 KB tile per copy, 128-byte swizzle, completion
// on an mbarrier per buffer) for head size 64 and by cp.async for 32.  fp32
// kernel: FFMA only (no TF32).
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>

#include "mra_async.cuh"
#include "mra_attn_common.cuh"
#include "mra_internal.cuh"
#include "mra_mma.cuh"
#include "mra_tcgen05.cuh"

namespace mra {
namespace {

using namespace attn;
using namespace mma;

struct AttnArgs {
    const void *q, *k, *v;
    const float *mask;
    const WorkItem *items;
    const int *head_items;
    const int *cols;
    int cap, H, N, nbr, full;
    float scale_log2;
    const float *mlo, *olo, *llo;
    unsigned char *partial;   // split-row partial slots
    int *row_arrive;
    int *slot_arrive; // split rows: arrivals per group of items (at the group's first slot)
    int *work_next;   // items handed out beyond the first wave (zeroed per call)
    void *out;
    // output layout: element (b, h, n, e) at b * ob + h * oh + n * orow + e
    long long ob;
    int oh, orow;
    GradStats gs;     // backward-pass statistics (gs.lse2 == nullptr: forward only)
    unsigned int *status;   // device status word (a bounded wait that expired)
};

constexpr int kBf16Threads = 64;
// K/V blocks of an item in flight: a ring of kBf16Stages buffers, the loads
// of block j + kBf16Stages - 1 issued before block j is computed.  Two (ten
// CTAs per SM) measured best: with cp.async loads three stages (seven CTAs)
// took 39.4 against 39.1 us on the N=4096 map and 138 against 119 us on the
// N=16384 map, four stages (six CTAs) 37.4 and 130 us; with the TMA loads
// three stages took 35.3 against 35.9 us and 121.8 against 106.5 us.
constexpr int kBf16Stages = 2;
// CTAs per SM that the ring's shared memory leaves room for (the launch
// bound and the persistent grid)
constexpr int kBf16CtasPerSm = kBf16Stages == 2 ? 10 : (kBf16Stages == 3 ? 7 : 6);

template <int D>
struct Bf16Smem {
    static constexpr int kTile = 32 * D;
    static constexpr size_t kKvBytes = sizeof(__nv_bfloat16) * 2 * kBf16Stages * kTile;
    static constexpr size_t kMergeBytes = partial_slot_bytes<D, __nv_bfloat16>() + sizeof(MergeSmem);
    // Q and the K/V ring first, 1024-byte aligned (the 128-byte swizzle of the
    // TMA copies repeats every 1024 bytes); after the block loop the ring's
    // bytes hold the output staging or, for split rows, the partial and the
    // merge scratch
    alignas(1024) __nv_bfloat16 q[kTile];
    alignas(1024) unsigned char kv_raw[kKvBytes > kMergeBytes ? kKvBytes : kMergeBytes];
    unsigned long long bar[kBf16Stages];   // TMA completion per buffer (Q rides on buffer 0's)
    float km[kBf16Stages][32];   // key mask per buffer
    int cols[kChunk];
    int last;
    int next[2];   // next work index, alternating so a write never races a read
};

// One work item (block row, chunk of selected columns) on a 64-thread CTA.
template <int D>
__device__ __forceinline__ void bf16_item(const AttnArgs &a, int slot, Bf16Smem<D> &sh, const CUtensorMap *map_q,
                                          const CUtensorMap *map_k, const CUtensorMap *map_v, uint32_t &ph) {
    constexpr int kTile = 32 * D;
    __nv_bfloat16 *sQ = sh.q;
    auto sKV = reinterpret_cast<__nv_bfloat16(*)[2][kTile]>(sh.kv_raw);   // [buffer][K or V]
    auto &sKm = sh.km;
    int &s_last = sh.last;
    const int bh = slot / a.cap, local = slot % a.cap;
    if (local >= a.head_items[bh]) return;
    const WorkItem it = a.items[slot];
    const int r = it.row % a.nbr;
    const int chunk = it.chunk_info & 0xffff, nchunks = it.chunk_info >> 16;
    const int b = bh / a.H;
    const size_t head_off = (size_t)bh * a.N * D;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q) + head_off;
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(a.k) + head_off;
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(a.v) + head_off;
    const float *mrow = a.mask ? a.mask + (size_t)b * a.N : nullptr;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tq = lane & 3;

    if constexpr (D != 64) load_tile_async<D, kBf16Threads>(sQ, qg + (size_t)r * kTile, tid);
    const int ncols = it.ncols;
    // the item's column list, read once (the loads below depend on it)
    int *s_cols = sh.cols;
    for (int j = tid; j < ncols; j += kBf16Threads) s_cols[j] = a.cols[it.col_start + j];
    __syncthreads();
    // the first blocks' loads: head size 64 by TMA on the buffers' mbarriers
    // (Q on the first one), head size 32 by cp.async, one commit group per
    // block (the first also holds Q; empty groups keep the count uniform).
    // Rows of this head in the [B*H*N][D] tensor maps:
    const int row0 = bh * a.N;
#pragma unroll
    for (int st = 0; st < kBf16Stages - 1; ++st) {
        if (st < ncols) {
            const int c0 = s_cols[st];
            if constexpr (D == 64) {
                if (tid == 0) {
                    // the previous item's epilogue wrote these bytes through
                    // the generic proxy; the copies go through the async one
                    if (st == 0) asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                    // Q rides on the first buffer's barrier
                    const uint32_t bar = async::saddr(&sh.bar[st]);
                    async::mbar_expect_tx(bar, (st == 0 ? 3 : 2) * kTile * 2);
                    if (st == 0) tc::tma_load_2d(async::saddr(sQ), map_q, 0, row0 + r * 32, bar);
                    tc::tma_load_2d(async::saddr(sKV[st][0]), map_k, 0, row0 + c0 * 32, bar);
                    tc::tma_load_2d(async::saddr(sKV[st][1]), map_v, 0, row0 + c0 * 32, bar);
                }
            } else {
                load_tile_async<D, kBf16Threads>(sKV[st][0], kg + (size_t)c0 * kTile, tid);
                load_tile_async<D, kBf16Threads>(sKV[st][1], vg + (size_t)c0 * kTile, tid);
            }
            if (tid < 32) sKm[st][tid] = mrow ? mrow[c0 * 32 + tid] : 1.0f;
        }
        if constexpr (D != 64) cp_async_commit();
    }

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;
    unsigned qf[D / 16][4];

    for (int j = 0; j < ncols; ++j) {
        const int buf = j % kBf16Stages;
        const int jn = j + kBf16Stages - 1;   // its buffer was consumed in iteration j - 1
        if (jn < ncols) {
            const int c1 = s_cols[jn];
            const int nb = jn % kBf16Stages;
            if constexpr (D == 64) {
                if (tid == 0) {
                    const uint32_t bar = async::saddr(&sh.bar[nb]);
                    async::mbar_expect_tx(bar, 2 * kTile * 2);
                    tc::tma_load_2d(async::saddr(sKV[nb][0]), map_k, 0, row0 + c1 * 32, bar);
                    tc::tma_load_2d(async::saddr(sKV[nb][1]), map_v, 0, row0 + c1 * 32, bar);
                }
            } else {
                load_tile_async<D, kBf16Threads>(sKV[nb][0], kg + (size_t)c1 * kTile, tid);
                load_tile_async<D, kBf16Threads>(sKV[nb][1], vg + (size_t)c1 * kTile, tid);
            }
            if (tid < 32) sKm[nb][tid] = mrow ? mrow[c1 * 32 + tid] : 1.0f;
        }
        if constexpr (D == 64) {
            // block j's copies (and, for j = 0, Q's) have landed; a wait that
            // runs out is reported and waited once more, so that no copy is
            // left in flight
            const uint32_t bar = async::saddr(&sh.bar[buf]);
            if (!async::mbar_wait(bar, (ph >> buf) & 1u)) {
                atomicOr(a.status, kDevTimeout);
                async::mbar_wait(bar, (ph >> buf) & 1u);
            }
            ph ^= 1u << buf;
        } else {
            cp_async_commit();
            cp_async_wait<kBf16Stages - 1>();   // block j's group is complete
        }
        __syncthreads();
        if (j == 0) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int ch = 2 * ks + (lane >> 4);
                ldsm_x4(qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], smem_u32(sQ + swz<D>(row, ch)));
            }
        }
        const __nv_bfloat16 *sK = sKV[buf][0];
        const __nv_bfloat16 *sV = sKV[buf][1];

        // S = Q K^T for this warp's 16 rows x 32 keys
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
                ldsm_x4(b0, b1, b2, b3, smem_u32(sK + swz<D>(key, ch)));
                mma16816(s[nt], qf[ks], b0, b1);
                mma16816(s[nt], qf[ks + 1], b2, b3);
            }
        }
        // online max / sum; scores stay raw (the scale is folded into exp2)
        if (mrow) {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int c = nt * 8 + tq * 2;
                const bool v0 = sKm[buf][c] > 0.0f, v1 = sKm[buf][c + 1] > 0.0f;
                if (!v0) s[nt][0] = s[nt][2] = -INFINITY;
                if (!v1) s[nt][1] = s[nt][3] = -INFINITY;
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
        // running maxima in log2 units
        const float mn_a = fmaxf(m_a, mx_a * a.scale_log2), mn_b = fmaxf(m_b, mx_b * a.scale_log2);
        if (__any_sync(0xffffffffu, mn_a != m_a || mn_b != m_b)) {
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
        // O += P V
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
                ldsm_x4_t(b0, b1, b2, b3, smem_u32(sV + swz<D>(key, ch)));
                mma16816(o[2 * nd2], pf, b0, b1);
                mma16816(o[2 * nd2 + 1], pf, b2, b3);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
    }
    __nv_bfloat16 *out_blk = static_cast<__nv_bfloat16 *>(a.out) + (size_t)b * a.ob + (size_t)(bh - b * a.H) * a.oh +
                             (size_t)r * 32 * a.orow;
    const int ra = warp * 16 + g, rb = ra + 8;
    __syncthreads();   // every warp is done with the K/V buffers
    if (nchunks == 1) {
        // whole row in this item: combine with the low-resolution part and
        // write the final output straight from the accumulators
        const float m_lo2 = a.full ? a.mlo[it.row] * kLog2e : 0.0f;
        const float l_lo = a.full ? a.llo[it.row] : 0.0f;
        const bool lo = a.full && l_lo > 0.0f;
        float fa_a, fb_a, fa_b, fb_b;   // output = O * fa + O_lo * fb, per row
        float lse_a, lse_b;             // base-2 log-sum-exp of the row (backward statistics)
        {
            auto factors = [&](float m, float l, int row, float &fa, float &fb, float &lse) {
                fa = fb = 0.0f;
                lse = INFINITY;
                const bool hi = l > 0.0f;
                float M = hi ? m : -INFINITY;
                if (lo) M = fmaxf(M, m_lo2);
                if (M == -INFINITY || (mrow && !(mrow[r * 32 + row] > 0.0f))) return;
                const float al = hi ? fast_exp2(m - M) : 0.0f;
                const float be = lo ? fast_exp2(m_lo2 - M) : 0.0f;
                const float den = al * l + be * l_lo;
                if (den > 0.0f) {
                    fa = al / den;
                    fb = be / den;
                    lse = M + log2f(den);
                }
            };
            factors(m_a, l_a, ra, fa_a, fb_a, lse_a);
            factors(m_b, l_b, rb, fa_b, fb_b, lse_b);
        }
        float dsum_a = 0.0f, dsum_b = 0.0f;   // dout . out of rows ra, rb (this thread's dims)
        __nv_bfloat16 *ostage = &sKV[0][0][0];   // [32][D] bf16 staging
        const size_t qbase = (size_t)bh * a.N + (size_t)r * 32;
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) {
            const int d = nd * 8 + tq * 2;
            float2 ol = make_float2(0.0f, 0.0f);
            if (lo) ol = *reinterpret_cast<const float2 *>(a.olo + (size_t)it.row * D + d);
            const float x0 = fmaf(o[nd][0], fa_a, ol.x * fb_a), x1 = fmaf(o[nd][1], fa_a, ol.y * fb_a);
            const float y0 = fmaf(o[nd][2], fa_b, ol.x * fb_b), y1 = fmaf(o[nd][3], fa_b, ol.y * fb_b);
            *reinterpret_cast<__nv_bfloat162 *>(ostage + ra * D + d) = __floats2bfloat162_rn(x0, x1);
            *reinterpret_cast<__nv_bfloat162 *>(ostage + rb * D + d) = __floats2bfloat162_rn(y0, y1);
            if (a.gs.lse2) {
                const size_t ia = (qbase + ra) * D + d, ib = (qbase + rb) * D + d;
                dsum_a += x0 * a.gs.dout_at(ia) + x1 * a.gs.dout_at(ia + 1);
                dsum_b += y0 * a.gs.dout_at(ib) + y1 * a.gs.dout_at(ib + 1);
            }
        }
        if (a.gs.lse2) {
#pragma unroll
            for (int off = 1; off < 4; off <<= 1) {
                dsum_a += __shfl_xor_sync(0xffffffffu, dsum_a, off);
                dsum_b += __shfl_xor_sync(0xffffffffu, dsum_b, off);
            }
            if (tq == 0) {
                a.gs.lse2[qbase + ra] = lse_a;
                a.gs.lse2[qbase + rb] = lse_b;
                a.gs.delta[qbase + ra] = dsum_a;
                a.gs.delta[qbase + rb] = dsum_b;
            }
        }
        __syncthreads();
#pragma unroll
        for (int e = tid; e < kTile / 8; e += kBf16Threads) {
            const int row = e / (D / 8), c = e - row * (D / 8);
            *reinterpret_cast<uint4 *>(out_blk + (size_t)row * a.orow + c * 8) =
                reinterpret_cast<const uint4 *>(ostage)[e];
        }
        return;
    }
    // row split across work items: (m, l) in fp32 and O in bf16 (the
    // accumulators relative to the item's own maximum), merged by the last one
    float *stage = reinterpret_cast<float *>(&sKV[0][0][0]);
    if (tq == 0) {
        stage[ra] = m_a;
        stage[rb] = m_b;
        stage[32 + ra] = l_a;
        stage[32 + rb] = l_b;
    }
    __nv_bfloat16 *ostage = reinterpret_cast<__nv_bfloat16 *>(stage + 64);
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        const int d = nd * 8 + tq * 2;
        *reinterpret_cast<__nv_bfloat162 *>(ostage + ra * D + d) = __floats2bfloat162_rn(o[nd][0], o[nd][1]);
        *reinterpret_cast<__nv_bfloat162 *>(ostage + rb * D + d) = __floats2bfloat162_rn(o[nd][2], o[nd][3]);
    }
    __syncthreads();
    MergeSmem &sm = *reinterpret_cast<MergeSmem *>(reinterpret_cast<unsigned char *>(stage) +
                                                   partial_slot_bytes<D, __nv_bfloat16>());
    GradStats gs = a.gs;
    gs.qbase = (size_t)bh * a.N + (size_t)r * 32;
    finish_item<D, kBf16Threads, __nv_bfloat16, __nv_bfloat16, SyncAll>(
        reinterpret_cast<const unsigned char *>(stage), slot, chunk, nchunks, it.row, a.full, a.mlo, a.olo,
        a.llo, a.partial, a.row_arrive, a.slot_arrive, mrow ? mrow + r * 32 : nullptr, out_blk, a.orow, sm, &s_last, gs);
}

// Persistent: the first wave takes items 0..gridDim.x-1, after that a CTA
// takes the next index from a global counter as it finishes an item, so the
// CTAs that drew short rows keep pulling work while the long ones run.  The
// index order is (item index within its head) major, head minor: the long
// rows of every head (the first-n prior rows) come first in their head's
// list and start in the first wave.  The next index is fetched at the start
// of an item, so the atomic's round trip hides behind the item's work.
template <int D>
__global__ void __launch_bounds__(kBf16Threads, kBf16CtasPerSm)
attn_bf16_kernel(const AttnArgs a, int total_slots, int heads, const __grid_constant__ CUtensorMap tq,
                 const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
    pdl_wait();
    __shared__ __align__(1024) Bf16Smem<D> sh;
    if constexpr (D == 64) {
        if (threadIdx.x == 0) {
            for (int b = 0; b < kBf16Stages; ++b) async::mbar_init(async::saddr(&sh.bar[b]), 1);
            async::mbar_init_fence();
        }
        __syncthreads();
    }
    uint32_t ph = 0;   // parity of the next completion of each buffer's barrier
    int i = blockIdx.x;
    for (int t = 0; i < total_slots; ++t) {
        if (threadIdx.x == 0) sh.next[t & 1] = (int)gridDim.x + atomicAdd(a.work_next, 1);
        const int slot = (i % heads) * a.cap + i / heads;
        bf16_item<D>(a, slot, sh, &tq, &tk, &tv, ph);
        __syncthreads();   // shared buffers are free for the next item; next[] is visible
        i = sh.next[t & 1];
    }
}

constexpr int kF32Threads = 128;

// fp32: four threads per query row, each owning D/4 output dimensions.
template <int D>
__global__ void __launch_bounds__(kF32Threads)
attn_f32_kernel(const AttnArgs a) {
    pdl_wait();
    constexpr int kTile = 32 * D;
    constexpr int kDp = D / 4;
    __shared__ __align__(16) float sK[kTile];
    __shared__ __align__(16) float sV[kTile];
    __shared__ float sKm[32];
    __shared__ __align__(16) float stage[32 * (D + 2)];
    __shared__ MergeSmem sm;
    __shared__ int s_last;

    const int slot = blockIdx.x;
    const int bh = slot / a.cap, local = slot % a.cap;
    if (local >= a.head_items[bh]) return;
    const WorkItem it = a.items[slot];
    const int r = it.row % a.nbr;
    const int chunk = it.chunk_info & 0xffff, nchunks = it.chunk_info >> 16;
    const int b = bh / a.H;
    const size_t head_off = (size_t)bh * a.N * D;
    const float *qg = static_cast<const float *>(a.q) + head_off;
    const float *kg = static_cast<const float *>(a.k) + head_off;
    const float *vg = static_cast<const float *>(a.v) + head_off;
    const float *mrow = a.mask ? a.mask + (size_t)b * a.N : nullptr;
    const int tid = threadIdx.x;
    const int qrow = tid >> 2, part = tid & 3;
    const int d0 = part * kDp;

    float qv[kDp], o[kDp];
#pragma unroll
    for (int i = 0; i < kDp; ++i) {
        qv[i] = qg[((size_t)r * 32 + qrow) * D + d0 + i];
        o[i] = 0.0f;
    }
    float m = -INFINITY, l = 0.0f;
    for (int j = 0; j < it.ncols; ++j) {
        const int c = a.cols[it.col_start + j];
        __syncthreads();
        for (int e = tid; e < kTile / 4; e += kF32Threads) {
            reinterpret_cast<float4 *>(sK)[e] = reinterpret_cast<const float4 *>(kg + (size_t)c * kTile)[e];
            reinterpret_cast<float4 *>(sV)[e] = reinterpret_cast<const float4 *>(vg + (size_t)c * kTile)[e];
        }
        if (tid < 32) sKm[tid] = mrow ? mrow[c * 32 + tid] : 1.0f;
        __syncthreads();
        float sc[32];
        float mx = -INFINITY;
#pragma unroll
        for (int kj = 0; kj < 32; ++kj) {
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < kDp; ++i) acc = fmaf(qv[i], sK[kj * D + d0 + i], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            sc[kj] = sKm[kj] > 0.0f ? acc * a.scale_log2 : -INFINITY;
            mx = fmaxf(mx, sc[kj]);
        }
        const float mn = fmaxf(m, mx);
        const float ref = (mn == -INFINITY) ? 0.0f : mn;
        const float al = exp2f(m - ref);
        m = mn;
        l *= al;
#pragma unroll
        for (int i = 0; i < kDp; ++i) o[i] *= al;
#pragma unroll
        for (int kj = 0; kj < 32; ++kj) {
            const float p = exp2f(sc[kj] - ref);
            l += p;
#pragma unroll
            for (int i = 0; i < kDp; ++i) o[i] = fmaf(p, sV[kj * D + d0 + i], o[i]);
        }
    }
    __syncthreads();
    if (part == 0) {
        stage[qrow] = m;
        stage[32 + qrow] = l;
    }
#pragma unroll
    for (int i = 0; i < kDp; ++i) stage[64 + qrow * D + d0 + i] = o[i];
    __syncthreads();
    float *out_blk = static_cast<float *>(a.out) + (size_t)b * a.ob + (size_t)(bh - b * a.H) * a.oh +
                     (size_t)r * 32 * a.orow;
    GradStats gs = a.gs;
    gs.qbase = (size_t)bh * a.N + (size_t)r * 32;
    finish_item<D, kF32Threads, float, float, SyncAll>(
        reinterpret_cast<const unsigned char *>(stage), slot, chunk, nchunks, it.row, a.full, a.mlo, a.olo,
        a.llo, a.partial, a.row_arrive, a.slot_arrive, mrow ? mrow + r * 32 : nullptr, out_blk, a.orow, sm, &s_last, gs);
}

}  // namespace

// bf16 forward passes with head size 64 on dense maps (at least 45 % of the
// block map selected: kTcMinShare20 / 20) run on the tcgen05 kernel; sparser
// maps, fp32, head size 32 and the backward pass's forward re-run (which
// exports per-row statistics) on the warp-level kernels above.  The tcgen05
// kernel works over the union of four block rows' selections, which on
// sparse maps is mostly disjoint, while the warp-level kernel (ten CTAs per
// SM) touches the selected blocks only.  Measured, whole forward step,
// tcgen05 against warp-level: N=2048 (64 x 64 blocks) with 16 blocks per row
// 133 against 99 us, 24 per row 106.5 against 130, 64 per row 128.6 against
// 273.5 (attention alone); N=4096 (128 x 128) with 32 per row 276.5 against
// 216.7, 48 per row 309 against 279, 64 per row 326 against 332, 80 per row
// 339 against 385; the sparse N=4096 and N=16384 maps (4 and 8 per row) and
// the BigBird pattern (19 per row) stay well below the line.
// MRA_ATTN_IMPL=tc or =mma (read once per process) forces either kernel.
constexpr int kTcMinShare20 = 9;

bool attention_uses_tc(const Problem &p, const GradStats *gs) {
    static const char *impl = getenv("MRA_ATTN_IMPL");
    if (gs || !attention_tc_supported(p)) return false;
    if (impl && impl[0] == 'm') return false;
    if (impl && impl[0] == 't') return true;
    return 20LL * p.k >= (long long)kTcMinShare20 * p.nbr * p.nbr;
}

cudaError_t launch_attention(const Problem &p, const Workspace &w, const void *q, const void *k,
                             const void *v, const float *mask, void *out, cudaStream_t s,
                             const GradStats *gs, const OutLayout *ol) {
    AttnArgs a;
    if (ol) {
        a.ob = ol->ob;
        a.oh = ol->oh;
        a.orow = ol->orow;
    } else {
        a.ob = (long long)p.H * p.N * p.D;
        a.oh = p.N * p.D;
        a.orow = p.D;
    }
    a.gs = gs ? *gs : GradStats{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.mask = mask;
    a.items = w.items;
    a.head_items = w.head_items;
    a.cols = w.cols;
    a.cap = p.cap;
    a.H = p.H;
    a.N = p.N;
    a.nbr = p.nbr;
    a.full = p.mode == 0 ? 1 : 0;
    a.scale_log2 = kLog2e / sqrtf((float)p.D);
    a.mlo = w.mlo;
    a.olo = w.olo;
    a.llo = w.llo;
    a.partial = reinterpret_cast<unsigned char *>(w.partial);
    a.row_arrive = w.row_arrive;
    a.slot_arrive = w.slot_arrive;
    a.work_next = w.work_next;
    a.out = out;
    a.status = w.status;
    const long long grid = (long long)p.BH * p.cap;
    if (attention_uses_tc(p, gs)) return launch_attention_tc(p, w, q, k, v, mask, out, ol, s);
    if (p.dtype == 0) {
        const long long pgrid = std::min<long long>(grid, (long long)kBf16CtasPerSm * device_sm_count());
        // [B*H*N][64] tensor maps of Q, K and V, 32-row boxes with the
        // 128-byte swizzle that the shared-memory tiles use (head size 64)
        CUtensorMap tq{}, tk{}, tv{};
        if (p.D == 64) {
            const unsigned long long rows = (unsigned long long)p.BH * p.N;
            if (!tc::make_map(&tq, q, rows) || !tc::make_map(&tk, k, rows) || !tc::make_map(&tv, v, rows))
                return cudaErrorInvalidValue;
            return launch_dependent(attn_bf16_kernel<64>, dim3((unsigned)pgrid), dim3(kBf16Threads), 0, s, a,
                                    (int)grid, p.BH, tq, tk, tv);
        }
        return launch_dependent(attn_bf16_kernel<32>, dim3((unsigned)pgrid), dim3(kBf16Threads), 0, s, a,
                                (int)grid, p.BH, tq, tk, tv);
    }
    if (p.D == 64) return launch_dependent(attn_f32_kernel<64>, dim3((unsigned)grid), dim3(kF32Threads), 0, s, a);
    return launch_dependent(attn_f32_kernel<32>, dim3((unsigned)grid), dim3(kF32Threads), 0, s, a);
}

}  // namespace mra
