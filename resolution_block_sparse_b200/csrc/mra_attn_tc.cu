// mra_attn_tc.cu - block-sparse attention on the 5th-generation tensor cores
// (tcgen05 MMA with tensor-memory accumulators, TMA tile loads), bf16, head
// size 64.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理":
//   step three - scores only on the selected 32x32 blocks, a stable softmax
//                (row max), exp(.) times V and the sum of weights;
//   step four  - full mode merges the low-resolution part under a shared
//                maximum; sparse mode normalises the high-resolution part alone.
//
// Tile = four adjacent query block rows of one head: M = 128 query rows, row
// i of the tile on tensor-memory lane i, so each softmax thread owns one query
// row.  The tile runs over the union of the four rows' selected key blocks
// (built by the group plan), four key blocks (128 keys) per step:
//   S = Q_128 . K_step^T           (M = 128, N = 32 * blocks <= 128, K = 64)
//   O += P . V_step                (M = 128, N = 64, K = 32 per block; P read
//                                   from tensor memory, V from the TMA tile)
// Two softmax warps share each tensor-memory lane quarter: warp (w, h) holds
// the 32 rows of block row 4g+w and key blocks 2h, 2h+1 of every step.  It
// turns each of its blocks into P against a lazy reference (the exponent
// reference moves only when the maximum grows by more than 2^8), then both
// warps of the quarter take the larger of their two references (one value
// per row through shared memory), so that they share one O; the one whose
// reference was lower rescales its P in registers.  A (row, key block) pair
// outside that row's selection gets no weight: its warp skips the block and
// writes zero P there, so the exponentials computed are exactly those of the
// selected blocks.  P has a tensor-memory buffer of its own, so S of the next
// step is computed while the softmax of this one runs.
//
// Work item = (group, chunk of at most gchunk union entries).  A group whose
// union is longer is split over several items; each writes (max, sum, O) for
// its 128 rows and the last to finish (arrival counter, no waiting) merges.
// Items are handed out dynamically: the producer warp takes the next index
// from a per-call counter and passes it to the other roles through a ring in
// shared memory.
//
// Warp roles (two CTAs per SM, 256 tensor-memory columns each: S 128, P 64,
// O 64): warps 0-7 softmax and epilogue (each writes 32 of the 64 output
// columns of its rows), warp 8 TMA producer (Q per item, K and V per step, two
// stages), warp 9 MMA issuer.  Every mbarrier wait is bounded: on expiry the
// kernel raises MRA_DEV_TIMEOUT in the status word, every role stops, the
// kernel waits (bounded) for its own loads and MMAs in flight, frees its
// tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>

#include "mra_async.cuh"
#include "mra_attn_common.cuh"
#include "mra_internal.cuh"
#include "mra_tcgen05.cuh"

namespace mra {
namespace {

using namespace async;
using namespace tc;
using attn::kLog2e;

constexpr int kSoftWarps = 8;                    // two per tensor-memory lane quarter
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 32 * (kSoftWarps + 2);
constexpr int kStack = 4;                        // key blocks per step (N = 128 keys)
constexpr int kHalf = kStack / 2;                // key blocks of a step per softmax warp
constexpr int kStages = 2;                       // K and V steps in flight
constexpr int kRing = 4;                         // work items in flight
constexpr int kTile = 32 * 64 * 2;               // one 32-token block, bf16, 4 KB
constexpr int kQBytes = kGroupRows * kTile;      // 128 query rows, 16 KB
constexpr int kStackBytes = kStack * kTile;      // 16 KB
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + 2 * kQBytes;
constexpr int kOffV = kOffK + kStages * kStackBytes;
constexpr int kSmemBytes = kOffV + kStages * kStackBytes;   // 96 KB
constexpr int kSmemAlloc = kSmemBytes + 1024;               // room to align the base to 1 KB
constexpr uint32_t kTmemCols = 256;
// S (128 fp32 columns, block j of a step in columns 32j..32j+31), P (the
// step's 128 keys in bf16, two per column) and O (64 columns)
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192;
constexpr float kRescale = 8.0f;                 // lazy-rescale threshold (log2 units)
constexpr int kRows = 32 * kGroupRows;           // 128
constexpr int kPartialFloats = kRows * (2 + 64); // m[128], l[128], O[128][64]
constexpr int kMaxUnion = 64;                    // largest gchunk (two entries per lane)
constexpr int kMergeBatch = 8;                   // split-group items whose (m, l) load at once
static_assert(kMaxUnion == 2 * 32, "union entries of an item: two per lane");

// instruction descriptors (kind::f16): D fp32, A and B bf16, M = 128
__host__ __device__ constexpr uint32_t idesc_s(int nblocks) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(32 * nblocks) >> 3 << 17) | ((128u >> 4) << 24);
}
// O += P V: B = V read MN-major (d contiguous in the tile), N = 64
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((64u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void named_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }
// Barrier over the two softmax warps of tensor-memory lane quarter wq
// (barrier ids 2-5, named as immediates).
__device__ __forceinline__ void pair_sync(int wq) {
    switch (wq) {
        case 0: asm volatile("bar.sync 2, 64;\n" ::: "memory"); break;
        case 1: asm volatile("bar.sync 3, 64;\n" ::: "memory"); break;
        case 2: asm volatile("bar.sync 4, 64;\n" ::: "memory"); break;
        default: asm volatile("bar.sync 5, 64;\n" ::: "memory"); break;
    }
}
// a bf16 pair times f (rounded to nearest)
__device__ __forceinline__ uint32_t scale_bf16_pair(uint32_t v, float f) {
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v));
    const __nv_bfloat162 y = __floats2bfloat162_rn(x.x * f, x.y * f);
    return *reinterpret_cast<const uint32_t *>(&y);
}
// Barrier over the 256 softmax threads that also ANDs a predicate.
__device__ __forceinline__ bool named_sync_and(bool v) {
    uint32_t out;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.and.pred q, 1, 256, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(out)
        : "r"((uint32_t)v)
        : "memory");
    return out != 0;
}

struct GArgs {
    const GroupItem *gitems;
    const int *head_gitems;
    const int *ucols;
    const float *mask;
    int BH, H, N, nbr, ngroups, gcap, full;
    float scale_log2;
    const float *mlo, *olo, *llo;
    float *partial;
    int *group_arrive;
    int *work_next;   // [1] item counter, [2] most items of any head
    __nv_bfloat16 *out;
    long long ob;     // output element (b, h, n, e) at b * ob + h * oh + n * orow + e
    int oh, orow;
    unsigned int *status;
    int expire_first_wait;   // test hook: the softmax's first wait gives up at once
};

__global__ void __launch_bounds__(kThreads, 2)
attn_group_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const GArgs a) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) unsigned long long bar_qfull[2], bar_qempty[2], bar_kfull[kStages],
        bar_kempty[kStages], bar_vfull[kStages], bar_vempty[kStages], bar_sfull, bar_sfree, bar_pfull, bar_pvdone,
        bar_ofull, bar_oempty, bar_ifull[kRing], bar_iempty[kRing], bar_fin;
    __shared__ float s_sum[2][kRows];       // each row's sums over its two key-block halves
    __shared__ float s_ref[2][2][kRows];    // (step parity, half, row): each half's reference after a step
    __shared__ int s_ring[kRing];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort, s_last;
    __shared__ int s_iss_q, s_iss_k, s_iss_v, s_con_q, s_con_k, s_con_v;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sQ = saddr(base + kOffQ), sK = saddr(base + kOffK), sV = saddr(base + kOffV);

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(saddr(&bar_qfull[i]), 1);
            mbar_init(saddr(&bar_qempty[i]), 1);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(saddr(&bar_kfull[i]), 1);
            mbar_init(saddr(&bar_kempty[i]), 1);
            mbar_init(saddr(&bar_vfull[i]), 1);
            mbar_init(saddr(&bar_vempty[i]), 1);
        }
        for (int i = 0; i < kRing; ++i) {
            mbar_init(saddr(&bar_ifull[i]), 1);
            mbar_init(saddr(&bar_iempty[i]), 1 + kSoftWarps);   // MMA thread + softmax warps
        }
        mbar_init(saddr(&bar_sfull), 1);
        mbar_init(saddr(&bar_sfree), kSoftWarps);
        mbar_init(saddr(&bar_pfull), kSoftWarps);
        mbar_init(saddr(&bar_pvdone), 1);
        mbar_init(saddr(&bar_ofull), 1);
        mbar_init(saddr(&bar_oempty), kSoftWarps);
        mbar_init(saddr(&bar_fin), 1);
        s_iss_q = s_iss_k = s_iss_v = s_con_q = s_con_k = s_con_v = 0;
        s_abort = 0;
        mbar_init_fence();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(saddr(&s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    // the group plan (and everything before it) is complete past this point
    pdl_wait();

    volatile int *abort_flag = &s_abort;
    unsigned int *const status = a.status;
    // bounded wait; false (and the kernel stops) once any role gave up
    auto waitb = [abort_flag, status](unsigned long long *bar, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (mbar_wait(saddr(bar), parity)) return true;
        *abort_flag = 1;
        atomicOr(status, kDevTimeout);
        return false;
    };

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const int total = a.work_next[2] * a.BH;
            int idx = blockIdx.x, n = 0, qn = 0, task = 0;
            bool ok = true;
            while (ok) {
                // next work item: index i = (rank j within its head) * BH + head,
                // so that every head's first items (the long prior rows of group
                // 0) start in the first wave; slots past a head's count are skipped
                int sidx = -1;
                while (idx < total) {
                    const int j = idx / a.BH, bh = idx - j * a.BH;
                    if (j < a.head_gitems[bh]) {
                        sidx = bh * a.gcap + j;
                        break;
                    }
                    idx = (int)gridDim.x + atomicAdd(a.work_next + 1, 1);
                }
                const int slot = n % kRing;
                if (n >= kRing && !waitb(&bar_iempty[slot], ((n / kRing) - 1) & 1)) break;
                s_ring[slot] = sidx;
                mbar_arrive(saddr(&bar_ifull[slot]));
                ++n;
                if (sidx < 0) break;
                // the next index's round trip overlaps this item's loads
                idx = (int)gridDim.x + atomicAdd(a.work_next + 1, 1);
                const GroupItem it = a.gitems[sidx];
                const int nst = (it.ucount + kStack - 1) / kStack;
                if (nst == 0) continue;
                const int bh = it.group / a.ngroups, g = it.group - bh * a.ngroups;
                const int qs = qn & 1;
                if (qn >= 2 && !waitb(&bar_qempty[qs], ((qn >> 1) - 1) & 1)) break;
                mbar_expect_tx(saddr(&bar_qfull[qs]), kQBytes);
                tma_load_2d(sQ + qs * kQBytes, &tq, 0, bh * a.N + g * kRows, saddr(&bar_qfull[qs]));
                s_iss_q = ++qn;
                for (int st = 0; st < nst && ok; ++st, ++task) {
                    const int sg = task % kStages, use = task / kStages;
                    const int nv = min(kStack, it.ucount - st * kStack);
                    int cb[kStack];
#pragma unroll
                    for (int i = 0; i < kStack; ++i)
                        cb[i] = i < nv ? (a.ucols[it.ustart + st * kStack + i] & 0xffff) : 0;
                    if (use >= 1 && !waitb(&bar_kempty[sg], (use - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(saddr(&bar_kfull[sg]), nv * kTile);
                    for (int i = 0; i < nv; ++i)
                        tma_load_2d(sK + sg * kStackBytes + i * kTile, &tk, 0, bh * a.N + cb[i] * 32,
                                    saddr(&bar_kfull[sg]));
                    s_iss_k = task + 1;
                    if (use >= 1 && !waitb(&bar_vempty[sg], (use - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(saddr(&bar_vfull[sg]), nv * kTile);
                    for (int i = 0; i < nv; ++i)
                        tma_load_2d(sV + sg * kStackBytes + i * kTile, &tv, 0, bh * a.N + cb[i] * 32,
                                    saddr(&bar_vfull[sg]));
                    s_iss_v = task + 1;
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // shared-memory descriptors of the first Q, K and V tiles; a tile at
            // byte offset d from one of them is its descriptor + d / 16 (every
            // address stays below 256 KB, inside the descriptor's 14-bit field)
            const uint64_t dQ = sdesc(sQ, 16, 1024), dK = sdesc(sK, 16, 1024), dV = sdesc(sV, 16, 1024);
            int n = 0, qn = 0, t = 0, npv = 0;
            bool ok = true, have = false;
            int p_t = 0, p_sg = 0, p_nv = 0, p_first = 0, p_last = 0;   // the step whose PV is pending
            // O += P V for the pending step, once its softmax wrote P
            auto issue_pv = [&]() -> bool {
                if (!waitb(&bar_vfull[p_sg], (p_t / kStages) & 1)) return false;
                s_con_v = p_t + 1;
                if (!waitb(&bar_pfull, p_t & 1)) return false;
                if (p_first && npv > 0 && !waitb(&bar_oempty, (npv - 1) & 1)) return false;
                tc_fence_after();
                const uint64_t dv = dV + (uint64_t)((p_sg * kStackBytes) >> 4);
#pragma unroll
                for (int j = 0; j < kStack; ++j) {
                    if (j < p_nv) {
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk)
                            mma_f16_ts(tmem + kColO, tmem + kColP + 16 * j + 8 * kk,
                                       dv + (uint64_t)((j * kTile + kk * 2048) >> 4), kIdescPV,
                                       (p_first && j == 0 && kk == 0) ? 0u : 1u);
                    }
                }
                mma_commit(saddr(&bar_vempty[p_sg]));
                mma_commit(saddr(&bar_pvdone));
                if (p_last) {
                    mma_commit(saddr(&bar_ofull));
                    ++npv;
                }
                return true;
            };
            while (ok) {
                const int slot = n % kRing;
                if (!waitb(&bar_ifull[slot], (n / kRing) & 1)) {
                    ok = false;
                    break;
                }
                const int sidx = s_ring[slot];
                mbar_arrive(saddr(&bar_iempty[slot]));
                ++n;
                if (sidx < 0) break;
                const GroupItem it = a.gitems[sidx];
                const int nst = (it.ucount + kStack - 1) / kStack;
                if (nst == 0) continue;
                const int qs = qn & 1;
                for (int st = 0; st < nst; ++st, ++t) {
                    const int sg = t % kStages;
                    const int nv = min(kStack, it.ucount - st * kStack);
                    if (!(ok = waitb(&bar_kfull[sg], (t / kStages) & 1))) break;
                    s_con_k = t + 1;
                    // S is rewritten once the softmax of step t - 1 has read it
                    if (t >= 1 && !(ok = waitb(&bar_sfree, (t - 1) & 1))) break;
                    if (st == 0) {
                        if (!(ok = waitb(&bar_qfull[qs], (qn >> 1) & 1))) break;
                        s_con_q = qn + 1;
                    }
                    tc_fence_after();
                    const uint32_t idesc = idesc_s(nv);
                    const uint64_t dq = dQ + (uint64_t)((qs * kQBytes) >> 4), dk = dK + (uint64_t)((sg * kStackBytes) >> 4);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16(tmem + kColS, dq + 2 * ks, dk + 2 * ks, idesc, ks > 0 ? 1u : 0u);
                    mma_commit(saddr(&bar_sfull));
                    mma_commit(saddr(&bar_kempty[sg]));
                    if (st == nst - 1) mma_commit(saddr(&bar_qempty[qs]));
                    // the PV of the previous step goes after this step's S, so
                    // that the softmax of this step overlaps it
                    if (have && !(ok = issue_pv())) break;
                    p_t = t;
                    p_sg = sg;
                    p_nv = nv;
                    p_first = st == 0;
                    p_last = st == nst - 1;
                    have = true;
                }
                ++qn;
            }
            if (ok && have) ok = issue_pv();
            // every MMA issued by this thread completes before TMEM is freed
            mma_commit(saddr(&bar_fin));
            mbar_wait(saddr(&bar_fin), 0);
        }
        __syncwarp();
    } else if (warp < kSoftWarps) {
        // ------------------------------------------------------------ softmax + epilogue
        const int wq = warp & 3, hh = warp >> 2;            // lane quarter, key-block half
        const uint32_t lq = (uint32_t)(wq * 32) << 16;     // this warp's TMEM lane quarter
        const uint32_t tS = tmem + lq + kColS + 32 * kHalf * hh, tP = tmem + lq + kColP + 16 * kHalf * hh,
                       tO = tmem + lq + kColO;
        const int row = wq * 32 + lane;                     // row of the 128-row tile
        int n = 0, t = 0, on = 0;
        while (true) {
            const int slot = n % kRing;
            const bool got = waitb(&bar_ifull[slot], (n / kRing) & 1);
            const int sidx = got ? s_ring[slot] : -1;
            __syncwarp();
            if (got && lane == 0) mbar_arrive(saddr(&bar_iempty[slot]));
            ++n;
            if (!named_sync_and(sidx >= 0)) break;
            const GroupItem it = a.gitems[sidx];
            const int bh = it.group / a.ngroups, g = it.group - bh * a.ngroups;
            const int b = bh / a.H, h = bh - b * a.H;
            const int r = g * kGroupRows + wq;   // this warp's block row
            const bool row_ok = r < a.nbr;
            const int nst = (it.ucount + kStack - 1) / kStack;
            const int e0 = lane < it.ucount ? a.ucols[it.ustart + lane] : 0;
            const int e1 = lane + 32 < it.ucount ? a.ucols[it.ustart + 32 + lane] : 0;
            const float *mrow = a.mask ? a.mask + (size_t)b * a.N : nullptr;
            float mref = -INFINITY, lsum = 0.0f;
            for (int st = 0; st < nst; ++st, ++t) {
                const int nv = min(kStack, it.ucount - st * kStack);
                int act = 0, part = 0, cb[kHalf];
#pragma unroll
                for (int jj = 0; jj < kHalf; ++jj) {
                    const int u = st * kStack + kHalf * hh + jj;
                    const int e = __shfl_sync(0xffffffffu, u < 32 ? e0 : e1, u & 31);
                    cb[jj] = e & 0xffff;
                    if (kHalf * hh + jj < nv && row_ok && ((e >> (kUnionRowShift + wq)) & 1)) {
                        act |= 1 << jj;
                        if (e & kUnionPartial) part |= 1 << jj;
                    }
                }
                if (a.expire_first_wait && t == 0) {
                    // a wait whose limit has run out (test hook, see the launcher)
                    *abort_flag = 1;
                    atomicOr(status, kDevTimeout);
                }
                waitb(&bar_sfull, t & 1);
                tc_fence_after();
                // this warp's blocks of S one at a time into registers (S is
                // free for the next step's scores once both are read), each
                // turned into P against this half's lazy reference; P of the
                // first block is rescaled in registers when the second moves it
                const float mstart = mref;
                float ls = 0.0f, ls2 = 0.0f;
                uint32_t pk[kHalf][16];
#pragma unroll
                for (int jj = 0; jj < kHalf; ++jj) {
                    if ((act >> jj) & 1) {
                        float x[32];
                        {
                            uint32_t r[32];
                            tmem_ld32(tS + 32 * jj, r);
                            tmem_wait_ld_regs(r);
#pragma unroll
                            for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]);
                        }
                        if (jj == kHalf - 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(saddr(&bar_sfree));
                        }
                        // padded keys of partly padded key blocks take no weight
                        if ((part >> jj) & 1) {
                            const unsigned kv = __ballot_sync(0xffffffffu, mrow[cb[jj] * 32 + lane] > 0.0f);
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (!((kv >> i) & 1u)) x[i] = -INFINITY;
                        }
                        float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
                        for (int i = 4; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], x[i]);
                        const float mxs = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * a.scale_log2;
                        if (mxs > mref + kRescale) {
                            if (jj > 0 && mref != -INFINITY) {
                                const float aj = fast_exp2(mref - mxs);
#pragma unroll
                                for (int i = 0; i < 16; ++i) pk[0][i] = scale_bf16_pair(pk[0][i], aj);
                                ls *= aj;
                                ls2 *= aj;
                            }
                            mref = mxs;
                        }
                        const float ref = (mref == -INFINITY) ? 0.0f : mref;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float p0 = fast_exp2(fmaf(x[2 * i], a.scale_log2, -ref));
                            const float p1 = fast_exp2(fmaf(x[2 * i + 1], a.scale_log2, -ref));
                            const __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
                            pk[jj][i] = *reinterpret_cast<const uint32_t *>(&hp);
                            ls += p0;
                            ls2 += p1;
                        }
                    } else {
                        if (jj == kHalf - 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(saddr(&bar_sfree));
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) pk[jj][i] = 0u;
                    }
                }
                // both halves of the row take the larger reference, so that
                // they share one O; the half whose reference was lower
                // rescales its P in registers
                s_ref[t & 1][hh][row] = mref;
                pair_sync(wq);
                const float mo = s_ref[t & 1][hh ^ 1][row];
                if (mo > mref) {
                    if (mref != -INFINITY) {
                        const float aj = fast_exp2(mref - mo);
#pragma unroll
                        for (int jj = 0; jj < kHalf; ++jj)
#pragma unroll
                            for (int i = 0; i < 16; ++i) pk[jj][i] = scale_bf16_pair(pk[jj][i], aj);
                        ls *= aj;
                        ls2 *= aj;
                    }
                    mref = mo;
                }
                const bool resc = mstart != -INFINITY && mref != mstart;
                const float alpha = resc ? fast_exp2(mstart - mref) : 1.0f;
                lsum = fmaf(lsum, alpha, ls + ls2);
                // P (and O, for a rescale) are free once the PV of step t - 1
                // is done
                if (t >= 1) waitb(&bar_pvdone, (t - 1) & 1);
                tc_fence_after();
#pragma unroll
                for (int jj = 0; jj < kHalf; ++jj)
                    if (kHalf * hh + jj < nv) tmem_st16(tP + 16 * jj, pk[jj]);
                // both warps of the quarter took the same decision; each
                // rescales its 32 columns of O
                if (__any_sync(0xffffffffu, resc)) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * hh, o);
                    tmem_wait_ld_regs(o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tO + 32 * hh, o);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(saddr(&bar_pfull));
            }
            // ---------------------------------------------------- epilogue
            // the row's two key-block halves under one maximum; this warp then
            // produces output columns 32*hh .. 32*hh+31 of its 32 rows
            const int chunk = it.chunk_info & 0xffff, nch = it.chunk_info >> 16;
            s_sum[hh][row] = lsum;
            named_sync();
            // both halves share the reference mref; O holds both
            float l_hi = lsum + s_sum[hh ^ 1][row];
            float m_hi = l_hi > 0.0f ? mref : -INFINITY;
            float o[32];
            if (nst > 0) {
                waitb(&bar_ofull, on & 1);
                ++on;
                tc_fence_after();
                uint32_t raw[32];
                tmem_ld32(tO + 32 * hh, raw);
                tmem_wait_ld_regs(raw);
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(raw[i]);
                // the accumulator is free for the next item's first PV
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(saddr(&bar_oempty));
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0.0f;
            }
            bool write = true;
            if (nch > 1) {
                // split group: this item's (max, sum, O) to its slot; the last
                // item of the group to arrive merges the slots
                float *P = a.partial + (size_t)sidx * kPartialFloats;
                if (hh == 0) {
                    P[row] = m_hi;
                    P[kRows + row] = l_hi;
                }
                uint4 *Po = reinterpret_cast<uint4 *>(P + 2 * kRows + row * 64 + 32 * hh);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    Po[i] = make_uint4(__float_as_uint(o[4 * i]), __float_as_uint(o[4 * i + 1]),
                                       __float_as_uint(o[4 * i + 2]), __float_as_uint(o[4 * i + 3]));
                __threadfence();
                named_sync();
                if (tid == 0) s_last = (atomicAdd(&a.group_arrive[it.group], 1) == nch - 1);
                named_sync();
                write = s_last != 0;
                if (write) {
                    __threadfence();
                    // shared maximum and normaliser over the group's items
                    // (the (m, l) pairs of kMergeBatch items in flight at once)
                    const float *P0 = a.partial + (size_t)(sidx - chunk) * kPartialFloats;
                    float M = -INFINITY, L = 0.0f;
                    for (int c0 = 0; c0 < nch; c0 += kMergeBatch) {
                        float mv[kMergeBatch], lv[kMergeBatch];
#pragma unroll
                        for (int i = 0; i < kMergeBatch; ++i) {
                            const bool in = c0 + i < nch;
                            mv[i] = in ? __ldcg(P0 + (size_t)(c0 + i) * kPartialFloats + row) : -INFINITY;
                            lv[i] = in ? __ldcg(P0 + (size_t)(c0 + i) * kPartialFloats + kRows + row) : 0.0f;
                        }
                        float Mb = M;
#pragma unroll
                        for (int i = 0; i < kMergeBatch; ++i)
                            if (lv[i] > 0.0f) Mb = fmaxf(Mb, mv[i]);
                        if (Mb != -INFINITY) {
                            L = (M == -INFINITY) ? 0.0f : L * fast_exp2(M - Mb);
#pragma unroll
                            for (int i = 0; i < kMergeBatch; ++i)
                                if (lv[i] > 0.0f) L = fmaf(fast_exp2(mv[i] - Mb), lv[i], L);
                            M = Mb;
                        }
                    }
                    m_hi = M;
                    l_hi = L;
                    // merged high-resolution part: this warp's 32 columns of
                    // every item's O
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0.0f;
                    for (int c = 0; c < nch; ++c) {
                        const float *Pc = P0 + (size_t)c * kPartialFloats;
                        const float lc = __ldcg(Pc + kRows + row);
                        const float wc = (lc > 0.0f) ? fast_exp2(__ldcg(Pc + row) - m_hi) : 0.0f;
                        const float4 *Oc = reinterpret_cast<const float4 *>(Pc + 2 * kRows + row * 64 + 32 * hh);
                        float4 x[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) x[i] = __ldcg(Oc + i);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            o[4 * i] = fmaf(wc, x[i].x, o[4 * i]);
                            o[4 * i + 1] = fmaf(wc, x[i].y, o[4 * i + 1]);
                            o[4 * i + 2] = fmaf(wc, x[i].z, o[4 * i + 2]);
                            o[4 * i + 3] = fmaf(wc, x[i].w, o[4 * i + 3]);
                        }
                    }
                    if (tid == 0) a.group_arrive[it.group] = 0;
                }
            }
            if (write && row_ok) {
                // combine with the low-resolution part (full mode) under the
                // shared maximum, normalise; padded queries and rows without a
                // term output 0
                const int rg = bh * a.nbr + r;
                const bool qv = !mrow || mrow[r * 32 + lane] > 0.0f;
                const float m_lo2 = a.full ? a.mlo[rg] * kLog2e : 0.0f;
                const float l_lo = a.full ? a.llo[rg] : 0.0f;
                const bool hi = l_hi > 0.0f, lo = a.full && l_lo > 0.0f;
                float M = hi ? m_hi : -INFINITY;
                if (lo) M = fmaxf(M, m_lo2);
                float fa = 0.0f, fb = 0.0f;
                if (M != -INFINITY && qv) {
                    const float al = hi ? exp2f(m_hi - M) : 0.0f;
                    const float be = lo ? exp2f(m_lo2 - M) : 0.0f;
                    const float den = al * l_hi + be * l_lo;
                    if (den > 0.0f) {
                        fa = al / den;
                        fb = be / den;
                    }
                }
                const float *olo_row = a.olo + (size_t)rg * 64 + 32 * hh;
                __nv_bfloat16 *op = a.out + (size_t)b * a.ob + (size_t)h * a.oh + (size_t)(r * 32 + lane) * a.orow + 32 * hh;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float lo_v = lo ? __ldg(olo_row + i) : 0.0f;
                    o[i] = fmaf(o[i], fa, lo_v * fb);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(op);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __nv_bfloat162 h0 = __floats2bfloat162_rn(o[8 * i], o[8 * i + 1]);
                    const __nv_bfloat162 h1 = __floats2bfloat162_rn(o[8 * i + 2], o[8 * i + 3]);
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[8 * i + 4], o[8 * i + 5]);
                    const __nv_bfloat162 h3 = __floats2bfloat162_rn(o[8 * i + 6], o[8 * i + 7]);
                    uint4 u;
                    u.x = *reinterpret_cast<const uint32_t *>(&h0);
                    u.y = *reinterpret_cast<const uint32_t *>(&h1);
                    u.z = *reinterpret_cast<const uint32_t *>(&h2);
                    u.w = *reinterpret_cast<const uint32_t *>(&h3);
                    dst[i] = u;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        // loads issued but never observed (only after a timeout): wait for
        // them (bounded) so that no copy lands in shared memory after exit
        for (int t = s_con_k; t < s_iss_k; ++t) mbar_wait(saddr(&bar_kfull[t % kStages]), (t / kStages) & 1);
        for (int t = s_con_v; t < s_iss_v; ++t) mbar_wait(saddr(&bar_vfull[t % kStages]), (t / kStages) & 1);
        for (int t = s_con_q; t < s_iss_q; ++t) mbar_wait(saddr(&bar_qfull[t & 1]), (t >> 1) & 1);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

}  // namespace

bool attention_tc_supported(const Problem &p) { return p.dtype == 0 && p.D == 64 && encode_fn() != nullptr; }

cudaError_t launch_attention_tc(const Problem &p, const Workspace &w, const void *q, const void *k,
                                const void *v, const float *mask, void *out, const OutLayout *ol,
                                cudaStream_t s) {
    CUtensorMap tq, tk, tv;
    const unsigned long long rows = (unsigned long long)p.BH * p.N;
    if (!make_map(&tq, q, rows, kRows) || !make_map(&tk, k, rows) || !make_map(&tv, v, rows))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemAlloc);
    if (e != cudaSuccess) return e;
    GArgs a;
    a.gitems = w.gitems;
    a.head_gitems = w.head_gitems;
    a.ucols = w.ucols;
    a.mask = mask;
    a.BH = p.BH;
    a.H = p.H;
    a.N = p.N;
    a.nbr = p.nbr;
    a.ngroups = p.ngroups;
    a.gcap = p.gcap;
    a.full = p.mode == 0 ? 1 : 0;
    a.scale_log2 = kLog2e / sqrtf((float)p.D);
    a.mlo = w.mlo;
    a.olo = w.olo;
    a.llo = w.llo;
    a.partial = w.partial;
    a.group_arrive = w.group_arrive;
    a.work_next = w.work_next;
    a.out = static_cast<__nv_bfloat16 *>(out);
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
    // MRA_TEST_EXPIRE_WAIT=1 (read at every launch) makes the first wait of
    // every CTA's softmax report expiry without waiting, to test the kernel's
    // timeout path: status bit, every role stopping, the copies and MMAs in
    // flight drained, tensor memory freed
    const char *expire = getenv("MRA_TEST_EXPIRE_WAIT");
    a.expire_first_wait = (expire && expire[0] == '1') ? 1 : 0;
    const long long slots = (long long)p.BH * p.gcap;
    const int grid = (int)std::max<long long>(1, std::min<long long>(slots, 2LL * device_sm_count()));
    return launch_dependent(attn_group_kernel, dim3(grid), dim3(kThreads), kSmemAlloc, s, tq, tk, tv, a);
}

}  // namespace mra
