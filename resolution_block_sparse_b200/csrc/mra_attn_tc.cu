// mra_attn_tc.cu - block-sparse attention on the 5th-generation tensor cores
// (tcgen05 MMA with TMEM accumulators, TMA tile loads), bf16, head size 64.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理":
//   step three - scores only on the selected 32x32 blocks, a stable softmax
//                (row max), exp(.) times V and the sum of weights;
//   step four  - full mode merges the low-resolution part under a shared
//                maximum.
//
// A query block has 32 rows, below the smallest tcgen05 M (64).  The kernel
// stacks up to four selected KEY blocks of one block row and computes the
// transposed scores  S^T = K_stack . Q^T  (M = 128 keys, N = 32 queries,
// K = 64): TMEM lane t holds key t's scores for the 32 queries.  The output
// is accumulated transposed too:  O^T += V_stack^T . P^T  (M = 64 head dims,
// N = 32 queries, K = 128 keys), A read MN-major straight from the TMA-loaded
// V tile, B = P^T written to shared memory by the softmax threads.  The
// per-query max over the 128 keys is a transposing butterfly over each warp
// plus a 4-way exchange; the running max is rescaled lazily (only when a new
// maximum exceeds the reference by 2^8).
//
// Warp roles (two CTAs per SM): warps 0-3 softmax and epilogue, warp 4 TMA
// producers (lane 0: Q per work item and K stacks; lane 1: V stacks, each
// through its own ring), warp 5 MMA issuer.
// S^T and P^T are double-buffered so that the MMAs of the next stack overlap
// the softmax of the current one.  Every mbarrier wait is bounded: on expiry
// the kernel raises MRA_DEV_TIMEOUT in the status word, drains its own loads
// and MMAs (again bounded), frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "mra_async.cuh"
#include "mra_tcgen05.cuh"
#include "mra_attn_common.cuh"
#include "mra_internal.cuh"

namespace mra {
namespace {

using namespace attn;
using namespace async;
using namespace tc;

constexpr int kConsumers = 128;
constexpr int kThreadsTC = kConsumers + 64;     // + producer warp + MMA warp
constexpr int kStages = 2;                      // K/V stacks in flight
constexpr int kStack = 4;                       // key blocks per stack
constexpr int kTile = 32 * 64 * 2;              // one 32 x 64 bf16 block (4 KB)
constexpr int kStackBytes = kStack * kTile;     // 16 KB
constexpr uint32_t kTmemCols = 128;             // S^T x2 at columns 0, 32; O^T at 64
constexpr float kRescale = 8.0f;                // lazy-rescale threshold (log2 units)

constexpr int kOffQ = 0;                                  // 2 x 4 KB
constexpr int kOffK = 2 * kTile;                          // kStages x 16 KB
constexpr int kOffV = kOffK + kStages * kStackBytes;      // kStages x 16 KB
constexpr int kOffP = kOffV + kStages * kStackBytes;      // 2 x 8 KB (keys 0-63, 64-127)
constexpr int kSmemBytes = kOffP + 4 * kTile;
constexpr int kSmemAlloc = kSmemBytes + 1024;             // room to align the base to 1 KB

// instruction descriptors (kind::f16): D fp32, A and B bf16
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((32u >> 3) << 17) | ((64u >> 4) << 24);

__device__ __forceinline__ void named_sync() { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }
// Named barrier over the 128 consumer threads that also ANDs a predicate.
__device__ __forceinline__ bool named_sync_and(bool v) {
    uint32_t out;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.and.pred q, 1, 128, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(out)
        : "r"((uint32_t)v)
        : "memory");
    return out != 0;
}

// After the call lane q holds op over the warp's 32 lanes of v[q]
// (a transposing butterfly: 31 shuffles for 32 columns).
template <bool kMax>
__device__ __forceinline__ float warp_columns(float (&v)[32], int lane) {
#pragma unroll
    for (int half = 16; half >= 1; half >>= 1) {
        const bool up = (lane & half) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, half);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
    return v[0];
}

struct TcArgs {
    const WorkItem *items;
    const int *head_items;
    const int *cols;
    const float *mask;
    int cap, H, N, nbr, total_slots, full;
    float scale_log2;
    const float *mlo, *olo, *llo;
    unsigned char *partial;   // split-row partial slots
    int *row_arrive;
    __nv_bfloat16 *out;
    unsigned int *status;
};

// The work items of this CTA, in order (the same walk for every role):
// grid stride over (item index within its head) major, head minor, so that
// the long first-n rows of every head start first.
struct ItemWalk {
    int idx;
    int slot;   // slot of the item returned by the last next()
    __device__ __forceinline__ explicit ItemWalk(int first) : idx(first), slot(-1) {}
    __device__ __forceinline__ bool next(const TcArgs &a, WorkItem &it) {
        const int heads = a.total_slots / a.cap;
        for (; idx < a.total_slots; idx += gridDim.x) {
            const int bh = idx % heads, local = idx / heads;
            if (local < a.head_items[bh]) {
                slot = bh * a.cap + local;
                it = a.items[slot];
                idx += gridDim.x;
                return true;
            }
        }
        return false;
    }
};

__global__ void __launch_bounds__(kThreadsTC, 2)
attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const TcArgs a) {
    pdl_wait();
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) unsigned long long bar_qfull[2], bar_qempty[2], bar_kfull[kStages],
        bar_kempty[kStages], bar_vfull[kStages], bar_vempty[kStages], bar_sfull[2], bar_sempty[2],
        bar_pfull[2], bar_pvdone[2], bar_ofull, bar_oempty, bar_fin;
    __shared__ uint32_t s_tmem;
    __shared__ int s_issued_k, s_issued_v, s_issued_q, s_consumed_k, s_consumed_v, s_consumed_q, s_last,
        s_abort;
    __shared__ float red[4][32];
    __shared__ __align__(16) float mw[4][32];
    __shared__ __align__(16) float aw[4][32];
    __shared__ __align__(16) float fac[3][32];
    __shared__ MergeSmem msm;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sQ = saddr(base + kOffQ), sK = saddr(base + kOffK), sV = saddr(base + kOffV),
                   sP = saddr(base + kOffP);
    unsigned char *pbuf = base + kOffP;
    // output staging (fp32, 32 x 64) aliases the P buffers: it is used only
    // after the item's last PV has completed
    float *obuf = reinterpret_cast<float *>(base + kOffP);

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(saddr(&bar_qfull[i]), 1);
            mbar_init(saddr(&bar_qempty[i]), 1);
            mbar_init(saddr(&bar_sfull[i]), 1);
            mbar_init(saddr(&bar_sempty[i]), 4);
            mbar_init(saddr(&bar_pfull[i]), 4);
            mbar_init(saddr(&bar_pvdone[i]), 1);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(saddr(&bar_kfull[i]), 1);
            mbar_init(saddr(&bar_kempty[i]), 1);
            mbar_init(saddr(&bar_vfull[i]), 1);
            mbar_init(saddr(&bar_vempty[i]), 1);
        }
        mbar_init(saddr(&bar_ofull), 1);
        mbar_init(saddr(&bar_oempty), 4);
        mbar_init(saddr(&bar_fin), 1);
        s_issued_k = s_issued_v = s_issued_q = s_consumed_k = s_consumed_v = s_consumed_q = 0;
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         saddr(&s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t tO = tmem + 64;
    bool ok = true;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producers
        // lane 0: Q and K stacks; lane 1: V stacks (K runs ahead of V, since
        // S^T needs K one stack before PV needs V)
        if (lane < 2) {
            const bool is_k = (lane == 0);
            int task = 0, qn = 0;
            ItemWalk walk(blockIdx.x);
            WorkItem it;
            while (ok && walk.next(a, it)) {
                if (it.ncols <= 0) continue;
                const int bh = it.row / a.nbr, r = it.row % a.nbr;
                if (is_k) {
                    const int qs = qn & 1;
                    if (qn >= 2) ok = mbar_wait(saddr(&bar_qempty[qs]), ((qn >> 1) - 1) & 1);
                    if (!ok) break;
                    mbar_expect_tx(saddr(&bar_qfull[qs]), kTile);
                    tma_load_2d(sQ + qs * kTile, &tq, 0, bh * a.N + r * 32, saddr(&bar_qfull[qs]));
                    s_issued_q = ++qn;
                }
                const int nst = (it.ncols + kStack - 1) / kStack;
                for (int st = 0; st < nst && ok; ++st, ++task) {
                    const int sg = task % kStages, use = task / kStages;
                    unsigned long long *full = is_k ? &bar_kfull[sg] : &bar_vfull[sg];
                    unsigned long long *empty = is_k ? &bar_kempty[sg] : &bar_vempty[sg];
                    if (use >= 1) ok = mbar_wait(saddr(empty), (use - 1) & 1);
                    if (!ok) break;
                    // blocks past the end of the chunk are not loaded: their
                    // score rows are never read and their PV k-steps are skipped
                    const int nvalid = min(kStack, it.ncols - st * kStack);
                    mbar_expect_tx(saddr(full), kTile * nvalid);
                    const uint32_t dst = (is_k ? sK : sV) + sg * kStackBytes;
                    for (int bi = 0; bi < nvalid; ++bi) {
                        const int c = a.cols[it.col_start + st * kStack + bi];
                        tma_load_2d(dst + bi * kTile, is_k ? &tk : &tv, 0, bh * a.N + c * 32, saddr(full));
                    }
                    if (is_k) s_issued_k = task + 1;
                    else s_issued_v = task + 1;
                }
            }
            if (!ok) {
                atomicOr(a.status, kDevTimeout);
                atomicExch(&s_abort, 1);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int got_k = 0, got_v = 0, got_q = 0;
            ItemWalk walk(blockIdx.x);
            int qn = 0, t = 0, s_next = 0;   // s_next: next stack to issue S for
            // per-stack bookkeeping for the two stacks in flight
            int nv_cur = 0, first_cur = 0, last_cur = 0, sg_cur = 0;
            // look-ahead state for the next S
            bool have_next = false;
            int nst_n = 0, st_n = 0, qs_n = 0, nv_n = 0;
            WorkItem itn{};
            auto advance = [&]() -> bool {   // position (itn, st_n) on the next stack
                if (have_next && st_n + 1 < nst_n) {
                    ++st_n;
                    nv_n = min(kStack, itn.ncols - st_n * kStack);
                    return true;
                }
                while (walk.next(a, itn)) {
                    if (itn.ncols <= 0) continue;
                    nst_n = (itn.ncols + kStack - 1) / kStack;
                    st_n = 0;
                    qs_n = qn & 1;
                    ++qn;
                    nv_n = min(kStack, itn.ncols);
                    have_next = true;
                    return true;
                }
                have_next = false;
                return false;
            };
            // issue S for the stack the look-ahead points at (task index s_next)
            auto issue_s = [&]() -> bool {
                const int sg = s_next % kStages, use = s_next / kStages;
                const int b = s_next & 1;
                if (!mbar_wait(saddr(&bar_kfull[sg]), use & 1)) return false;
                ++got_k;
                if (s_next >= 2 && !mbar_wait(saddr(&bar_sempty[b]), ((s_next >> 1) - 1) & 1)) return false;
                if (st_n == 0) {
                    if (!mbar_wait(saddr(&bar_qfull[qs_n]), ((qn - 1) >> 1) & 1)) return false;
                    ++got_q;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tmem + 32 * b, sdesc(sK + sg * kStackBytes + ks * 32, 16, 1024),
                            sdesc(sQ + qs_n * kTile + ks * 32, 16, 1024), kIdescS, ks > 0);
                mma_commit(saddr(&bar_sfull[b]));
                mma_commit(saddr(&bar_kempty[sg]));
                if (st_n == nst_n - 1) mma_commit(saddr(&bar_qempty[qs_n]));
                ++s_next;
                return true;
            };
            bool more = advance();
            if (more) ok = issue_s();
            int items_done = 0;
            while (ok && more) {
                // the stack whose S was issued last-but-pending is task t
                nv_cur = nv_n;
                first_cur = (st_n == 0);
                last_cur = (st_n == nst_n - 1);
                sg_cur = t % kStages;
                more = advance();
                if (more) ok = issue_s();
                if (!ok) break;
                const int b = t & 1;
                ok = mbar_wait(saddr(&bar_vfull[sg_cur]), (t / kStages) & 1);
                if (!ok) break;
                ++got_v;
                ok = mbar_wait(saddr(&bar_pfull[b]), (t >> 1) & 1);
                if (!ok) break;
                if (first_cur && items_done >= 1) {
                    ok = mbar_wait(saddr(&bar_oempty), (items_done - 1) & 1);
                    if (!ok) break;
                }
                tc_fence_after();
                const int ksteps = nv_cur * 2;   // 16 keys per MMA, missing blocks skipped
                for (int kk = 0; kk < ksteps; ++kk)
                    mma_f16(tO, sdesc(sV + sg_cur * kStackBytes + kk * 2048, 16, 1024),
                            sdesc(sP + b * 2 * kTile + (kk >> 2) * kTile + (kk & 3) * 32, 16, 1024),
                            kIdescPV, (!first_cur || kk > 0) ? 1u : 0u);
                mma_commit(saddr(&bar_vempty[sg_cur]));
                mma_commit(saddr(&bar_pvdone[b]));
                if (last_cur) {
                    mma_commit(saddr(&bar_ofull));
                    ++items_done;
                }
                ++t;
            }
            if (!ok) {
                atomicOr(a.status, kDevTimeout);
                atomicExch(&s_abort, 1);
            }
            // every MMA issued by this thread completes before TMEM is freed
            mma_commit(saddr(&bar_fin));
            mbar_wait(saddr(&bar_fin), 0);
            s_consumed_k = got_k;
            s_consumed_v = got_v;
            s_consumed_q = got_q;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        int t = 0, on = 0;
        ItemWalk walk(blockIdx.x);
        WorkItem it;
        float mref[32], lp[32];
        while (walk.next(a, it)) {
            const int bh = it.row / a.nbr, r = it.row % a.nbr;
            const int b = bh / a.H;
            const int chunk = it.chunk_info & 0xffff, nchunks = it.chunk_info >> 16;
            const float *mrow = a.mask ? a.mask + (size_t)b * a.N : nullptr;
            const float *qmask = mrow ? mrow + r * 32 : nullptr;
            __nv_bfloat16 *out_blk = a.out + ((size_t)bh * a.N + (size_t)r * 32) * 64;
            const int nst = it.ncols > 0 ? (it.ncols + kStack - 1) / kStack : 0;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                mref[q] = -INFINITY;
                lp[q] = 0.0f;
            }
            for (int st = 0; st < nst; ++st, ++t) {
                const int nvalid = min(kStack, it.ncols - st * kStack);
                const int sb = t & 1;
                // validity of this thread's key (block `warp` of the stack, token `lane`)
                bool kvalid = warp < nvalid;
                if (kvalid && mrow) {
                    const int c = a.cols[it.col_start + st * kStack + warp];
                    kvalid = mrow[c * 32 + lane] > 0.0f;
                }
                ok = mbar_wait(saddr(&bar_sfull[sb]), (t >> 1) & 1) && ok;
                tc_fence_after();
                float s[32];
                if (warp < nvalid) {
                    uint32_t raw[32];
                    tmem_ld32(tmem + 32 * sb + ((uint32_t)(warp * 32) << 16), raw);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) s[q] = __uint_as_float(raw[q]);
                    if (!kvalid) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) s[q] = -INFINITY;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(saddr(&bar_sempty[sb]));
                if (warp < nvalid) {
                    float v[32];
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] = s[q];
                    red[warp][lane] = warp_columns<true>(v, lane);
                } else {
                    red[warp][lane] = -INFINITY;
                }
                if (!named_sync_and(ok && !*reinterpret_cast<volatile int *>(&s_abort))) {
                    ok = false;
                    break;
                }
                // new reference max per query (lane q), identical in every warp
                {
                    const float cmax = fmaxf(fmaxf(red[0][lane], red[1][lane]), fmaxf(red[2][lane], red[3][lane])) *
                                       a.scale_log2;
                    const float cur = (st == 0) ? -INFINITY : mw[warp][lane];
                    float nref = cur, alpha = 1.0f;
                    if (cmax > cur + kRescale || (cur == -INFINITY && cmax != -INFINITY)) {
                        nref = cmax;
                        alpha = (cur == -INFINITY) ? 0.0f : exp2f(cur - cmax);
                    }
                    mw[warp][lane] = nref;
                    aw[warp][lane] = alpha;
                }
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 32; q += 4) {
                    const float4 m4 = *reinterpret_cast<const float4 *>(&mw[warp][q]);
                    mref[q] = m4.x;
                    mref[q + 1] = m4.y;
                    mref[q + 2] = m4.z;
                    mref[q + 3] = m4.w;
                }
                const bool rescale = st > 0 && __any_sync(0xffffffffu, aw[warp][lane] != 1.0f);
                if (rescale) {
                    float al[32];
#pragma unroll
                    for (int q = 0; q < 32; q += 4) {
                        const float4 a4 = *reinterpret_cast<const float4 *>(&aw[warp][q]);
                        al[q] = a4.x;
                        al[q + 1] = a4.y;
                        al[q + 2] = a4.z;
                        al[q + 3] = a4.w;
                    }
#pragma unroll
                    for (int q = 0; q < 32; ++q) lp[q] *= al[q];
                    // O^T may be rescaled only once the previous stack's PV is done
                    ok = mbar_wait(saddr(&bar_pvdone[(t - 1) & 1]), ((t - 1) >> 1) & 1) && ok;
                    tc_fence_after();
                    uint32_t o[32];
                    tmem_ld32(tO + ((uint32_t)(warp * 32) << 16), o);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * al[q]);
                    tmem_st32(tO + ((uint32_t)(warp * 32) << 16), o);
                    tmem_wait_st();
                    tc_fence_before();
                }
                // the P buffer is reused once the PV of two stacks back is done
                if (t >= 2) ok = mbar_wait(saddr(&bar_pvdone[sb]), ((t - 2) >> 1) & 1) && ok;
                if (warp < nvalid) {
                    // P = exp2(s * scale - ref) into the K-major, 128-byte-swizzled P^T tile;
                    // the normaliser sums the same bf16 weights that PV uses, so the
                    // rounding of the weights cancels between numerator and denominator
                    unsigned char *prow = pbuf + sb * 2 * kTile + (tid >> 6) * kTile;
                    const int kk = tid & 63, ch = kk >> 3, within = (kk & 7) * 2;
#pragma unroll
                    for (int q = 0; q < 32; q += 2) {
                        const float r0 = (mref[q] == -INFINITY) ? 0.0f : mref[q];
                        const float r1 = (mref[q + 1] == -INFINITY) ? 0.0f : mref[q + 1];
                        const uint32_t u0 = __float_as_uint(fast_exp2(fmaf(s[q], a.scale_log2, -r0)));
                        const uint32_t u1 = __float_as_uint(fast_exp2(fmaf(s[q + 1], a.scale_log2, -r1)));
                        // bf16 by truncation, two at a time with one byte permute
                        // (integer pipe; the special-function pipe keeps only exp2)
                        const uint32_t pk = __byte_perm(u0, u1, 0x7632);
                        lp[q] += __uint_as_float(u0 & 0xffff0000u);
                        lp[q + 1] += __uint_as_float(u1 & 0xffff0000u);
                        *reinterpret_cast<unsigned short *>(prow + q * 128 + (((ch ^ (q & 7)) << 4) | within)) =
                            (unsigned short)(pk & 0xffffu);
                        *reinterpret_cast<unsigned short *>(prow + (q + 1) * 128 +
                                                            (((ch ^ ((q + 1) & 7)) << 4) | within)) =
                            (unsigned short)(pk >> 16);
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(saddr(&bar_pfull[sb]));
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            {
                float v[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] = lp[q];
                red[warp][lane] = warp_columns<false>(v, lane);
            }
            uint32_t o[32];
            if (nst > 0) {
                ok = mbar_wait(saddr(&bar_ofull), on & 1) && ok;
                ++on;
                tc_fence_after();
                tmem_ld32(tO + ((uint32_t)(warp * 32) << 16), o);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(saddr(&bar_oempty));
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) o[q] = 0u;
            }
            if (!named_sync_and(ok && !*reinterpret_cast<volatile int *>(&s_abort))) {
                ok = false;
                break;
            }
            const float m_hi = (nst > 0) ? mw[0][lane] : -INFINITY;
            const float l_hi = red[0][lane] + red[1][lane] + red[2][lane] + red[3][lane];
            if (nchunks == 1) {
                // final output straight from the accumulator: lane q of warp 0
                // derives query q's factors, threads holding O^T rows write
                if (warp == 0) {
                    const float m_lo2 = a.full ? a.mlo[it.row] * kLog2e : 0.0f;
                    const float l_lo = a.full ? a.llo[it.row] : 0.0f;
                    const bool hi = l_hi > 0.0f, lo = a.full && l_lo > 0.0f;
                    float M = -INFINITY;
                    if (hi) M = m_hi;
                    if (lo) M = fmaxf(M, m_lo2);
                    float al = 0.0f, be = 0.0f, inv = 0.0f;
                    if (M != -INFINITY && (!qmask || qmask[lane] > 0.0f)) {
                        al = hi ? exp2f(m_hi - M) : 0.0f;
                        be = lo ? exp2f(m_lo2 - M) : 0.0f;
                        const float den = al * l_hi + be * l_lo;
                        inv = den > 0.0f ? 1.0f / den : 0.0f;
                    }
                    fac[0][lane] = al * inv;
                    fac[1][lane] = be * inv;
                }
                named_sync();
                if (lane < 16) {
                    const int d = warp * 16 + lane;
                    const float ol = a.full ? a.olo[(size_t)it.row * 64 + d] : 0.0f;
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        obuf[q * 64 + d] = fmaf(__uint_as_float(o[q]), fac[0][q], ol * fac[1][q]);
                }
                named_sync();
                // 32 x 64 outputs = 256 x 8 values: two 16-byte bf16 stores per thread
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int e = tid + u * kConsumers;
                    const float4 x0 = reinterpret_cast<const float4 *>(obuf)[2 * e];
                    const float4 x1 = reinterpret_cast<const float4 *>(obuf)[2 * e + 1];
                    __nv_bfloat162 h[4] = {__floats2bfloat162_rn(x0.x, x0.y), __floats2bfloat162_rn(x0.z, x0.w),
                                           __floats2bfloat162_rn(x1.x, x1.y), __floats2bfloat162_rn(x1.z, x1.w)};
                    reinterpret_cast<uint4 *>(out_blk)[e] = *reinterpret_cast<const uint4 *>(h);
                }
            } else {
                // row split across work items: (max, sum, O) partial, the last
                // item of the row merges (shared epilogue)
                constexpr size_t kSlot = partial_slot_bytes<64, float>();
                const int slot = walk.slot;
                float *dst = reinterpret_cast<float *>(a.partial + (size_t)slot * kSlot);
                if (warp == 0) {
                    dst[lane] = m_hi;
                    dst[32 + lane] = l_hi;
                }
                if (lane < 16) {
                    const int d = warp * 16 + lane;
#pragma unroll
                    for (int q = 0; q < 32; ++q) dst[64 + q * 64 + d] = __uint_as_float(o[q]);
                }
                __threadfence();
                named_sync();
                if (tid == 0) s_last = (atomicAdd(&a.row_arrive[it.row], 1) == nchunks - 1);
                named_sync();
                if (s_last) {
                    __threadfence();
                    const float m_lo2 = a.full ? a.mlo[it.row] * kLog2e : 0.0f;
                    const float l_lo = a.full ? a.llo[it.row] : 0.0f;
                    const float *olo_row = a.full ? a.olo + (size_t)it.row * 64 : nullptr;
                    merge_write<64, kConsumers, true, __nv_bfloat16, float, SyncNamed128>(
                        a.partial + (size_t)(slot - chunk) * kSlot, kSlot, nchunks, a.full, m_lo2, l_lo,
                        olo_row, qmask, out_blk, 64, msm, tid, GradStats{});
                    if (tid == 0) a.row_arrive[it.row] = 0;
                }
            }
            named_sync();
        }
        if (!ok && tid == 0) {
            atomicOr(a.status, kDevTimeout);
            atomicExch(&s_abort, 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        // loads issued but never observed (only after a timeout): wait for
        // them (bounded) so that no copy lands in shared memory after exit
        for (int t = s_consumed_k; t < s_issued_k; ++t)
            mbar_wait(saddr(&bar_kfull[t % kStages]), (t / kStages) & 1);
        for (int t = s_consumed_v; t < s_issued_v; ++t)
            mbar_wait(saddr(&bar_vfull[t % kStages]), (t / kStages) & 1);
        for (int t = s_consumed_q; t < s_issued_q; ++t) mbar_wait(saddr(&bar_qfull[t & 1]), (t >> 1) & 1);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

int g_num_sms = 0;

}  // namespace

bool attention_tc_supported(const Problem &p) { return p.dtype == 0 && p.D == 64 && encode_fn() != nullptr; }

cudaError_t launch_attention_tc(const Problem &p, const Workspace &w, const void *q, const void *k,
                                const void *v, const float *mask, void *out, cudaStream_t s) {
    CUtensorMap tq, tk, tv;
    const unsigned long long rows = (unsigned long long)p.BH * p.N;
    if (!make_map(&tq, q, rows) || !make_map(&tk, k, rows) || !make_map(&tv, v, rows))
        return cudaErrorInvalidValue;
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_num_sms <= 0) g_num_sms = 148;
    }
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemAlloc);
    if (e != cudaSuccess) return e;
    TcArgs a;
    a.items = w.items;
    a.head_items = w.head_items;
    a.cols = w.cols;
    a.mask = mask;
    a.cap = p.cap;
    a.H = p.H;
    a.N = p.N;
    a.nbr = p.nbr;
    a.total_slots = p.BH * p.cap;
    a.full = p.mode == 0 ? 1 : 0;
    a.scale_log2 = kLog2e / sqrtf((float)p.D);
    a.mlo = w.mlo;
    a.olo = w.olo;
    a.llo = w.llo;
    a.partial = reinterpret_cast<unsigned char *>(w.partial);
    a.row_arrive = w.row_arrive;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.status = w.status;
    const int grid = (int)std::min<long long>((long long)a.total_slots, 2LL * g_num_sms);
    return launch_dependent(attn_tc_kernel, dim3(grid), dim3(kThreadsTC), kSmemAlloc, s, tq, tk, tv, a);
}

}  // namespace mra
