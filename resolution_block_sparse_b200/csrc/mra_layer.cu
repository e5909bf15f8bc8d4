// mra_layer.cu - the MraSelfAttention layer around the MRA-2 forward pass:
// the Q/K/V projection as one tcgen05 GEMM (CTA pairs, cta_group::2) whose
// epilogue adds the bias,
// splits the heads, zero-pads a head size below the kernel's 32 or 64 and
// writes bf16 Q, K, V in [B][H][N][Dp]; and the merge of the attention output
// back into [B][N][H*d].
//
// Page "深入解析 Transformers 中的 MRA 模型" (blog.gitcode.com): the layer
// follows BERT's self-attention (query, key and value linear maps of the
// hidden states, heads of size hidden/H); when the head size is below 32 the
// layer pads Q, K and V with zeros to 32 before the attention and cuts the
// result back (section "源码级原理", the engineering notes after step four).
// Reading: the padding is meant to leave the result unchanged, so the scores
// keep the 1/sqrt(d) of the true head size d: Q is scaled by sqrt(Dp/d) in
// the epilogue, which turns the kernel's 1/sqrt(Dp) into 1/sqrt(d).
#include <cuda_bf16.h>

#include "mra.h"
#include "mra_async.cuh"
#include "mra_internal.cuh"
#include "mra_tcgen05.cuh"

namespace mra {
namespace {

using namespace async;
using namespace tc;

// A pair of CTAs (a cluster of two) computes one 256 x 256 tile with
// tcgen05.mma.cta_group::2: each CTA holds 128 rows of x and 128 rows of W
// (half of the tile's output columns) per 64-deep K step, the even CTA issues
// the MMAs for both, and each CTA's tensor memory holds its own 128 rows of
// the 256 columns.  Per CTA and K step that is 32 KB of operands for a
// 128 x 256 x 64 product, two thirds of what a one-CTA 128 x 256 tile reads,
// and six 32 KB stages keep five K steps of loads in flight.  Two TMEM
// accumulators of 256 columns let the epilogue of one tile overlap the MMAs
// of the next.
constexpr int kGM = 256, kGN = 256, kGK = 64, kGStages = 6;
constexpr int kHalf = 128;                     // rows of x and of W per CTA
constexpr uint32_t kABytes = kHalf * kGK * 2;
constexpr uint32_t kBBytes = kHalf * kGK * 2;
constexpr uint32_t kGStageBytes = kABytes + kBBytes;
constexpr int kGThreads = 192;   // warp 0: TMA, warp 1: MMA (even CTA), warps 2-5: epilogue
constexpr uint32_t kGTmemCols = 2 * kGN;
// epilogue staging for the TMA stores of 64-wide heads: two 32 x 64 bf16
// boxes (4 KB, 128-byte swizzle) per epilogue warp
constexpr uint32_t kStgBytes = 32 * 64 * 2;
constexpr uint32_t kStgOffset = kGStages * kGStageBytes;
constexpr size_t kGemmSmem = (size_t)kStgOffset + 4 * 2 * kStgBytes + 1024;
// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 256 (the pair)
constexpr uint32_t kIdescG =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kGN >> 3) << 17) | ((uint32_t)(kGM >> 4) << 24);

struct ProjArgs {
    int M, NC, ktiles;      // rows B*N, output columns 3*hidden, K steps
    int mtiles, ntiles;
    int B, N, H, d, Dp, hidden;
    float qscale;           // sqrt(Dp / d), applied to Q
    const float *bias;      // [3*hidden] or null
    __nv_bfloat16 *qkv;     // [3][B][H][N][Dp]
    unsigned int *status;
    int tma_out;            // d == Dp == 64: heads leave through TMA stores
};

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// the shared-memory sources of all but the newest group have been read
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// --- the CTA pair (cluster of two)
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared variable in CTA `rank`
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void pair_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier of the pair (here: the even CTA's)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y,
                                                 uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.cta_group::2 [%0], [%1, {%2, %3}], [%4];\n"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrives on one mbarrier (a shared::cluster address: this CTA's or the odd
// CTA's) once the MMAs issued so far have completed
__device__ __forceinline__ void commit_pair_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
                 : "memory");
}
// arrives on the mbarrier at the same offset in both CTAs of the pair (two
// commits, one per CTA)
__device__ __forceinline__ void commit_pair(uint32_t bar) {
    commit_pair_local(bar);
    commit_pair_local(map_rank(bar, 1));
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(bar_cluster) : "memory");
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Writes the 32 accumulator columns c0 .. c0+31 of row m.
__device__ __forceinline__ void store_chunk(const ProjArgs &a, int m, int c0, const uint32_t (&r)[32]) {
    const int b = m / a.N, n = m - b * a.N;
    if (a.d == a.Dp && (a.d & 31) == 0) {
        // the chunk is 32 consecutive elements of one head
        const int which = c0 / a.hidden, within = c0 - which * a.hidden;
        const int h = within / a.d, e0 = within - h * a.d;
        const float *bias = a.bias ? a.bias + c0 : nullptr;
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float x0 = __uint_as_float(r[2 * i]), x1 = __uint_as_float(r[2 * i + 1]);
            if (bias) {
                x0 += __ldg(bias + 2 * i);
                x1 += __ldg(bias + 2 * i + 1);
            }
            w[i] = pack2(x0, x1);
        }
        __nv_bfloat16 *dst = a.qkv + ((((size_t)which * a.B + b) * a.H + h) * a.N + n) * a.Dp + e0;
        uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        return;
    }
    // general head size: element by element; the column that ends a head
    // also writes the head's zero padding
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int c = c0 + i;
        if (c >= a.NC) continue;
        const int which = c / a.hidden, within = c - which * a.hidden;
        const int h = within / a.d, e = within - h * a.d;
        float x = __uint_as_float(r[i]) + (a.bias ? __ldg(a.bias + c) : 0.0f);
        if (which == 0) x *= a.qscale;
        __nv_bfloat16 *row = a.qkv + ((((size_t)which * a.B + b) * a.H + h) * a.N + n) * a.Dp;
        row[e] = __float2bfloat16_rn(x);
        if (e == a.d - 1)
            for (int z = a.d; z < a.Dp; ++z) row[z] = __float2bfloat16_rn(0.0f);
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
qkv_proj_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
                const __grid_constant__ CUtensorMap ty, ProjArgs a) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) unsigned long long bar_full[kGStages], bar_empty[kGStages];
    __shared__ __align__(8) unsigned long long bar_tfull[2], bar_tempty[2], bar_fin;
    __shared__ uint32_t s_tmem;
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = saddr(base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();   // 0: issues the MMAs of the pair
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
    const int ntotal = a.mtiles * a.ntiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kGStages; ++i) {
            mbar_init(saddr(&bar_full[i]), 1);
            mbar_init(saddr(&bar_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(saddr(&bar_tfull[i]), 1);
            mbar_init(saddr(&bar_tempty[i]), 8);   // the epilogue warps of both CTAs
        }
        mbar_init(saddr(&bar_fin), 1);
        mbar_init_fence();
    }
    if (warp == 1) {
        // one warp of each CTA allocates the pair's accumulators together
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(saddr(&s_tmem)),
                     "r"(kGTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    pair_sync();   // both CTAs' barriers are initialised before either signals the other
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            bool ok = true;
            int it = 0;
            for (int t = pair; t < ntotal && ok; t += npairs) {
                const int mt = t % a.mtiles, nt = t / a.mtiles;
                for (int kt = 0; kt < a.ktiles; ++kt, ++it) {
                    const int s = it % kGStages, use = it / kGStages;
                    if (use > 0 && !mbar_wait(saddr(&bar_empty[s]), (use - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = sbase + s * kGStageBytes;
                    const uint32_t full0 = map_rank(saddr(&bar_full[s]), 0);
                    if (rank == 0) mbar_expect_tx(saddr(&bar_full[s]), 2 * kGStageBytes);
                    tma_load_2d_pair(sa, &tx, kt * kGK, mt * kGM + (int)rank * kHalf, full0);
                    tma_load_2d_pair(sa + kABytes, &tw, kt * kGK, nt * kGN + (int)rank * kHalf, full0);
                }
            }
            if (!ok) atomicOr(a.status, kDevTimeout);
            // the even CTA's full barriers count the bytes of both CTAs: once
            // the last phase of each stage is complete no load of the pair is
            // still writing shared memory (the pair waits for each other below)
            if (rank == 0)
                for (int s = 0; s < kGStages && s < it; ++s) {
                    const int last = it - 1 - ((it - 1 - s) % kGStages);
                    mbar_wait(saddr(&bar_full[s]), (last / kGStages) & 1);
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0 && rank == 0) {
            bool ok = true;
            int it = 0, tl = 0;
            for (int t = pair; t < ntotal && ok; t += npairs, ++tl) {
                const int buf = tl & 1, ub = tl >> 1;
                if (ub > 0 && !mbar_wait(saddr(&bar_tempty[buf]), (ub - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + buf * kGN;
                for (int kt = 0; kt < a.ktiles; ++kt, ++it) {
                    const int s = it % kGStages, use = it / kGStages;
                    if (!mbar_wait(saddr(&bar_full[s]), use & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = sbase + s * kGStageBytes;
#pragma unroll
                    for (int ks = 0; ks < kGK / 16; ++ks)
                        mma_pair(acc, sdesc(sa + ks * 32, 16, 1024), sdesc(sa + kABytes + ks * 32, 16, 1024),
                                 kIdescG, (kt | ks) != 0);
                    commit_pair(saddr(&bar_empty[s]));   // the stage is free in both CTAs
                }
                if (ok) commit_pair(saddr(&bar_tfull[buf]));
            }
            if (!ok) atomicOr(a.status, kDevTimeout);
            // every MMA issued here has completed before the pair frees TMEM
            commit_pair_local(saddr(&bar_fin));
            mbar_wait(saddr(&bar_fin), 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3;   // the TMEM lanes this warp may read
        const uint32_t stg = sbase + kStgOffset + (warp - 2) * 2 * kStgBytes;
        const uint32_t tempty_a = map_rank(saddr(&bar_tempty[0]), 0), tempty_b = map_rank(saddr(&bar_tempty[1]), 0);
        int n_stores = 0;
        int tl = 0;
        for (int t = pair; t < ntotal; t += npairs, ++tl) {
            const int mt = t % a.mtiles, nt = t / a.mtiles;
            const int buf = tl & 1, ub = tl >> 1;
            if (!mbar_wait(saddr(&bar_tfull[buf]), ub & 1)) {
                atomicOr(a.status, kDevTimeout);
                break;
            }
            tc_fence_after();
            const int m0 = mt * kGM + (int)rank * kHalf + quarter * 32;
            const uint32_t row_addr = tmem + ((uint32_t)(quarter * 32) << 16) + buf * kGN;
            if (a.tma_out) {
                // each 64-column group is one head: the warp's 32 rows of it
                // go through a swizzled staging box and one TMA store
#pragma unroll 1
                for (int g = 0; g < kGN / 64; ++g) {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(row_addr + g * 64, r0);
                    tmem_ld32(row_addr + g * 64 + 32, r1);
                    tmem_wait_ld();
                    const int c0 = nt * kGN + g * 64;
                    if (m0 >= a.M || c0 >= a.NC) continue;   // warp-uniform
                    const float b0 = a.bias ? __ldg(a.bias + c0 + lane) : 0.0f;
                    const float b1 = a.bias ? __ldg(a.bias + c0 + 32 + lane) : 0.0f;
                    if (n_stores >= 2 && lane == 0) bulk_wait_read1();
                    __syncwarp();
                    const uint32_t box = stg + (n_stores & 1) * kStgBytes;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t w[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int col = 8 * c + 2 * i;   // 0..63
                            const float x0 = __uint_as_float(col < 32 ? r0[col] : r1[col - 32]) +
                                             __shfl_sync(0xffffffffu, col < 32 ? b0 : b1, col & 31);
                            const float x1 = __uint_as_float(col < 32 ? r0[col + 1] : r1[col - 31]) +
                                             __shfl_sync(0xffffffffu, col < 32 ? b0 : b1, (col + 1) & 31);
                            w[i] = pack2(x0, x1);
                        }
                        const uint32_t dst = box + lane * 128 + ((c ^ (lane & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(dst), "r"(w[0]), "r"(w[1]),
                                     "r"(w[2]), "r"(w[3])
                                     : "memory");
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int which = c0 / a.hidden, h = (c0 - which * a.hidden) >> 6;
                        const int b = m0 / a.N, n0 = m0 - b * a.N;
                        tma_store_2d(&ty, box, 0, ((which * a.B + b) * a.H + h) * a.N + n0);
                        bulk_commit();
                    }
                    ++n_stores;
                }
            } else {
                const int m = m0 + lane;
#pragma unroll 1
                for (int j = 0; j < kGN / 32; ++j) {
                    uint32_t r[32];
                    tmem_ld32(row_addr + j * 32, r);
                    tmem_wait_ld();
                    const int c0 = nt * kGN + j * 32;
                    if (m < a.M && c0 < a.NC) store_chunk(a, m, c0, r);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(buf ? tempty_b : tempty_a);   // the even CTA's barrier
        }
        // the TMA stores have finished before the CTA (and its shared memory) goes
        if (lane == 0 && n_stores > 0) bulk_wait_all();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    // neither CTA leaves (or frees the pair's TMEM) while the other may still
    // read its shared memory through the MMAs or signal its barriers
    pair_sync();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kGTmemCols)
                     : "memory");
}

// Attention output [B][H][N][Dp] -> context [B][N][H*d] (the padding cut),
// for head sizes other than 32 and 64 (those are written merged by the
// attention kernel itself).  One thread per 16-byte chunk (d % 8 == 0) or
// per element; the host keeps B*N*hidden below 2^31, so 32-bit indices hold.
__global__ void merge_heads_vec_kernel(const __nv_bfloat16 *__restrict__ o, __nv_bfloat16 *__restrict__ out,
                                       int B, int N, int H, int d, int Dp) {
    pdl_wait();
    const unsigned chunks = (unsigned)d >> 3, per_row = (unsigned)H * chunks;
    const unsigned total = (unsigned)B * N * per_row;
    for (unsigned i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
        const unsigned tok = i / per_row, within = i - tok * per_row;
        const unsigned h = within / chunks, c = within - h * chunks;
        const unsigned b = tok / N, n = tok - b * N;
        const uint4 v = *reinterpret_cast<const uint4 *>(o + (((size_t)b * H + h) * N + n) * Dp + c * 8);
        *reinterpret_cast<uint4 *>(out + (size_t)i * 8) = v;
    }
}

__global__ void merge_heads_kernel(const __nv_bfloat16 *__restrict__ o, __nv_bfloat16 *__restrict__ out, int B,
                                   int N, int H, int d, int Dp) {
    pdl_wait();
    const unsigned per_row = (unsigned)H * d;
    const unsigned total = (unsigned)B * N * per_row;
    for (unsigned i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
        const unsigned tok = i / per_row, within = i - tok * per_row;
        const unsigned h = within / d, e = within - h * d;
        const unsigned b = tok / N, n = tok - b * N;
        out[i] = o[(((size_t)b * H + h) * N + n) * Dp + e];
    }
}

int sm_count() { return device_sm_count(); }

}  // namespace

int head_padded_size(int d) { return d <= 32 ? 32 : 64; }

cudaError_t launch_qkv_projection(const void *x, const void *w, const float *bias, void *qkv, int B, int N,
                                  int hidden, int H, unsigned int *status, cudaStream_t s) {
    const int d = hidden / H, Dp = head_padded_size(d);
    CUtensorMap tx, tw, ty;
    const unsigned long long M = (unsigned long long)B * N, NC = 3ull * hidden;
    if (!make_map_2d(&tx, x, hidden, M, kGK, kHalf) || !make_map_2d(&tw, w, hidden, NC, kGK, kHalf))
        return cudaErrorInvalidValue;
    const int tma_out = (d == 64) ? 1 : 0;
    // [3*B*H*N][64] view of Q, K, V; 32 x 64 boxes
    if (tma_out && !make_map_2d(&ty, qkv, 64, 3ull * B * H * N, 64, 32)) return cudaErrorInvalidValue;
    if (!tma_out) ty = tx;   // unused
    ProjArgs a;
    a.M = (int)M;
    a.NC = (int)NC;
    a.ktiles = (hidden + kGK - 1) / kGK;
    a.mtiles = (int)((M + kGM - 1) / kGM);
    a.ntiles = (int)((NC + kGN - 1) / kGN);
    a.B = B;
    a.N = N;
    a.H = H;
    a.d = d;
    a.Dp = Dp;
    a.hidden = hidden;
    a.qscale = sqrtf((float)Dp / (float)d);
    a.bias = bias;
    a.qkv = static_cast<__nv_bfloat16 *>(qkv);
    a.status = status;
    a.tma_out = tma_out;
    // per call: the attribute belongs to the current device's context
    cudaError_t e = cudaFuncSetAttribute(qkv_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kGemmSmem);
    if (e != cudaSuccess) return e;
    const int tiles = a.mtiles * a.ntiles;
    const int pairs = tiles < sm_count() / 2 ? tiles : sm_count() / 2;
    qkv_proj_kernel<<<2 * pairs, kGThreads, kGemmSmem, s>>>(tx, tw, ty, a);
    return cudaGetLastError();
}

cudaError_t launch_merge_heads(const void *o, void *out, int B, int N, int H, int d, cudaStream_t s) {
    const int Dp = head_padded_size(d);
    const auto *src = static_cast<const __nv_bfloat16 *>(o);
    auto *dst = static_cast<__nv_bfloat16 *>(out);
    const int grid = 4 * sm_count();
    if ((d & 7) == 0) return launch_dependent(merge_heads_vec_kernel, dim3(grid), dim3(256), 0, s, src, dst, B, N, H, d, Dp);
    return launch_dependent(merge_heads_kernel, dim3(grid), dim3(256), 0, s, src, dst, B, N, H, d, Dp);
}

}  // namespace mra
