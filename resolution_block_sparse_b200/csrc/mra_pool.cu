// mra_pool.cu - masked 32-token block means of Q, K and V.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理", step one: the
// sequence is cut into 32-token blocks and each block is replaced by the mean
// of its valid tokens (count-weighted when a mask is given), giving the
// low-resolution Q and K (and, in full mode, the block-pooled V of step four).
//
// Unit = one (tensor, head, block): 32 rows, one contiguous 32*D-element
// span.  A CTA takes 64 KB worth of consecutive units and has the copy engine
// bring them into shared memory (one bulk copy per unit, completion counted on
// one mbarrier), so the bytes in flight cost no registers and every SM keeps
// about 192 KB of reads outstanding.  Each warp then reduces its units from
// shared memory, every lane holding one 16-byte column slice of several rows;
// partial sums are folded across the lanes that share a slice.  HBM-bound:
// the algorithmic traffic is the bytes of Q, K (, V) read plus 4*D bytes
// written per block and tensor.
#include <cuda_bf16.h>

#include "mra_async.cuh"
#include "mra_internal.cuh"

namespace mra {
namespace {

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int kElems = 8;
    __device__ __forceinline__ static void to_float(const uint4 &r, float *f) {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
};
template <>
struct Vec16<float> {
    static constexpr int kElems = 4;
    __device__ __forceinline__ static void to_float(const uint4 &r, float *f) {
        f[0] = __uint_as_float(r.x);
        f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z);
        f[3] = __uint_as_float(r.w);
    }
};

constexpr int kPoolWarps = 8;
constexpr int kPoolStageBytes = 64 * 1024;   // shared memory per CTA: three CTAs per SM

template <typename T, int D>
constexpr int unit_bytes() { return kBlock * D * (int)sizeof(T); }
template <typename T, int D>
constexpr int units_per_cta() { return kPoolStageBytes / unit_bytes<T, D>(); }

// Masked mean of one 32-row block held in registers (raw: the warp's 16-byte
// slices) and the valid-token count; lanes < kCpr store the D means.
template <typename T, int D>
__device__ __forceinline__ void reduce_block(const uint4 (&raw)[kBlock / (32 / (D / Vec16<T>::kElems))],
                                             float mine, float *dst, int lane) {
    constexpr int kEpc = Vec16<T>::kElems;
    constexpr int kCpr = D / kEpc;
    constexpr int kRpp = 32 / kCpr;
    constexpr int kPasses = kBlock / kRpp;
    const int row0 = lane / kCpr;
    float c = mine;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    float acc[kEpc];
#pragma unroll
    for (int e = 0; e < kEpc; ++e) acc[e] = 0.0f;
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        const float m = __shfl_sync(0xffffffffu, mine, p * kRpp + row0);
        float f[kEpc];
        Vec16<T>::to_float(raw[p], f);
#pragma unroll
        for (int e = 0; e < kEpc; ++e) acc[e] = fmaf(m, f[e], acc[e]);
    }
#pragma unroll
    for (int o = kCpr; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < kEpc; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (lane < kCpr) {
#pragma unroll
        for (int e = 0; e < kEpc; e += 4) {
            float4 o4;
            o4.x = c > 0.0f ? acc[e + 0] / c : 0.0f;
            o4.y = c > 0.0f ? acc[e + 1] / c : 0.0f;
            o4.z = c > 0.0f ? acc[e + 2] / c : 0.0f;
            o4.w = c > 0.0f ? acc[e + 3] / c : 0.0f;
            *reinterpret_cast<float4 *>(dst + lane * kEpc + e) = o4;
        }
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kPoolWarps * 32)
pool_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
            const float *__restrict__ mask, int H, int N, int nbr, int BH, int ntensors,
            float *__restrict__ pooled, int *__restrict__ cnt_out, uint4 *__restrict__ zero,
            long long zero_n16, unsigned int *__restrict__ status) {
    using namespace async;
    constexpr int kEpc = Vec16<T>::kElems;          // elements per 16-byte slice
    constexpr int kCpr = D / kEpc;                  // slices per row
    constexpr int kRpp = 32 / kCpr;                 // rows per warp pass
    constexpr int kPasses = kBlock / kRpp;
    constexpr int kUnits = units_per_cta<T, D>();
    constexpr int kUpw = kUnits / kPoolWarps;       // units per warp
    constexpr uint32_t kUnitBytes = unit_bytes<T, D>();
    static_assert(kCpr >= 1 && kCpr <= 32 && 32 % kCpr == 0, "unsupported D");
    static_assert(kUnits % kPoolWarps == 0 && kUnitBytes % 16 == 0, "unit layout");
    extern __shared__ __align__(128) unsigned char stage[];   // [kUnits][32 rows][D]
    __shared__ __align__(8) unsigned long long bar;

    // unit index = (tensor * BH + head) * nbr + block, below 2^31 for every
    // accepted size (BH <= 65535, nbr <= 2048); 32-bit index math throughout
    const int plane = BH * nbr;   // units per tensor
    const int total = ntensors * plane;
    const int u_first = (int)blockIdx.x * kUnits;
    const int nu = min(kUnits, total - u_first);
    if (threadIdx.x == 0) {
        mbar_init(saddr(&bar), 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // the units of one tensor are consecutive in memory (block-major
        // within a head, heads back to back): one copy per tensor touched
        mbar_expect_tx(saddr(&bar), (uint32_t)nu * kUnitBytes);
        for (int u = 0; u < nu;) {
            const int gw = u_first + u;
            const int t = gw / plane;
            const int in_t = gw - t * plane;
            const int n = min(nu - u, plane - in_t);
            const T *x = (t == 0) ? q : (t == 1 ? k : v);
            bulk_load(saddr(stage + (size_t)u * kUnitBytes), x + (size_t)in_t * kBlock * D,
                      (uint32_t)n * kUnitBytes, saddr(&bar));
            u += n;
        }
    }

    // while the copies fly: clear the per-call counters and histograms of
    // the later phases, and fetch the mask weights of this warp's units
    const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long gs = (long long)gridDim.x * blockDim.x;
    for (long long i = gt; i < zero_n16; i += gs) zero[i] = make_uint4(0u, 0u, 0u, 0u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = lane % kCpr;
    const int row0 = lane / kCpr;
    float mine[kUpw];
    int where[kUpw];   // (tensor, head, block) of the warp's units, packed as the unit index
#pragma unroll
    for (int j = 0; j < kUpw; ++j) {
        const int u = warp * kUpw + j;
        mine[j] = 0.0f;
        where[j] = u_first + u;
        if (u >= nu) continue;
        const int in_t = where[j] % plane;
        const int bh = in_t / nbr, blk = in_t - bh * nbr;
        mine[j] = mask ? mask[(size_t)(bh / H) * N + (size_t)blk * kBlock + lane] : 1.0f;
    }
    if (!mbar_wait(saddr(&bar), 0)) {
        // the copies never completed: report, and wait (bounded) once more so
        // that no copy still targets this CTA's shared memory when it exits
        if (threadIdx.x == 0) atomicOr(status, kDevTimeout);
        mbar_wait(saddr(&bar), 0);
        return;
    }
#pragma unroll
    for (int j = 0; j < kUpw; ++j) {
        const int u = warp * kUpw + j;
        if (u >= nu) continue;
        const int t = where[j] / plane;
        const int in_t = where[j] - t * plane;
        const int bh = in_t / nbr, blk = in_t - bh * nbr;
        const T *tile = reinterpret_cast<const T *>(stage + (size_t)u * kUnitBytes);
        uint4 raw[kPasses];
#pragma unroll
        for (int p = 0; p < kPasses; ++p)
            raw[p] = reinterpret_cast<const uint4 *>(tile + (size_t)(p * kRpp + row0) * D)[slice];
        float *dst = pooled + ((size_t)t * plane + in_t) * D;
        reduce_block<T, D>(raw, mine[j], dst, lane);
        // block valid-token counts (one writer per (batch, block))
        if (t == 0 && (bh % H) == 0) {
            float c = mine[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
            if (lane == 0) cnt_out[(size_t)(bh / H) * nbr + blk] = (int)c;
        }
    }
}

template <typename T, int D>
cudaError_t launch_typed(const Problem &p, const Workspace &w, const void *q, const void *k,
                         const void *v, const float *mask, cudaStream_t s) {
    const int ntensors = (p.mode == 0) ? 3 : 2;
    const long long units = (long long)ntensors * p.BH * p.nbr;
    const long long per_cta = units_per_cta<T, D>();
    const long long grid = (units + per_cta - 1) / per_cta;
    const size_t smem = (size_t)per_cta * unit_bytes<T, D>();
    auto kern = pool_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)grid, kPoolWarps * 32, smem, s>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), mask,
        p.H, p.N, p.nbr, p.BH, ntensors, w.pooled, w.cnt, static_cast<uint4 *>(w.zero_base),
        (long long)((lowres_select_fused_supported(p) ? w.zero_bytes_no_hist : w.zero_bytes) / 16), w.status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const Problem &p, const Workspace &w, const void *q, const void *k,
                        const void *v, const float *mask, cudaStream_t s) {
    if (p.dtype == 0) {
        return p.D == 64 ? launch_typed<__nv_bfloat16, 64>(p, w, q, k, v, mask, s)
                         : launch_typed<__nv_bfloat16, 32>(p, w, q, k, v, mask, s);
    }
    return p.D == 64 ? launch_typed<float, 64>(p, w, q, k, v, mask, s)
                     : launch_typed<float, 32>(p, w, q, k, v, mask, s);
}

}  // namespace mra
