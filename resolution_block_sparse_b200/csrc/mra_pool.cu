// mra_pool.cu - masked 32-token block means of Q, K and V.
//
// Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理", step one: the
// sequence is cut into 32-token blocks and each block is replaced by the mean
// of its valid tokens (count-weighted when a mask is given), giving the
// low-resolution Q and K (and, in full mode, the block-pooled V of step four).
//
// Unit = one (tensor, head, block): 32 rows, one contiguous 32*D-element
// span.  One warp reduces one unit: every lane issues all of its 16-byte loads
// of the unit at once (a column slice of several rows), the partial sums are
// folded across the lanes that share a slice, and lanes holding a slice write
// its means.  Four 256-thread CTAs per SM keep 32 units (128 KB of bf16 reads)
// in flight per SM.  HBM-bound: the algorithmic traffic is the bytes of Q,
// K (, V) read plus 4*D bytes written per block and tensor.
#include <cuda_bf16.h>

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
constexpr int pool_min_blocks() { return sizeof(T) == 2 ? 4 : 2; }   // fp32 units need twice the registers

template <typename T, int D>
__global__ void __launch_bounds__(256, pool_min_blocks<T, D>())
pool_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
            const float *__restrict__ mask, int H, int N, int nbr, int BH, int ntensors,
            float *__restrict__ pooled, int *__restrict__ cnt_out, uint4 *__restrict__ zero,
            long long zero_n16) {
    constexpr int kEpc = Vec16<T>::kElems;          // elements per 16-byte slice
    constexpr int kCpr = D / kEpc;                  // slices per row
    constexpr int kRpp = 32 / kCpr;                 // rows per warp pass
    constexpr int kPasses = kBlock / kRpp;
    static_assert(kCpr >= 1 && kCpr <= 32 && 32 % kCpr == 0, "unsupported D");
    // unit index = (tensor * BH + head) * nbr + block, below 2^31 for every
    // accepted size (BH <= 65535, nbr <= 2048); 32-bit index math
    const int plane = BH * nbr;
    const int total = ntensors * plane;
    const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long gs = (long long)gridDim.x * blockDim.x;
    // the per-call counters and histograms of the later phases
    for (long long i = gt; i < zero_n16; i += gs) zero[i] = make_uint4(0u, 0u, 0u, 0u);
    const int lane = threadIdx.x & 31;
    const int slice = lane % kCpr, row0 = lane / kCpr;
    const int nw = (int)(gs >> 5);
    for (int u = (int)(gt >> 5); u < total; u += nw) {
        const int t = u / plane, in_t = u - t * plane;
        const int bh = in_t / nbr, blk = in_t - bh * nbr;
        const T *src = ((t == 0) ? q : (t == 1 ? k : v)) + (size_t)in_t * kBlock * D;
        uint4 raw[kPasses];
#pragma unroll
        for (int p = 0; p < kPasses; ++p)
            raw[p] = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)(p * kRpp + row0) * D) + slice);
        const float mine = mask ? mask[(size_t)(bh / H) * N + (size_t)blk * kBlock + lane] : 1.0f;
        reduce_block<T, D>(raw, mine, pooled + ((size_t)t * plane + in_t) * D, lane);
        // block valid-token counts (one writer per (batch, block))
        if (t == 0 && (bh % H) == 0) {
            float c = mine;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
            if (lane == 0) cnt_out[(size_t)(bh / H) * nbr + blk] = (int)c;
        }
    }
}

template <typename T, int D>
cudaError_t launch_typed(const Problem &p, const Workspace &w, const void *q, const void *k,
                         const void *v, const float *mask, cudaStream_t s) {
    const int sms = device_sm_count();
    const int ntensors = (p.mode == 0) ? 3 : 2;
    const long long units = (long long)ntensors * p.BH * p.nbr;
    long long grid = (units + 7) / 8;   // one unit per warp, eight warps per CTA
    const long long cap = (long long)pool_min_blocks<T, D>() * sms;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    pool_kernel<T, D><<<(unsigned)grid, 256, 0, s>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), mask,
        p.H, p.N, p.nbr, p.BH, ntensors, w.pooled, w.cnt, static_cast<uint4 *>(w.zero_base),
        (long long)((lowres_select_fused_supported(p) ? w.zero_bytes_no_hist : w.zero_bytes) / 16));
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
