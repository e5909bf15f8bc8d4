// mra_noalloc.cu - a forward-pass entry point that allocates no device memory.
//
// Some callers cannot call cudaMalloc: code that runs while another framework
// owns the device allocator (a caching allocator that must see every byte),
// plugins that are forbidden to allocate, and hosts that enqueue work from
// contexts where an allocation could block or fail mid-stream.  For them this
// file keeps the forward pass's scratch memory in one file-scope __device__
// array of fixed size, so calling the entry point never allocates.
//
// The array is part of the library's device image: every GPU on which the
// library is loaded holds kNoAllocScratchBytes (16 MiB) until the process
// exits.  Host code cannot use the array's name as a device address (on the
// host it only names a shadow symbol), so the device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the first
// call made on it.
#include <cuda_runtime.h>

#include <mutex>

#include "mra.h"
#include "mra_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)MRA_NOALLOC_SCRATCH_BYTES;
constexpr size_t kStatusBytes = 256;   // this entry point's own status word
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
unsigned char *g_scratch_ptr[kMaxDevices] = {};

// Once per device, with that device current: the device address of the array.
int scratch_address(int dev, cudaStream_t stream, unsigned char **out) {
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return MRA_ERR_CUDA;
        }
        // the status word starts at zero; everything else is cleared or
        // written by the kernels of each call before it is read
        if (cudaMemsetAsync(p, 0, kStatusBytes, stream) != cudaSuccess) return MRA_ERR_CUDA;
        g_scratch_ptr[dev] = static_cast<unsigned char *>(p);
    }
    *out = g_scratch_ptr[dev];
    return MRA_OK;
}

}  // namespace

extern "C" int mra_attention_fwd_noalloc(const void *q, const void *k, const void *v,
                                         const float *key_mask, void *out, int B, int H, int N,
                                         int D, int block_per_row, int approx_mode, int first_n,
                                         int diag_n, cudaStream_t stream) {
    using namespace mra;
    int rc = validate(q, k, v, out, B, H, N, D, block_per_row, approx_mode, first_n, diag_n);
    if (rc != MRA_OK) return rc;
    if (key_mask && (((uintptr_t)key_mask) & 3u)) return MRA_ERR_INVALID_ARG;
    const Problem p = make_problem(B, H, N, D, block_per_row, approx_mode, first_n, diag_n,
                                   MRA_DTYPE_BF16);
    const size_t need = carve_workspace(p, nullptr, nullptr);
    if (need > kNoAllocScratchBytes - kStatusBytes) return MRA_ERR_TOO_LARGE;

    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MRA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MRA_ERR_UNSUPPORTED;
    unsigned char *base = nullptr;
    rc = scratch_address(dev, stream, &base);
    if (rc != MRA_OK) return rc;
    Workspace w;
    carve_workspace(p, reinterpret_cast<char *>(base + kStatusBytes), &w);
    w.status = reinterpret_cast<unsigned int *>(base);
    int launches = 0;
    return enqueue_forward(p, w, q, k, v, key_mask, out, nullptr, nullptr, nullptr, stream,
                           /*profile=*/false, &launches);
}

// The status word of the no-allocation calls on the current device: copied to
// the host on `stream` (after the work already queued there), then cleared on
// the same stream.  Neither step allocates.  0 when the entry point has not
// run on this device yet.
extern "C" int mra_get_noalloc_status(cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -MRA_ERR_CUDA;
    unsigned char *base = g_scratch_ptr[dev];
    if (!base) return 0;
    unsigned int word = 0;
    if (cudaMemcpyAsync(&word, base, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return -MRA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -MRA_ERR_CUDA;
    if (cudaMemsetAsync(base, 0, sizeof(word), stream) != cudaSuccess) return -MRA_ERR_CUDA;
    return (int)word;
}

