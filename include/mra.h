/*
 * mra.h - C ABI of the B200 (sm_100a) MRA-2 approximate self-attention
 * forward pass.
 *
 * The method is the mra2_attention path described on the page
 * "深入解析 Transformers 中的 MRA 模型：多分辨率近似自注意力机制的架构、配置与实战"
 * (blog.gitcode.com), cited here as [MRA page]:
 *   step one   - 32-token block mean-pooling of Q and K (masked by valid-token
 *                counts) and the low-resolution block-logit map;
 *   step two   - global top-num_block selection over that map, with the
 *                first-n and diagonal priors biased in;
 *   step three - exact softmax attention on the selected 32x32 blocks only;
 *   step four  - in "full" mode, the low-resolution correction for every
 *                unselected block (block-pooled V weighted by low-resolution
 *                attention), brought to a shared maximum and normaliser.
 * The knobs block_per_row, approx_mode, initial_prior_first_n_blocks and
 * initial_prior_diagonal_n_blocks are the four MraConfig parameters of the
 * page's section "MraConfig：四个专属参数与完整默认值".
 *
 * Conventions shared by every entry point
 *   - Tensors q, k, v, out are contiguous row-major [B][H][N][D] in DEVICE
 *     memory, 16-byte aligned.  bf16 entry points read and write bfloat16,
 *     the _f32 entry points float32.
 *   - key_mask is a DEVICE float array [B][N] of 0/1 shared by all heads of a
 *     batch entry (1 = valid token), or NULL for "every token valid".  It
 *     masks keys, values and queries alike; outputs of padded queries are 0.
 *   - N must be a positive multiple of 32 ([MRA page], paragraph on
 *     engineering details: the sequence length must divide by the 32-token
 *     block), N <= 65536; D must be 32 or 64 (callers with a smaller head
 *     size zero-pad to 32, as the page's self-attention module does).
 *   - num_block = min((N/32) * block_per_row, (N/32)^2) blocks are selected
 *     per (batch, head) ([MRA page], num_block formula).
 *   - approx_mode: MRA_FULL (0) or MRA_SPARSE (1).  0 <= first_n, diag_n <= N/32.
 *   - Work is enqueued on `stream` and returns without synchronising.  The
 *     caller owns every pointer; the library owns a per-device workspace that
 *     it allocates on first use (and grows when a larger problem arrives),
 *     so the first call of a given size should precede any stream capture.
 *     Calls that share the workspace are serialised by the library's host
 *     lock, but kernels of two calls on different streams may overlap on
 *     the GPU and then race on the workspace: issue them on one stream.
 *   - Errors are returned synchronously, before any launch, as mra_status
 *     values; nothing aborts or prints.
 *   - Two environment switches choose between equivalent kernels (results
 *     agree within the stated tolerances; the defaults are the faster ones):
 *     MRA_FUSED=1 runs maps of at most 16x16 blocks as one launch per call
 *     wherever the head fits in shared memory, MRA_FUSED=0 never (by default
 *     only bf16 problems with at least 64 heads take it).  bf16 forward
 *     passes with D = 64 run the exact attention on the tcgen05 tensor cores
 *     (groups of four block rows over the union of their selected blocks);
 *     MRA_ATTN_IMPL=mma (read once per process) keeps them on the warp-level
 *     kernel that fp32, D = 32 and the backward pass use.
 */
#ifndef MRA_B200_H
#define MRA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef __CUDA_RUNTIME_H__
struct CUstream_st;
typedef struct CUstream_st *cudaStream_t;
#endif

#if defined(__GNUC__)
#define MRA_API __attribute__((visibility("default")))
#else
#define MRA_API
#endif

typedef enum {
    MRA_OK = 0,
    MRA_ERR_INVALID_ARG = 1,     /* a size, mode, prior or pointer is invalid      */
    MRA_ERR_UNSUPPORTED = 2,     /* D not in {32, 64}, or N above the maximum       */
    MRA_ERR_CUDA = 3,            /* a CUDA call or launch failed                    */
    MRA_ERR_ALLOC = 4,           /* workspace allocation failed                     */
    MRA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device wait gave up (the MRA_DEV_TIMEOUT
                                    bit of a status word, see mra_status_from_device) */
    MRA_ERR_TOO_LARGE = 6        /* the problem needs more scratch than the static
                                    array of mra_attention_fwd_noalloc holds         */
} mra_status;

enum { MRA_FULL = 0, MRA_SPARSE = 1 };
enum { MRA_DTYPE_BF16 = 0, MRA_DTYPE_F32 = 1 };

/* Bits of the device status word read by mra_get_device_status. */
enum {
    MRA_DEV_KEY_RANGE = 1,   /* some |l - rowmax| >= 2500: the tier order may
                                differ from exact additive biases              */
    MRA_DEV_COUNT = 2,       /* selected-block count per head differed from k  */
    MRA_DEV_TIMEOUT = 4      /* a bounded wait inside a kernel gave up; that
                                kernel's output is incomplete                  */
};

/* Forward pass, bf16 in/out, fp32 accumulation.  Steps one to four of the
 * [MRA page]; see the conventions above for layout and errors. */
MRA_API int mra_attention_fwd(const void *q, const void *k, const void *v, const float *key_mask,
                      void *out, int B, int H, int N, int D, int block_per_row,
                      int approx_mode, int first_n, int diag_n, cudaStream_t stream);

/* Forward pass, fp32 in/out (no TF32 anywhere on this path). */
MRA_API int mra_attention_fwd_f32(const float *q, const float *k, const float *v,
                          const float *key_mask, float *out, int B, int H, int N, int D,
                          int block_per_row, int approx_mode, int first_n, int diag_n,
                          cudaStream_t stream);

/* Forward pass that also exports intermediates (each pointer may be NULL):
 *   sel_idx      int32 [B*H][num_block]  selected flat block indices r*(N/32)+c,
 *                                        ascending (row-major order)
 *   lowres_logit float [B*H][N/32][N/32] low-resolution logits qhat.khat/sqrt(D)
 *   pooled       float [3][B*H][N/32][D] qhat, khat, vhat (vhat only in full mode;
 *                                        zero in sparse mode)
 * dtype is MRA_DTYPE_BF16 or MRA_DTYPE_F32; all pointers are device pointers. */
MRA_API int mra_attention_fwd_ex(const void *q, const void *k, const void *v, const float *key_mask,
                         void *out, int B, int H, int N, int D, int block_per_row,
                         int approx_mode, int first_n, int diag_n, int dtype, int32_t *sel_idx,
                         float *lowres_logit, float *pooled, cudaStream_t stream);

/* End-to-end convenience call on HOST buffers: copies q, k, v (and the mask)
 * from host memory to a library-owned device staging area, runs the forward
 * pass and copies `out` back, then synchronises.  The work is cut into about
 * eight chunks of heads (within one batch entry each): inputs go in on a
 * library copy stream, each chunk's forward pass runs on `stream` once its
 * inputs have landed, and its output goes back on a second library copy
 * stream, so transfers in both directions overlap the computation.  The
 * copies start after the work already queued on `stream`.  Pinned host
 * memory gives asynchronous copies; pageable memory works but is slower.
 * Same arguments as mra_attention_fwd_ex without intermediates. */
MRA_API int mra_attention_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                           const float *key_mask_host, void *out_host, int B, int H, int N,
                           int D, int block_per_row, int approx_mode, int first_n, int diag_n,
                           int dtype, cudaStream_t stream);

/* Backward pass: gradients of the forward output (same arguments, same
 * selection) with respect to q, k and v, for the incoming gradient dout.
 *
 * Page "深入解析 Transformers 中的 MRA 模型", section "源码级原理", steps three
 * and four: the block-sparse products are differentiated through transposed
 * block indices; the selected set (the top-k) is held fixed; in "sparse" mode
 * the low-resolution branch only chooses blocks and takes no gradient; in
 * "full" mode its output is part of the result, so the gradient also flows
 * through the masked block means of q, k and v.  Padded queries (output 0)
 * pass no gradient.
 *
 * q, k, v, dout: device, [B][H][N][D] row-major, 16-byte aligned; bf16 for
 * mra_attention_bwd, fp32 for mra_attention_bwd_f32.  key_mask as in the
 * forward pass.  dq, dk, dv: device fp32 [B][H][N][D], 16-byte aligned,
 * written (not accumulated); dq is also the scratch of the internal forward
 * pass.  The call re-runs the forward pass (the selection is deterministic,
 * so it is the one the forward call made) and needs no saved state.
 * Asynchronous on `stream`; errors as for mra_attention_fwd. */
MRA_API int mra_attention_bwd(const void *q, const void *k, const void *v, const float *key_mask,
                              const void *dout, float *dq, float *dk, float *dv, int B, int H, int N,
                              int D, int block_per_row, int approx_mode, int first_n, int diag_n,
                              cudaStream_t stream);
MRA_API int mra_attention_bwd_f32(const float *q, const float *k, const float *v,
                                  const float *key_mask, const float *dout, float *dq, float *dk,
                                  float *dv, int B, int H, int N, int D, int block_per_row,
                                  int approx_mode, int first_n, int diag_n, cudaStream_t stream);

/* Size of the static device array behind mra_attention_fwd_noalloc. */
#define MRA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* Forward pass, bf16, for callers that cannot allocate device memory.
 *
 * The method's pages have no counterpart of this entry point; it exists for
 * callers that are not allowed to call cudaMalloc or any allocating routine:
 * code running under another framework's caching allocator, plugins that
 * must not allocate, and hosts that enqueue work where an allocation could
 * block or fail.  The caller passes q, k, v, key_mask and out exactly as for
 * mra_attention_fwd (device memory, same layout); all scratch memory comes
 * from one static __device__ array of MRA_NOALLOC_SCRATCH_BYTES (16 MiB) that
 * every GPU loading the library holds until the process exits.  Nothing here
 * calls cudaMalloc, cudaFree or an allocating library routine.
 *
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, that device current) and clears its status
 *     word; make that first call before any stream capture.
 *   - Problems whose scratch does not fit return MRA_ERR_TOO_LARGE before any
 *     launch (for example B*H = 4, N = 1024, block_per_row = 4 fits; the
 *     N = 4096 benchmark workload does not).
 *   - Every call reuses the same array and leaves its contents behind; each
 *     call clears what must start at zero.  Calls whose kernels overlap on the
 *     GPU (different streams, or several host threads with different streams)
 *     race on the array and give wrong results: issue them on one stream.
 *   - Device status flags of these calls (MRA_DEV_*) are kept in a word of
 *     the static array and reported by mra_get_noalloc_status, not by
 *     mra_get_device_status.
 * Returns mra_status values like mra_attention_fwd. */
MRA_API int mra_attention_fwd_noalloc(const void *q, const void *k, const void *v,
                                      const float *key_mask, void *out, int B, int H, int N,
                                      int D, int block_per_row, int approx_mode, int first_n,
                                      int diag_n, cudaStream_t stream);

/* Status word of the mra_attention_fwd_noalloc calls on the current device:
 * copied to the host on `stream` after the work queued there (the call waits
 * for it), then cleared on `stream`; allocates nothing.  Returns the bitwise
 * OR of the MRA_DEV_* flags raised since the previous read (0 before the
 * first no-allocation call on the device), or -MRA_ERR_CUDA. */
MRA_API int mra_get_noalloc_status(cudaStream_t stream);

/* Block-sparse attention on a given set of 32x32 blocks per (batch, head):
 * the attention of step three with the softmax over the union of the given
 * blocks only (the sparse mode of step four), for any block pattern - the
 * BigBird pattern of mra_bigbird_block_list among them.  ([MRA page] steps
 * three and four; page "Transformers 中的 BigBird：面向超长序列的稀疏注意力
 * 模型完全指南", section on the attention mechanism, for the pattern.)
 *   q, k, v, out, key_mask: as in the forward pass; dtype MRA_DTYPE_BF16 or
 *     MRA_DTYPE_F32 selects the element type of q, k, v and out.
 *   block_idx: DEVICE int32 [B*H][cap_sel], 4-byte aligned; row bh lists the
 *     head's blocks as flat indices r * (N/32) + c (query block row r, key
 *     block c) in strictly ascending order, followed by -1 padding.  Heads
 *     may hold different counts; 1 <= cap_sel <= (N/32)^2.
 *   Query rows whose block row holds no block, and padded queries, get 0.
 *   A head whose list is not ascending, holds an index outside
 *   [0, (N/32)^2) or has an entry >= 0 after a -1 gets no output (out is not
 *   written for it) and sets MRA_DEV_COUNT in the device status word; the
 *   other heads are unaffected.
 * Two kernels; asynchronous on `stream`.  Returns an mra_status value. */
MRA_API int mra_blocksparse_attention_fwd(const void *q, const void *k, const void *v,
                                          const float *key_mask, void *out, int B, int H, int N,
                                          int D, const int32_t *block_idx, int cap_sel, int dtype,
                                          cudaStream_t stream);

/* The BigBird block pattern of one head as ascending flat 32-token block
 * indices, host code (page "Transformers 中的 BigBird：面向超长序列的稀疏注意力
 * 模型完全指南", sections on the attention mechanism and the usage notes):
 * with nb = N / block_size blocks, block i attends to the window
 * {i-1, i, i+1} (clipped at the ends), to the first and the last block (the
 * two global blocks, which also attend to every block) and to its
 * num_random random blocks rand_blocks[i][0..num_random) (HOST int32
 * [nb][num_random], each in [0, nb), drawn by the caller); a block chosen
 * twice counts once; when nb <= 5 + 2 * num_random every block attends to
 * every block.  block_size is a multiple of 32 that divides N; each
 * block_size block maps to the (block_size/32)^2 32-token blocks it covers.
 * out: HOST int32 [capacity]; *count gets the number written.  Returns
 * MRA_ERR_INVALID_ARG for bad sizes or random blocks, MRA_ERR_TOO_LARGE when
 * capacity is short, MRA_ERR_UNSUPPORTED for N > 65536. */
MRA_API int mra_bigbird_block_list(int N, int block_size, int num_random, const int32_t *rand_blocks,
                                   int32_t *out, int capacity, int *count);

/* The MraSelfAttention layer ([MRA page]: a BERT-style self-attention whose
 * attention is mra2_attention; heads of size d = hidden / H, zero-padded to
 * 32 when d < 32, section "源码级原理", notes after step four):
 *   q, k, v = x W_q^T + b_q, x W_k^T + b_k, x W_v^T + b_v, split into H heads
 *   (feature h*d + e of a projection is element e of head h), the MRA-2
 *   forward pass per head with scores scaled by 1/sqrt(d), and the heads
 *   merged back: out[b][n][h*d + e].
 *   x:     DEVICE bf16 [B][N][hidden], 16-byte aligned (the hidden states).
 *   w_qkv: DEVICE bf16 [3*hidden][hidden], 16-byte aligned: the query, key
 *          and value weights stacked in that order, each [hidden out][hidden
 *          in] (a linear layer's weight layout).
 *   b_qkv: DEVICE fp32 [3*hidden] or NULL (no bias).
 *   key_mask, block_per_row, approx_mode, first_n, diag_n: as in the forward
 *          pass; out: DEVICE bf16 [B][N][hidden], 16-byte aligned.
 *   hidden must be a multiple of H and of 8, d = hidden / H <= 64; heads
 *   with d < 32 are padded to 32 and 32 < d < 64 to 64 (Q is scaled by
 *   sqrt(padded / d) so that the scores keep 1/sqrt(d)).  The projected
 *   Q, K, V live in bf16, as the kernels' inputs do.
 * The projection runs on the tcgen05 tensor cores; the library's workspace
 * holds the projected heads.  Asynchronous on `stream`; returns an
 * mra_status value. */
MRA_API int mra_self_attention_fwd(const void *x, const void *w_qkv, const float *b_qkv,
                                   const float *key_mask, void *out, int B, int N, int hidden, int H,
                                   int block_per_row, int approx_mode, int first_n, int diag_n,
                                   cudaStream_t stream);

/* The layer's projection alone: qkv (DEVICE bf16 [3][B][H][N][Dp], 16-byte
 * aligned, Dp = 32 when d <= 32 else 64) gets the projected, head-split,
 * zero-padded Q (scaled by sqrt(Dp / d)), K and V of mra_self_attention_fwd.
 * Arguments as there.  Returns an mra_status value. */
MRA_API int mra_qkv_projection(const void *x, const void *w_qkv, const float *b_qkv, void *qkv,
                               int B, int N, int hidden, int H, cudaStream_t stream);

/* num_block = min((N/32) * block_per_row, (N/32)^2); 0 for invalid input. */
MRA_API size_t mra_num_block(int N, int block_per_row);

/* Static text for an mra_status value. */
MRA_API const char *mra_status_string(int status);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device (a bitwise OR of MRA_DEV_* flags set by kernels since the
 * previous read), or -MRA_ERR_CUDA on a CUDA error. */
MRA_API int mra_get_device_status(cudaStream_t stream);

/* Maps a status word returned by mra_get_device_status or
 * mra_get_noalloc_status to an mra_status: a negative word is the negated
 * error of the read itself; MRA_DEV_TIMEOUT gives MRA_ERR_DEVICE_TIMEOUT (a
 * kernel stopped early, its output is incomplete); MRA_DEV_COUNT gives
 * MRA_ERR_INVALID_ARG (a selection or block list the kernels refused: those
 * heads have no output); MRA_DEV_KEY_RANGE alone (the selection order may
 * differ from exact additive biases, the output is still computed) and 0
 * give MRA_OK.  Host code, no CUDA call. */
MRA_API int mra_status_from_device(int word);

/* Kernel timing for benchmarks.  When enabled, the library records CUDA events
 * on `stream` around each kernel phase of every call; mra_profile_read
 * synchronises on the last recorded event and returns, per phase, the number
 * of launches and the summed milliseconds since the previous read.  Phase
 * names are static strings.  Returns the number of phases written (<= max). */
MRA_API void mra_profile_enable(int enable);
MRA_API int mra_profile_read(const char **names, int *launches, double *total_ms, int max);

/* Number of kernel launches issued by the most recent forward call. */
MRA_API int mra_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MRA_B200_H */
