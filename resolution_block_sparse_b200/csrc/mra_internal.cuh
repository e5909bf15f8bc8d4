// mra_internal.cuh - shared declarations of the B200 MRA-2 forward library.
//
// The forward pass of the page "深入解析 Transformers 中的 MRA 模型" (steps one
// to four of "源码级原理：MRA 两级注意力到底怎么算") is split into these phases,
// all enqueued on the caller's stream:
//   pool        masked 32-token block means of Q, K (and V in full mode)
//   lowres      low-resolution logits, row max, 64-bit selection keys, first
//               radix histogram of the global top-k
//   select      remaining radix passes, per-row counts, row scan with the
//               attention work list, CSR column lists
//   lowres_pv   (full mode) low-resolution weights times pooled V for the
//               unselected blocks of every block row
//   attention   exact softmax attention on the selected 32x32 blocks with an
//               online max/sum, merged with the low-resolution part
#pragma once

#include <cuda_bf16.h>

#include <utility>

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mra {

constexpr int kBlock = 32;            // tokens per block (fixed by the method)
constexpr int kChunk = 32;            // upper bound of the blocks per attention work item
constexpr int kHist0Bits = 11;        // radix digit widths over the 35-bit key
constexpr int kHist1Bits = 12;
constexpr int kHist2Bits = 12;
constexpr int kHistBins = 4096;       // per-pass histogram stride per head
constexpr int kMaxN = 65536;

// Device status bits (mirrors of the public MRA_DEV_* values).
constexpr unsigned kDevKeyRange = 1u;
constexpr unsigned kDevCount = 2u;
constexpr unsigned kDevTimeout = 4u;

struct SelState {
    unsigned long long prefix;  // key bits fixed so far (threshold after the last pass)
    unsigned int need;          // elements still to take from the current bucket
    unsigned int pad;
};

struct WorkItem {
    int row;         // global block row id: bh * nbr + r
    int col_start;   // offset into cols[] of the first column of this chunk
    int ncols;       // number of selected columns in this chunk (0..kChunk)
    int chunk_info;  // chunk | (nchunks << 16)
};

// Work item of the tcgen05 attention kernel: a group of kGroupRows adjacent
// block rows of one head (M = 128 query rows) and a chunk of the union of
// their selected key blocks.
constexpr int kGroupRows = 4;
struct GroupItem {
    int group;       // bh * ngroups + g (block rows kGroupRows*g ..)
    int ustart;      // index into ucols[] of the chunk's first union entry
    int ucount;      // union entries in this chunk (0..gchunk)
    int chunk_info;  // chunk | (nchunks << 16)
};
// Union entry: key block c | (rows of the group that selected it, 4 bits) << 16
// | (the key block is partly padded) << 20.
constexpr int kUnionRowShift = 16;
constexpr int kUnionPartial = 1 << 20;

struct Problem {
    int B, H, N, D, nbr, BH;
    long long nbr2;
    int k;            // num_block
    int mode;         // 0 full, 1 sparse
    int first_n, diag_n;
    int dtype;        // 0 bf16, 1 f32
    int chunk;        // selected blocks per attention work item (8, 16 or 32)
    int cap;          // work-item slots per head: nbr + k / chunk
    int r_tile;       // rows per CTA of the low-res kernels
    int lowres_ctas;  // CTAs per head of the low-res key kernel
    int bwd;          // the workspace also holds the backward pass's buffers
    int layer;        // the workspace also holds the layer's Q/K/V and output (bf16 [B][H][N][D] each)
    int fused;        // single-launch pass for small maps: -1 by preference, 0 never, 1 wherever it fits
    int ngroups;      // groups of kGroupRows block rows per head
    int gchunk;       // union key blocks per tcgen05 work item (16, 32 or 64)
    int gcap;         // tcgen05 work-item slots per head: ngroups + k / gchunk
};

struct Workspace {
    // zero-initialised every call (one memset)
    unsigned int *hist;      // [BH][3][kHistBins]
    unsigned int *arrive;    // [BH][4]
    int *row_arrive;         // [BH*nbr]
    int *work_next;          // [4]: [0] attention work-item counter, [1] the tcgen05
                             // kernel's counter, [2] most tcgen05 items of any head
    int *group_arrive;       // [BH*ngroups]: split-group arrivals (tcgen05 kernel)
    int *slot_arrive;        // [BH*cap]: arrivals of a split row's item groups (warp-level kernels)
    size_t zero_bytes;       // the whole region
    size_t zero_bytes_no_hist;   // the region without the radix histograms and the candidate counts
    void *zero_base;
    // written before read every call
    int *cnt;                // [B][nbr]
    float *pooled;           // [3][BH][nbr][D]
    unsigned long long *keys;// [BH][nbr2]
    float *lo_logits;        // [BH][nbr2] low-resolution logit map (full mode, maps over 128 x 128)
    float *lo_pmax;          // [BH][nbr][ceil(nbr / 128)] per-tile row maxima of the logit map
    float *mlo;              // [BH][nbr]
    SelState *state;         // [BH]
    int *ccount;             // [BH] candidates of the first digit's bucket (zeroed region)
    unsigned long long *cand_key;   // [BH][nbr2] the bucket's keys (maps over 128 x 128)
    int *cand_idx;           // [BH][nbr2] their flat indices r * nbr + c
    unsigned int *tiebits;   // [BH*nbr][words_per_row] keys equal to the threshold
    int *above_cnt;          // [BH*nbr] per row: keys above the first digit's bucket
    int *row_start;          // [BH*nbr] CSR offset of each row's columns in cols[]
    int *row_take;           // [BH*nbr] keys equal to the threshold that each row takes
    int *cols;               // [BH*k]
    unsigned int *bitmap;    // [BH*nbr][words_per_row]
    int words_per_row;
    WorkItem *items;         // [BH*cap]
    int *head_items;         // [BH]
    float *lo_opart;         // [splits][BH*nbr][D] partial low-resolution outputs (tensor-core kernel)
    float *lo_lpart;         // [splits][BH*nbr] partial normalisers
    float *olo;              // [BH*nbr][D]
    float *llo;              // [BH*nbr]
    float *partial;          // [BH*cap][32*(D+2)], or [BH*gcap][128*(D+2)] for the tcgen05 kernel
    int *ucols;              // [BH*k]: union entries of the groups (tcgen05 kernel)
    GroupItem *gitems;       // [BH*gcap]
    int *head_gitems;        // [BH]
    unsigned int *status;    // 1 word, persistent across calls
    // backward pass only (Problem::bwd)
    float *lse2, *delta;     // [BH*N]: base-2 log-sum-exp and dout . out per query
    float *lo_ab;            // [BH*nbr][D+4]: A, B, R, valid of each row block
    float *lo_dxh;           // [3][BH][nbr][D]: gradients of the block means
    // layer only (Problem::layer)
    void *lqkv;              // [3][B][H][N][D] bf16: projected, head-split Q, K, V
    void *lout;              // [B][H][N][D] bf16: attention output before the head merge
};

// Number of SMs of the current device (cached per device; thread-safe).
int device_sm_count();

// Planning and the launch sequence shared by the entry points (mra_api.cu).
int validate_sizes(int B, int H, int N, int D, int bpr, int mode, int first_n, int diag_n);
int validate(const void *q, const void *k, const void *v, const void *out, int B, int H, int N,
             int D, int bpr, int mode, int first_n, int diag_n);
Problem make_problem(int B, int H, int N, int D, int bpr, int mode, int first_n, int diag_n,
                     int dtype);
// Sets the per-head block budget k and the work-item plan that follows from it.
void set_budget(Problem &p, int k);
// Carves the workspace out of base (size only when base is null); returns bytes.
size_t carve_workspace(const Problem &p, char *base, Workspace *w);
int enqueue_forward(const Problem &p, const Workspace &w, const void *q, const void *k,
                    const void *v, const float *mask, void *out, int32_t *sel_out,
                    float *logit_out, float *pooled_out, cudaStream_t s, bool profile,
                    int *launch_count, const struct GradStats *gs = nullptr,
                    const struct OutLayout *ol = nullptr);

// Launchers (each returns cudaGetLastError() of its launches).
// What the backward pass takes from a forward run, per query row: the base-2
// log-sum-exp of the row's terms (high and low resolution, under the true
// maximum; +inf where the output is the constant 0) and delta = dout . out
// from the fp32 output before rounding.  lse2 == nullptr: not wanted.
struct GradStats {
    const void *dout;   // [rows][D] in the input dtype
    int dout_f32;
    float *lse2, *delta;
    size_t qbase;       // global query row of the block's first row
    __device__ __forceinline__ float dout_at(size_t i) const {
        return dout_f32 ? static_cast<const float *>(dout)[i]
                        : __bfloat162float(static_cast<const __nv_bfloat16 *>(dout)[i]);
    }
};

// ---------------------------------------------------------------- dependent launches
// Every kernel after the first of a forward pass is launched with
// programmatic stream serialization: it may be scheduled while the kernel
// before it drains, and it calls pdl_wait() (which returns once every earlier
// kernel of the stream has completed and its writes are visible) before it
// touches their results.  No kernel triggers its dependents early: dependents
// made resident early took SM space from the running kernel (the N=4096
// graph-replayed pass 3 us slower).  Without the launch attribute the wait is
// a no-op.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

cudaError_t launch_pool(const Problem &p, const Workspace &w, const void *q, const void *k,
                        const void *v, const float *mask, cudaStream_t s);
cudaError_t launch_lowres_keys(const Problem &p, const Workspace &w, float *logit_out,
                               cudaStream_t s);
// Selection of maps above 128 x 128 after the keys kernel: one pass over the
// keys (certain selections into the bitmap, the first digit's bucket into a
// candidate list); then one CTA per head (threshold, row counts, scan, work
// list) followed by the column lists, one warp per row (both launched by
// launch_select_finalize).
cudaError_t launch_select_scan(const Problem &p, const Workspace &w, cudaStream_t s);
cudaError_t launch_select_finalize(const Problem &p, const Workspace &w, int32_t *sel_out, cudaStream_t s);
// Low-resolution logits, keys and the whole selection in one kernel: one
// thread-block cluster per head (nbr <= 128).
bool lowres_select_fused_supported(const Problem &p);
cudaError_t launch_lowres_select_fused(const Problem &p, const Workspace &w, float *logit_out,
                                       int32_t *sel_out, cudaStream_t s);
cudaError_t launch_lowres_pv(const Problem &p, const Workspace &w, const float *logit_out, cudaStream_t s);
// column splits of the low-resolution kernel (1: no partials)
int lowres_pv_splits(const Problem &p);
// Output layout of the attention kernels: element (b, h, n, e) of the
// [B][H][N][D] result at out[b * ob + h * oh + n * orow + e] (null: the
// contiguous [B][H][N][D] layout).
struct OutLayout {
    long long ob;
    int oh, orow;
};
cudaError_t launch_attention(const Problem &p, const Workspace &w, const void *q, const void *k,
                             const void *v, const float *mask, void *out, cudaStream_t s,
                             const GradStats *gs = nullptr, const OutLayout *ol = nullptr);
cudaError_t launch_backward_items(const Problem &p, const Workspace &w, const void *q, const void *k,
                                  const void *v, const float *mask, const void *dout, float *dq, float *dk,
                                  float *dv, cudaStream_t s);
cudaError_t launch_backward_lowres(const Problem &p, const Workspace &w, const float *mask, const void *dout,
                                   float *dq, float *dk, float *dv, cudaStream_t s);
// tcgen05 / TMA attention (bf16, D = 64): groups of four block rows over the
// union of their selected key blocks.  group_plan builds the unions and the
// work items from the per-row items and column lists of the selection (or of
// a block list); launch_attention runs the kernel when supported.
bool attention_tc_supported(const Problem &p);
// have_counts: the pool kernel's valid-token counts of this call are in the
// workspace (not so for block lists).
cudaError_t launch_group_plan(const Problem &p, const Workspace &w, const float *mask, bool have_counts,
                              cudaStream_t s);
// Whether launch_attention takes the tcgen05 kernel for this problem (gs: the
// backward pass's statistics are wanted, which the warp-level kernels export).
bool attention_uses_tc(const Problem &p, const GradStats *gs);
cudaError_t launch_attention_tc(const Problem &p, const Workspace &w, const void *q, const void *k,
                                const void *v, const float *mask, void *out, const OutLayout *ol,
                                cudaStream_t s);
// Block-sparse attention on caller-given block lists (mra_blocklist.cu): the
// work items, column lists and per-call counters from lists [BH][cap_sel]
// of ascending flat block indices padded with -1 (p.k == cap_sel).
cudaError_t launch_blocklist_items(const Problem &p, const Workspace &w, const int32_t *lists, int cap_sel,
                                   cudaStream_t s);
// The MraSelfAttention layer (mra_layer.cu): head size d padded to 32 or 64;
// the Q/K/V projection (tcgen05 GEMM, head-split epilogue) and the head merge.
int head_padded_size(int d);
cudaError_t launch_qkv_projection(const void *x, const void *w, const float *bias, void *qkv, int B, int N,
                                  int hidden, int H, unsigned int *status, cudaStream_t s);
cudaError_t launch_merge_heads(const void *o, void *out, int B, int N, int H, int d, cudaStream_t s);
// The whole forward pass of one (batch, head) per CTA for maps of at most
// 16 x 16 blocks whose head fits in shared memory (mra_fused.cu); writes the
// same intermediates as the multi-kernel path when asked.
bool fused_small_supported(const Problem &p);
bool fused_small_preferred(const Problem &p);
cudaError_t launch_fused_small(const Problem &p, const Workspace &w, const void *q, const void *k, const void *v,
                               const float *mask, void *out, int32_t *sel_out, float *logit_out, float *pooled_out,
                               const OutLayout *ol, cudaStream_t s);
// The BigBird pattern of one head as ascending flat 32-token block indices
// (host code); returns an mra_status value.
int bigbird_block_list(int N, int block_size, int num_random, const int32_t *rand_blocks, int32_t *out,
                       int capacity, int *count);

// ---------------------------------------------------------------- device helpers
#ifdef __CUDACC__
// Order-preserving map of a float to an unsigned integer (larger float ->
// larger integer); -0 is canonicalised to +0 before the call.
__device__ __forceinline__ unsigned int float_order_bits(float x) {
    unsigned int u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float float_from_order_bits(unsigned int u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
// Diagonal prior of width g: key-block offsets c - r in -(g/2) .. (g+1)/2 - 1.
__device__ __forceinline__ int prior_band(int r, int c, int g) {
    if (g <= 0) return 0;
    const int off = c - r;
    return (off >= -(g / 2) && off <= (g + 1) / 2 - 1) ? 1 : 0;
}
// Selection key of block (r, c) (page "深入解析 Transformers 中的 MRA 模型",
// section "源码级原理", step two): the additive priors as the exact pair
// (tier, x), x = l - rowmax in fp32 (canonical +0), packed as
// (tier + 4) << 32 | order bits of x.  range_err is set when |x| >= 2500,
// where the pair's order could differ from the order of the biased sums.
__device__ __forceinline__ unsigned long long selection_key(float l, float rowmax, int r, int c, int first_n,
                                                            int diag_n, bool row_empty, bool col_empty,
                                                            int &range_err) {
    float x = l - rowmax;
    if (x == 0.0f) x = 0.0f;
    if (!(fabsf(x) < 2500.0f)) range_err = 1;
    int tier = 0;
    if (first_n > 0 && (r < first_n || c < first_n)) ++tier;
    tier += prior_band(r, c, diag_n);
    if (row_empty) tier -= 2;
    if (col_empty) tier -= 2;
    return ((unsigned long long)(tier + 4) << 32) | (unsigned long long)float_order_bits(x);
}
#endif

}  // namespace mra
