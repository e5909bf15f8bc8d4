// mra_api.cu - the C ABI of include/mra.h: argument checks, the per-device
// workspace, and the stream-ordered launch sequence of the forward pass.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "mra.h"
#include "mra_internal.cuh"

using namespace mra;

namespace mra {

// ---------------------------------------------------------------- planning
size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

int device_sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

int validate_sizes(int B, int H, int N, int D, int bpr, int mode, int first_n, int diag_n) {
    if (B < 1 || H < 1 || N < kBlock || (N % kBlock) != 0 || bpr < 1) return MRA_ERR_INVALID_ARG;
    if (mode != MRA_FULL && mode != MRA_SPARSE) return MRA_ERR_INVALID_ARG;
    const int nbr = N / kBlock;
    if (first_n < 0 || first_n > nbr || diag_n < 0 || diag_n > nbr) return MRA_ERR_INVALID_ARG;
    if (D != 32 && D != 64) return MRA_ERR_UNSUPPORTED;
    if (N > kMaxN) return MRA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    if (BH > 65535) return MRA_ERR_UNSUPPORTED;
    const long long kk = std::min<long long>((long long)nbr * bpr, (long long)nbr * nbr);
    if (BH * kk > 0x7fffffffLL || BH * ((long long)nbr + kk / 8) > 0x7fffffffLL)
        return MRA_ERR_UNSUPPORTED;
    return MRA_OK;
}

int validate(const void *q, const void *k, const void *v, const void *out, int B, int H, int N,
             int D, int bpr, int mode, int first_n, int diag_n) {
    if (!q || !k || !v || !out) return MRA_ERR_INVALID_ARG;
    if ((((uintptr_t)q) | ((uintptr_t)k) | ((uintptr_t)v) | ((uintptr_t)out)) & 15u)
        return MRA_ERR_INVALID_ARG;
    return validate_sizes(B, H, N, D, bpr, mode, first_n, diag_n);
}

Problem make_problem(int B, int H, int N, int D, int bpr, int mode, int first_n, int diag_n,
                     int dtype) {
    Problem p;
    p.bwd = 0;
    p.layer = 0;
    p.fused = -1;
    p.B = B;
    p.H = H;
    p.N = N;
    p.D = D;
    p.nbr = N / kBlock;
    p.BH = B * H;
    p.nbr2 = (long long)p.nbr * p.nbr;
    p.mode = mode;
    p.first_n = first_n;
    p.diag_n = diag_n;
    p.dtype = dtype;
    set_budget(p, (int)std::min<long long>((long long)p.nbr * bpr, p.nbr2));
    // low-res rows per CTA: the logits of a CTA's rows stay in shared memory
    // (at most 64 KB), so longer maps take fewer rows per CTA
    p.r_tile = p.nbr > 1024 ? 8 : 16;
    p.lowres_ctas = (p.nbr + p.r_tile - 1) / p.r_tile;
    return p;
}

void set_budget(Problem &p, int k) {
    p.k = k;
    // work items of at most `chunk` blocks: short items keep the critical path
    // of the long (prior) rows short when rows hold few blocks on average;
    // longer items amortise the split-row merge when rows are dense
    const int per_row = (p.k + p.nbr - 1) / p.nbr;
    p.chunk = per_row <= 4 ? 8 : (per_row <= 16 ? 16 : kChunk);
    p.cap = p.nbr + p.k / p.chunk;
    // tcgen05 kernel: items of at most gchunk union key blocks per group of
    // four block rows; sparse maps take short items so that the long prior
    // rows split over many CTAs, dense maps long ones (fewer merges)
    p.ngroups = (p.nbr + kGroupRows - 1) / kGroupRows;
    p.gchunk = per_row <= 4 ? 16 : (per_row <= 16 ? 32 : 64);
    p.gcap = p.ngroups + p.k / p.gchunk;
}

// Carves the workspace; with base == nullptr only computes the size.
size_t carve_workspace(const Problem &p, char *base, Workspace *w) {
    size_t off = 0;
    auto take = [&](size_t bytes) -> char * {
        char *ptr = base ? base + off : nullptr;
        off += align_up(bytes);
        return ptr;
    };
    const size_t BH = (size_t)p.BH, nbr = (size_t)p.nbr, D = (size_t)p.D;
    Workspace t{};
    // zeroed region (the radix histograms last: the fused selection does
    // not use them, so its calls clear only the part before them)
    t.arrive = (unsigned int *)take(sizeof(unsigned int) * BH * 4);
    t.row_arrive = (int *)take(sizeof(int) * BH * nbr);
    t.work_next = (int *)take(sizeof(int) * 4);
    t.group_arrive = (int *)take(sizeof(int) * BH * (size_t)p.ngroups);
    t.slot_arrive = (int *)take(sizeof(int) * BH * (size_t)p.cap);
    t.zero_bytes_no_hist = off;
    t.hist = (unsigned int *)take(sizeof(unsigned int) * BH * 3 * kHistBins);
    t.ccount = (int *)take(sizeof(int) * BH);
    t.zero_base = t.arrive;
    t.zero_bytes = off;
    t.cnt = (int *)take(sizeof(int) * (size_t)p.B * nbr);
    t.pooled = (float *)take(sizeof(float) * 3 * BH * nbr * D);
    t.keys = (unsigned long long *)take(sizeof(unsigned long long) * BH * (size_t)p.nbr2);
    t.lo_logits = (float *)take(sizeof(float) * BH * (size_t)p.nbr2);
    t.lo_pmax = (float *)take(sizeof(float) * BH * nbr * ((nbr + 127) / 128));
    t.mlo = (float *)take(sizeof(float) * BH * nbr);
    t.state = (SelState *)take(sizeof(SelState) * BH);
    t.cols = (int *)take(sizeof(int) * BH * (size_t)p.k);
    t.words_per_row = (p.nbr + 31) / 32;
    t.bitmap = (unsigned int *)take(sizeof(unsigned int) * BH * nbr * (size_t)t.words_per_row);
    if (!lowres_select_fused_supported(p)) {   // the multi-kernel selection
        t.cand_key = (unsigned long long *)take(sizeof(unsigned long long) * BH * (size_t)p.nbr2);
        t.cand_idx = (int *)take(sizeof(int) * BH * (size_t)p.nbr2);
        t.tiebits = (unsigned int *)take(sizeof(unsigned int) * BH * nbr * (size_t)t.words_per_row);
        t.above_cnt = (int *)take(sizeof(int) * BH * nbr);
        t.row_start = (int *)take(sizeof(int) * BH * nbr);
        t.row_take = (int *)take(sizeof(int) * BH * nbr);
    }
    t.items = (WorkItem *)take(sizeof(WorkItem) * BH * (size_t)p.cap);
    t.head_items = (int *)take(sizeof(int) * BH);
    {
        const int sp = lowres_pv_splits(p);
        if (sp > 1) {
            t.lo_opart = (float *)take(sizeof(float) * (size_t)sp * BH * nbr * D);
            t.lo_lpart = (float *)take(sizeof(float) * (size_t)sp * BH * nbr);
        }
    }
    t.olo = (float *)take(sizeof(float) * BH * nbr * D);
    t.llo = (float *)take(sizeof(float) * BH * nbr);
    t.partial = (float *)take(sizeof(float) * BH * (D + 2) *
                              std::max((size_t)p.cap * 32, (size_t)p.gcap * 32 * kGroupRows));
    t.ucols = (int *)take(sizeof(int) * BH * (size_t)p.k);
    t.gitems = (GroupItem *)take(sizeof(GroupItem) * BH * (size_t)p.gcap);
    t.head_gitems = (int *)take(sizeof(int) * BH);
    if (p.bwd) {
        t.lse2 = (float *)take(sizeof(float) * BH * (size_t)p.N);
        t.delta = (float *)take(sizeof(float) * BH * (size_t)p.N);
        t.lo_ab = (float *)take(sizeof(float) * BH * nbr * (D + 4));
        t.lo_dxh = (float *)take(sizeof(float) * 3 * BH * nbr * D);
    }
    if (p.layer) {
        t.lqkv = take(2 * 3 * BH * (size_t)p.N * D);
        t.lout = take(2 * BH * (size_t)p.N * D);
    }
    if (w) *w = t;
    return off;
}

}  // namespace mra

namespace {

constexpr int kMaxDevices = 64;

struct DeviceCtx {
    void *ws = nullptr;
    size_t ws_bytes = 0;
    unsigned int *status = nullptr;  // persistent status word
    void *stage = nullptr;           // host-entry staging buffers
    size_t stage_bytes = 0;
    // host entry: copy streams (inputs in, outputs out) and per-chunk events
    cudaStream_t s_in = nullptr, s_out = nullptr;
    std::vector<cudaEvent_t> events;
};

std::mutex g_mutex;
DeviceCtx g_dev[kMaxDevices];
int g_last_launches = 0;

// ---------------------------------------------------------------- profiling
struct PhaseStat {
    const char *name;
    int launches;
    double ms;
};
struct PendingEvent {
    int phase;
    cudaEvent_t start, stop;
};
bool g_prof = false;
std::vector<PhaseStat> g_phase;
std::vector<PendingEvent> g_pending;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

int phase_index(const char *name) {
    for (size_t i = 0; i < g_phase.size(); ++i)
        if (std::strcmp(g_phase[i].name, name) == 0) return (int)i;
    g_phase.push_back({name, 0, 0.0});
    return (int)g_phase.size() - 1;
}

struct PhaseScope {
    bool on;
    PendingEvent pe;
    cudaStream_t s;
    PhaseScope(const char *name, cudaStream_t st, bool enabled) : on(enabled), s(st) {
        if (!on) return;
        pe.phase = phase_index(name);
        pe.start = take_event();
        pe.stop = take_event();
        cudaEventRecord(pe.start, s);
    }
    ~PhaseScope() {
        if (!on) return;
        cudaEventRecord(pe.stop, s);
        g_pending.push_back(pe);
    }
};

int ensure_workspace(int dev, const Problem &p, Workspace *w) {
    DeviceCtx &ctx = g_dev[dev];
    if (!ctx.status) {
        if (cudaMalloc(&ctx.status, 256) != cudaSuccess) return MRA_ERR_ALLOC;
        if (cudaMemset(ctx.status, 0, 256) != cudaSuccess) return MRA_ERR_CUDA;
    }
    const size_t need = carve_workspace(p, nullptr, nullptr);
    if (need > ctx.ws_bytes) {
        // MRA_TEST_FAIL_ALLOC=1 (read at every growth) makes the growth fail
        // as an allocation failure would, before any CUDA call: the error path
        // of every entry point can be tested without exhausting the device
        const char *fail = getenv("MRA_TEST_FAIL_ALLOC");
        if (fail && fail[0] == '1') return MRA_ERR_ALLOC;
        if (ctx.ws) {
            cudaDeviceSynchronize();
            cudaFree(ctx.ws);
            ctx.ws = nullptr;
            ctx.ws_bytes = 0;
        }
        size_t bytes = need + need / 4;
        if (cudaMalloc(&ctx.ws, bytes) != cudaSuccess) {
            cudaGetLastError();
            return MRA_ERR_ALLOC;
        }
        ctx.ws_bytes = bytes;
    }
    carve_workspace(p, static_cast<char *>(ctx.ws), w);
    w->status = ctx.status;
    return MRA_OK;
}

int current_device(int *dev) {
    if (cudaGetDevice(dev) != cudaSuccess) return MRA_ERR_CUDA;
    if (*dev < 0 || *dev >= kMaxDevices) return MRA_ERR_UNSUPPORTED;
    return MRA_OK;
}

#define MRA_TRY(expr)                              \
    do {                                           \
        cudaError_t e_ = (expr);                   \
        if (e_ != cudaSuccess) return MRA_ERR_CUDA; \
    } while (0)

}  // namespace

namespace mra {

// The stream-ordered launch sequence of one forward pass on a prepared
// workspace (shared by every entry point).  profile enables the per-phase
// CUDA events of mra_profile_enable.
int enqueue_forward(const Problem &p, const Workspace &w, const void *q, const void *k,
                    const void *v, const float *mask, void *out, int32_t *sel_out,
                    float *logit_out, float *pooled_out, cudaStream_t s, bool profile,
                    int *launch_count, const GradStats *gs, const OutLayout *ol) {
    const bool prof = profile && g_prof;
    int launches = 0;
    // small maps: the whole pass of a head in one CTA, one launch, where that
    // is faster (MRA_FUSED=1 takes it wherever it fits, MRA_FUSED=0 never)
    const char *fused_env = getenv("MRA_FUSED");
    const bool fused = fused_env && fused_env[0] == '0'   ? false
                       : fused_env && fused_env[0] == '1' ? true
                       : p.fused >= 0                     ? p.fused == 1
                                                          : fused_small_preferred(p);
    if (!gs && fused && fused_small_supported(p)) {
        PhaseScope ps("fused", s, prof);
        MRA_TRY(launch_fused_small(p, w, q, k, v, mask, out, sel_out, logit_out, pooled_out, ol, s));
        *launch_count = 1;
        return MRA_OK;
    }
    {
        // the pool kernel also clears the per-call counters and histograms
        PhaseScope ps("pool", s, prof);
        MRA_TRY(launch_pool(p, w, q, k, v, mask, s));
        ++launches;
    }
    if (lowres_select_fused_supported(p)) {
        PhaseScope ps("lowres_select", s, prof);
        MRA_TRY(launch_lowres_select_fused(p, w, logit_out, sel_out, s));
        ++launches;
    } else {
        {
            PhaseScope ps("lowres_keys", s, prof);
            MRA_TRY(launch_lowres_keys(p, w, logit_out, s));
            ++launches;
        }
        PhaseScope ps("select", s, prof);
        MRA_TRY(launch_select_scan(p, w, s));
        MRA_TRY(launch_select_finalize(p, w, sel_out, s));
        launches += 3;
    }
    if (p.mode == MRA_FULL) {
        PhaseScope ps("lowres_pv", s, prof);
        MRA_TRY(launch_lowres_pv(p, w, logit_out, s));
        ++launches;
    }
    if (attention_uses_tc(p, gs)) {
        PhaseScope ps("group_plan", s, prof);
        MRA_TRY(launch_group_plan(p, w, mask, true, s));
        ++launches;
    }
    {
        PhaseScope ps("attention", s, prof);
        MRA_TRY(launch_attention(p, w, q, k, v, mask, out, s, gs, ol));
        ++launches;
    }
    if (pooled_out) {
        const size_t plane = sizeof(float) * (size_t)p.BH * p.nbr * p.D;
        MRA_TRY(cudaMemcpyAsync(pooled_out, w.pooled, p.mode == MRA_FULL ? 3 * plane : 2 * plane,
                                cudaMemcpyDeviceToDevice, s));
        if (p.mode != MRA_FULL)
            MRA_TRY(cudaMemsetAsync(reinterpret_cast<char *>(pooled_out) + 2 * plane, 0, plane, s));
    }
    *launch_count = launches;
    return MRA_OK;
}

}  // namespace mra

namespace {

// The forward pass proper; the caller holds g_mutex.
int forward_locked(const void *q, const void *k, const void *v, const float *mask, void *out,
                   int B, int H, int N, int D, int bpr, int mode, int first_n, int diag_n,
                   int dtype, int32_t *sel_out, float *logit_out, float *pooled_out,
                   cudaStream_t s, int fused = -1) {
    int rc = validate(q, k, v, out, B, H, N, D, bpr, mode, first_n, diag_n);
    if (rc != MRA_OK) return rc;
    if (dtype != MRA_DTYPE_BF16 && dtype != MRA_DTYPE_F32) return MRA_ERR_INVALID_ARG;
    if (mask && (((uintptr_t)mask) & 3u)) return MRA_ERR_INVALID_ARG;
    int dev;
    rc = current_device(&dev);
    if (rc != MRA_OK) return rc;
    Problem p = make_problem(B, H, N, D, bpr, mode, first_n, diag_n, dtype);
    p.fused = fused;
    Workspace w;
    rc = ensure_workspace(dev, p, &w);
    if (rc != MRA_OK) return rc;

    int launches = 0;
    rc = enqueue_forward(p, w, q, k, v, mask, out, sel_out, logit_out, pooled_out, s, true,
                         &launches);
    if (rc != MRA_OK) return rc;
    g_last_launches = launches;
    return MRA_OK;
}

// The backward pass: the forward pass (same selection, the attention kernel
// exporting each query's log-sum-exp and dout . out, its output written to
// dq as scratch), then the gradient kernels.  The caller holds g_mutex.
int backward_locked(const void *q, const void *k, const void *v, const float *mask, const void *dout,
                    float *dq, float *dk, float *dv, int B, int H, int N, int D, int bpr, int mode,
                    int first_n, int diag_n, int dtype, cudaStream_t s) {
    int rc = validate(q, k, v, dq, B, H, N, D, bpr, mode, first_n, diag_n);
    if (rc != MRA_OK) return rc;
    if (!dout || !dk || !dv) return MRA_ERR_INVALID_ARG;
    if ((((uintptr_t)dout) | ((uintptr_t)dk) | ((uintptr_t)dv)) & 15u) return MRA_ERR_INVALID_ARG;
    if (mask && (((uintptr_t)mask) & 3u)) return MRA_ERR_INVALID_ARG;
    int dev;
    rc = current_device(&dev);
    if (rc != MRA_OK) return rc;
    Problem p = make_problem(B, H, N, D, bpr, mode, first_n, diag_n, dtype);
    p.bwd = 1;
    Workspace w;
    rc = ensure_workspace(dev, p, &w);
    if (rc != MRA_OK) return rc;
    GradStats gs{};
    gs.dout = dout;
    gs.dout_f32 = dtype == MRA_DTYPE_F32 ? 1 : 0;
    gs.lse2 = w.lse2;
    gs.delta = w.delta;
    int launches = 0;
    rc = enqueue_forward(p, w, q, k, v, mask, dq, nullptr, nullptr, nullptr, s, true, &launches, &gs);
    if (rc != MRA_OK) return rc;
    const bool prof = g_prof;
    if (mode == MRA_FULL) {
        // the low-resolution pass writes every element of dq, dk and dv
        PhaseScope ps("bwd_lowres", s, prof);
        MRA_TRY(launch_backward_lowres(p, w, mask, dout, dq, dk, dv, s));
    } else {
        PhaseScope ps("bwd_clear", s, prof);
        const size_t bytes = sizeof(float) * (size_t)B * H * N * D;
        MRA_TRY(cudaMemsetAsync(dq, 0, bytes, s));
        MRA_TRY(cudaMemsetAsync(dk, 0, bytes, s));
        MRA_TRY(cudaMemsetAsync(dv, 0, bytes, s));
    }
    {
        PhaseScope ps("bwd_items", s, prof);
        MRA_TRY(launch_backward_items(p, w, q, k, v, mask, dout, dq, dk, dv, s));
    }
    g_last_launches = launches + (mode == MRA_FULL ? 4 : 1);
    return MRA_OK;
}

// Block-sparse attention on given block lists: the list kernel (work items,
// column lists, per-call counters), then the attention kernel in sparse
// mode.  The caller holds g_mutex.
int blocksparse_locked(const void *q, const void *k, const void *v, const float *mask, void *out, int B, int H,
                       int N, int D, const int32_t *lists, int cap_sel, int dtype, cudaStream_t s) {
    if (N < kBlock || (N % kBlock) != 0) return MRA_ERR_INVALID_ARG;
    const long long nbr = N / kBlock;
    if (cap_sel < 1 || cap_sel > nbr * nbr || !lists || (((uintptr_t)lists) & 3u)) return MRA_ERR_INVALID_ARG;
    const int bpr = (int)((cap_sel + nbr - 1) / nbr);
    int rc = validate(q, k, v, out, B, H, N, D, bpr, MRA_SPARSE, 0, 0);
    if (rc != MRA_OK) return rc;
    if (dtype != MRA_DTYPE_BF16 && dtype != MRA_DTYPE_F32) return MRA_ERR_INVALID_ARG;
    if (mask && (((uintptr_t)mask) & 3u)) return MRA_ERR_INVALID_ARG;
    int dev;
    rc = current_device(&dev);
    if (rc != MRA_OK) return rc;
    Problem p = make_problem(B, H, N, D, bpr, MRA_SPARSE, 0, 0, dtype);
    set_budget(p, cap_sel);
    Workspace w;
    rc = ensure_workspace(dev, p, &w);
    if (rc != MRA_OK) return rc;
    {
        PhaseScope ps("blocklist_items", s, g_prof);
        MRA_TRY(launch_blocklist_items(p, w, lists, cap_sel, s));
    }
    const bool tc = attention_uses_tc(p, nullptr);
    if (tc) {
        PhaseScope ps("group_plan", s, g_prof);
        MRA_TRY(launch_group_plan(p, w, mask, false, s));
    }
    {
        PhaseScope ps("attention", s, g_prof);
        MRA_TRY(launch_attention(p, w, q, k, v, mask, out, s));
    }
    g_last_launches = tc ? 3 : 2;
    return MRA_OK;
}

// Checks of the layer's arguments; d gets the head size.
int validate_layer(const void *x, const void *w_qkv, const float *b_qkv, const void *out, int B, int N, int hidden,
                   int H, int *d) {
    if (!x || !w_qkv || !out) return MRA_ERR_INVALID_ARG;
    if ((((uintptr_t)x) | ((uintptr_t)w_qkv) | ((uintptr_t)out)) & 15u) return MRA_ERR_INVALID_ARG;
    if (b_qkv && (((uintptr_t)b_qkv) & 3u)) return MRA_ERR_INVALID_ARG;
    if (B < 1 || N < kBlock || (N % kBlock) != 0 || H < 1 || hidden < H || hidden % H != 0) return MRA_ERR_INVALID_ARG;
    *d = hidden / H;
    if (*d > 64 || (hidden % 8) != 0) return MRA_ERR_UNSUPPORTED;
    if ((long long)B * N * 3 * hidden > 0x7fffffffLL) return MRA_ERR_UNSUPPORTED;
    return MRA_OK;
}

// The layer: projection, the forward pass on the projected heads, head merge.
// The caller holds g_mutex.
int layer_locked(const void *x, const void *w_qkv, const float *b_qkv, const float *mask, void *out, int B, int N,
                 int hidden, int H, int bpr, int mode, int first_n, int diag_n, cudaStream_t s) {
    int d = 0;
    int rc = validate_layer(x, w_qkv, b_qkv, out, B, N, hidden, H, &d);
    if (rc != MRA_OK) return rc;
    const int Dp = head_padded_size(d);
    rc = validate_sizes(B, H, N, Dp, bpr, mode, first_n, diag_n);
    if (rc != MRA_OK) return rc;
    if (mask && (((uintptr_t)mask) & 3u)) return MRA_ERR_INVALID_ARG;
    int dev;
    rc = current_device(&dev);
    if (rc != MRA_OK) return rc;
    Problem p = make_problem(B, H, N, Dp, bpr, mode, first_n, diag_n, MRA_DTYPE_BF16);
    p.layer = 1;
    Workspace w;
    rc = ensure_workspace(dev, p, &w);
    if (rc != MRA_OK) return rc;
    const size_t plane = 2 * (size_t)B * H * N * Dp;
    char *qkv = static_cast<char *>(w.lqkv);
    {
        PhaseScope ps("qkv_proj", s, g_prof);
        MRA_TRY(launch_qkv_projection(x, w_qkv, b_qkv, qkv, B, N, hidden, H, w.status, s));
    }
    int launches = 0;
    if (d == Dp) {
        // the attention writes the merged heads itself: element (b, h, n, e)
        // of the result is out[b][n][h*d + e]
        const OutLayout ol{(long long)N * hidden, d, hidden};
        rc = enqueue_forward(p, w, qkv, qkv + plane, qkv + 2 * plane, mask, out, nullptr, nullptr, nullptr, s,
                             true, &launches, nullptr, &ol);
        if (rc != MRA_OK) return rc;
        g_last_launches = launches + 1;
        return MRA_OK;
    }
    rc = enqueue_forward(p, w, qkv, qkv + plane, qkv + 2 * plane, mask, w.lout, nullptr, nullptr, nullptr, s, true,
                         &launches);
    if (rc != MRA_OK) return rc;
    {
        PhaseScope ps("merge_heads", s, g_prof);
        MRA_TRY(launch_merge_heads(w.lout, out, B, N, H, d, s));
    }
    g_last_launches = launches + 2;
    return MRA_OK;
}

}  // namespace

extern "C" {

int mra_blocksparse_attention_fwd(const void *q, const void *k, const void *v, const float *key_mask, void *out,
                                  int B, int H, int N, int D, const int32_t *block_idx, int cap_sel, int dtype,
                                  cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    return blocksparse_locked(q, k, v, key_mask, out, B, H, N, D, block_idx, cap_sel, dtype, stream);
}

int mra_qkv_projection(const void *x, const void *w_qkv, const float *b_qkv, void *qkv, int B, int N, int hidden,
                       int H, cudaStream_t stream) {
    int d = 0;
    int rc = validate_layer(x, w_qkv, b_qkv, qkv, B, N, hidden, H, &d);
    if (rc != MRA_OK) return rc;
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    rc = current_device(&dev);
    if (rc != MRA_OK) return rc;
    DeviceCtx &ctx = g_dev[dev];
    if (!ctx.status) {
        if (cudaMalloc(&ctx.status, 256) != cudaSuccess) return MRA_ERR_ALLOC;
        if (cudaMemset(ctx.status, 0, 256) != cudaSuccess) return MRA_ERR_CUDA;
    }
    MRA_TRY(launch_qkv_projection(x, w_qkv, b_qkv, qkv, B, N, hidden, H, ctx.status, stream));
    g_last_launches = 1;
    return MRA_OK;
}

int mra_self_attention_fwd(const void *x, const void *w_qkv, const float *b_qkv, const float *key_mask, void *out,
                           int B, int N, int hidden, int H, int block_per_row, int approx_mode, int first_n,
                           int diag_n, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    return layer_locked(x, w_qkv, b_qkv, key_mask, out, B, N, hidden, H, block_per_row, approx_mode, first_n,
                        diag_n, stream);
}

int mra_bigbird_block_list(int N, int block_size, int num_random, const int32_t *rand_blocks, int32_t *out,
                           int capacity, int *count) {
    return bigbird_block_list(N, block_size, num_random, rand_blocks, out, capacity, count);
}

int mra_attention_bwd(const void *q, const void *k, const void *v, const float *key_mask,
                      const void *dout, float *dq, float *dk, float *dv, int B, int H, int N, int D,
                      int block_per_row, int approx_mode, int first_n, int diag_n, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    return backward_locked(q, k, v, key_mask, dout, dq, dk, dv, B, H, N, D, block_per_row, approx_mode,
                           first_n, diag_n, MRA_DTYPE_BF16, stream);
}

int mra_attention_bwd_f32(const float *q, const float *k, const float *v, const float *key_mask,
                          const float *dout, float *dq, float *dk, float *dv, int B, int H, int N, int D,
                          int block_per_row, int approx_mode, int first_n, int diag_n, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    return backward_locked(q, k, v, key_mask, dout, dq, dk, dv, B, H, N, D, block_per_row, approx_mode,
                           first_n, diag_n, MRA_DTYPE_F32, stream);
}

int mra_attention_fwd(const void *q, const void *k, const void *v, const float *key_mask,
                      void *out, int B, int H, int N, int D, int block_per_row, int approx_mode,
                      int first_n, int diag_n, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    return forward_locked(q, k, v, key_mask, out, B, H, N, D, block_per_row, approx_mode, first_n,
                          diag_n, MRA_DTYPE_BF16, nullptr, nullptr, nullptr, stream);
}

int mra_attention_fwd_f32(const float *q, const float *k, const float *v, const float *key_mask,
                          float *out, int B, int H, int N, int D, int block_per_row,
                          int approx_mode, int first_n, int diag_n, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    return forward_locked(q, k, v, key_mask, out, B, H, N, D, block_per_row, approx_mode, first_n,
                          diag_n, MRA_DTYPE_F32, nullptr, nullptr, nullptr, stream);
}

int mra_attention_fwd_ex(const void *q, const void *k, const void *v, const float *key_mask,
                         void *out, int B, int H, int N, int D, int block_per_row,
                         int approx_mode, int first_n, int diag_n, int dtype, int32_t *sel_idx,
                         float *lowres_logit, float *pooled, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    return forward_locked(q, k, v, key_mask, out, B, H, N, D, block_per_row, approx_mode, first_n,
                          diag_n, dtype, sel_idx, lowres_logit, pooled, stream);
}

int mra_attention_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                           const float *key_mask_host, void *out_host, int B, int H, int N, int D,
                           int block_per_row, int approx_mode, int first_n, int diag_n, int dtype,
                           cudaStream_t stream) {
    if (!q_host || !k_host || !v_host || !out_host) return MRA_ERR_INVALID_ARG;
    if (dtype != MRA_DTYPE_BF16 && dtype != MRA_DTYPE_F32) return MRA_ERR_INVALID_ARG;
    int vrc = validate_sizes(B, H, N, D, block_per_row, approx_mode, first_n, diag_n);
    if (vrc != MRA_OK) return vrc;
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    int rc = current_device(&dev);
    if (rc != MRA_OK) return rc;
    const size_t esz = dtype == MRA_DTYPE_BF16 ? 2 : 4;
    const size_t tensor = align_up(esz * (size_t)B * H * N * D);
    const size_t mbytes = key_mask_host ? align_up(sizeof(float) * (size_t)B * N) : 0;
    const size_t need = 4 * tensor + mbytes;
    DeviceCtx &ctx = g_dev[dev];
    if (need > ctx.stage_bytes) {
        if (ctx.stage) {
            cudaDeviceSynchronize();
            cudaFree(ctx.stage);
            ctx.stage = nullptr;
            ctx.stage_bytes = 0;
        }
        if (cudaMalloc(&ctx.stage, need) != cudaSuccess) {
            cudaGetLastError();
            return MRA_ERR_ALLOC;
        }
        ctx.stage_bytes = need;
    }
    if (!ctx.s_in) {
        MRA_TRY(cudaStreamCreateWithFlags(&ctx.s_in, cudaStreamNonBlocking));
        MRA_TRY(cudaStreamCreateWithFlags(&ctx.s_out, cudaStreamNonBlocking));
    }
    // Chunks of heads within one batch entry (about eight in all): the
    // inputs of chunk c + 1 cross PCIe while chunk c is computed, and chunk
    // c's output goes back on a second copy stream while later inputs still
    // arrive.  Every (batch, head) is independent, so a chunk is a forward
    // pass of its own with B = 1.
    const int hc = std::max(1, std::min(H, (B * H + 7) / 8));
    const int per_b = (H + hc - 1) / hc;
    const int nchunks = B * per_b;
    while ((int)ctx.events.size() < 2 * nchunks + 1) {
        cudaEvent_t e = nullptr;
        MRA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
        ctx.events.push_back(e);
    }
    char *base = static_cast<char *>(ctx.stage);
    char *qd = base, *kd = base + tensor, *vd = base + 2 * tensor, *od = base + 3 * tensor;
    float *md = key_mask_host ? reinterpret_cast<float *>(base + 4 * tensor) : nullptr;
    // the copies follow the work already queued on `stream`
    MRA_TRY(cudaEventRecord(ctx.events[2 * nchunks], stream));
    MRA_TRY(cudaStreamWaitEvent(ctx.s_in, ctx.events[2 * nchunks], 0));
    if (md)
        MRA_TRY(cudaMemcpyAsync(md, key_mask_host, sizeof(float) * (size_t)B * N, cudaMemcpyHostToDevice,
                                ctx.s_in));
    const size_t head_bytes = esz * (size_t)N * D;
    for (int c = 0; c < nchunks; ++c) {
        const int b = c / per_b, h0 = (c % per_b) * hc, nh = std::min(hc, H - h0);
        const size_t off = ((size_t)b * H + h0) * head_bytes, bytes = (size_t)nh * head_bytes;
        MRA_TRY(cudaMemcpyAsync(qd + off, static_cast<const char *>(q_host) + off, bytes, cudaMemcpyHostToDevice,
                                ctx.s_in));
        MRA_TRY(cudaMemcpyAsync(kd + off, static_cast<const char *>(k_host) + off, bytes, cudaMemcpyHostToDevice,
                                ctx.s_in));
        MRA_TRY(cudaMemcpyAsync(vd + off, static_cast<const char *>(v_host) + off, bytes, cudaMemcpyHostToDevice,
                                ctx.s_in));
        MRA_TRY(cudaEventRecord(ctx.events[2 * c], ctx.s_in));
    }
    // the chunks take the path the whole problem would take, so that the
    // result is the device entry's, bit for bit
    const int fused = fused_small_preferred(make_problem(B, H, N, D, block_per_row, approx_mode, first_n, diag_n,
                                                         dtype)) ? 1 : 0;
    int launches = 0;
    for (int c = 0; c < nchunks; ++c) {
        const int b = c / per_b, h0 = (c % per_b) * hc, nh = std::min(hc, H - h0);
        const size_t off = ((size_t)b * H + h0) * head_bytes, bytes = (size_t)nh * head_bytes;
        MRA_TRY(cudaStreamWaitEvent(stream, ctx.events[2 * c], 0));
        rc = forward_locked(qd + off, kd + off, vd + off, md ? md + (size_t)b * N : nullptr, od + off, 1, nh, N, D,
                            block_per_row, approx_mode, first_n, diag_n, dtype, nullptr, nullptr, nullptr, stream,
                            fused);
        if (rc != MRA_OK) return rc;
        launches += g_last_launches;
        MRA_TRY(cudaEventRecord(ctx.events[2 * c + 1], stream));
        MRA_TRY(cudaStreamWaitEvent(ctx.s_out, ctx.events[2 * c + 1], 0));
        MRA_TRY(cudaMemcpyAsync(static_cast<char *>(out_host) + off, od + off, bytes, cudaMemcpyDeviceToHost,
                                ctx.s_out));
    }
    g_last_launches = launches;
    MRA_TRY(cudaStreamSynchronize(ctx.s_out));
    MRA_TRY(cudaStreamSynchronize(stream));
    return MRA_OK;
}

size_t mra_num_block(int N, int block_per_row) {
    if (N < kBlock || (N % kBlock) != 0 || block_per_row < 1) return 0;
    const long long nbr = N / kBlock;
    return (size_t)std::min<long long>(nbr * block_per_row, nbr * nbr);
}

const char *mra_status_string(int status) {
    switch (status) {
        case MRA_OK: return "ok";
        case MRA_ERR_INVALID_ARG: return "invalid argument";
        case MRA_ERR_UNSUPPORTED: return "unsupported size or head dimension";
        case MRA_ERR_CUDA: return "CUDA error";
        case MRA_ERR_ALLOC: return "workspace allocation failed";
        case MRA_ERR_DEVICE_TIMEOUT: return "bounded device wait gave up";
        case MRA_ERR_TOO_LARGE:
            return "problem needs more scratch than the no-allocation entry point's static array";
        default: return "unknown status";
    }
}

int mra_get_device_status(cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    if (current_device(&dev) != MRA_OK) return -MRA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -MRA_ERR_CUDA;
    DeviceCtx &ctx = g_dev[dev];
    if (!ctx.status) return 0;
    unsigned int word = 0;
    if (cudaMemcpy(&word, ctx.status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return -MRA_ERR_CUDA;
    if (cudaMemset(ctx.status, 0, sizeof(word)) != cudaSuccess) return -MRA_ERR_CUDA;
    return (int)word;
}

int mra_status_from_device(int word) {
    if (word < 0) return -word;
    if (word & MRA_DEV_TIMEOUT) return MRA_ERR_DEVICE_TIMEOUT;
    if (word & MRA_DEV_COUNT) return MRA_ERR_INVALID_ARG;
    return MRA_OK;
}

void mra_profile_enable(int enable) {
    std::lock_guard<std::mutex> lock(g_mutex);
    g_prof = enable != 0;
}

int mra_profile_read(const char **names, int *launches, double *total_ms, int max) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_pending.empty()) cudaEventSynchronize(g_pending.back().stop);
    for (const PendingEvent &pe : g_pending) {
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, pe.start, pe.stop) == cudaSuccess) {
            g_phase[pe.phase].ms += ms;
            g_phase[pe.phase].launches += 1;
        }
        g_event_pool.push_back(pe.start);
        g_event_pool.push_back(pe.stop);
    }
    g_pending.clear();
    int n = 0;
    for (PhaseStat &st : g_phase) {
        if (n >= max) break;
        if (names) names[n] = st.name;
        if (launches) launches[n] = st.launches;
        if (total_ms) total_ms[n] = st.ms;
        st.launches = 0;
        st.ms = 0.0;
        ++n;
    }
    return n;
}

int mra_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
