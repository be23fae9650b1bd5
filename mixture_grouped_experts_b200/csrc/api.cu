// C ABI of the MoGE layer (declared in include/moge.h): argument checks,
// workspace carve-up and the launch sequences. No entry point allocates
// device memory; all of them only enqueue work on the caller's stream.
#include <mutex>
#include <string.h>

#include <string>

#include "common.cuh"
#include "moge_internal.h"

namespace moge {

static thread_local std::string g_last_error;

static int fail(int code, const std::string &msg) {
    g_last_error = msg;
    return code;
}
static int cuda_fail(cudaError_t e, const char *where) {
    return fail(MOGE_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// router: the config's router runs (the bf16 router needs N % 8 == 0); the
// expert-parallel sub-problems route nothing themselves
static int check_config(const moge_config *c, bool router = true) {
    if (!c) return fail(MOGE_ERR_INVALID_ARG, "config is NULL");
    if (c->T < 0 || c->d <= 0 || c->N <= 0 || c->M <= 0 || c->Kp <= 0 || c->S < 0 || c->I <= 0)
        return fail(MOGE_ERR_INVALID_ARG, "config has a non-positive size");
    if (c->dtype != MOGE_F32 && c->dtype != MOGE_BF16)
        return fail(MOGE_ERR_INVALID_ARG, "dtype must be MOGE_F32 or MOGE_BF16");
    if (c->N > kMaxExperts) return fail(MOGE_ERR_UNSUPPORTED, "N > 256");
    if (c->S > kMaxExperts) return fail(MOGE_ERR_UNSUPPORTED, "S > 256");
    if (c->N % c->M != 0) return fail(MOGE_ERR_UNSUPPORTED, "N is not a multiple of M");
    if (c->Kp > c->N / c->M) return fail(MOGE_ERR_UNSUPPORTED, "Kp > N/M");
    if (c->d % 8 != 0 || c->I % 8 != 0)
        return fail(MOGE_ERR_UNSUPPORTED, "d and I must be multiples of 8");
    if (router && c->dtype == MOGE_BF16 && c->N % 8 != 0)
        return fail(MOGE_ERR_UNSUPPORTED, "bf16 router needs N % 8 == 0");
    const long long rows = (long long)c->T * (c->M * c->Kp + c->S);
    if (rows >= (1ll << 31) || (long long)c->T * c->M * c->Kp * (long long)c->d >= (1ll << 62))
        return fail(MOGE_ERR_UNSUPPORTED, "T*(K+S) rows exceed int32");
    return MOGE_OK;
}

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

Workspace carve_workspace(const moge_config &c, void *base) {
    Workspace w;
    const size_t K = (size_t)c.M * c.Kp, T = (size_t)c.T, N = (size_t)c.N;
    const size_t tiles = (T + kRouterTile - 1) / kRouterTile;
    const size_t E = N + (size_t)c.S;
    const size_t esz = c.dtype == MOGE_BF16 ? 2 : 4;
    char *p = static_cast<char *>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *r = p ? p + off : nullptr;
        off += align256(bytes > 0 ? bytes : 1);
        return r;
    };
    w.hist = (int32_t *)take(tiles * N * 4);
    w.base = (int32_t *)take(tiles * N * 4);
    w.rank = (int32_t *)take(T * K * 4);
    w.topk_idx = (int32_t *)take(T * K * 4);
    w.topk_w = (float *)take(T * K * 4);
    w.counts = (int32_t *)take(N * 4);
    w.offsets = (int32_t *)take((N + 1) * 4);
    w.perm_src = (int32_t *)take(T * K * 4);
    w.perm_dst = (int32_t *)take(T * K * 4);
    w.plan.up = (ExpertWork *)take(E * sizeof(ExpertWork));
    w.plan.down = (ExpertWork *)take(E * sizeof(ExpertWork));
    w.plan.up_start = (int *)take((E + 1) * 4);
    w.plan.down_start = (int *)take((E + 1) * 4);
    w.plan.sync = (int *)take((E + 2) * 4);
    w.x_perm = take(T * K * c.d * esz);
    w.h = take(T * (K + c.S) * c.I * esz);
    w.y_perm = take(T * (K + c.S) * c.d * esz);
    w.total = off;
    return w;
}

static int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

#define MOGE_NEED(p, what)                                                       \
    do {                                                                         \
        if (!(p)) return fail(MOGE_ERR_INVALID_ARG, std::string(what) + " is NULL"); \
        if (!aligned16(p))                                                       \
            return fail(MOGE_ERR_UNSUPPORTED, std::string(what) + " is not 16-byte aligned"); \
    } while (0)
#define MOGE_NEED4(p, what)                                                      \
    do {                                                                         \
        if (!(p)) return fail(MOGE_ERR_INVALID_ARG, std::string(what) + " is NULL"); \
        if (!aligned4(p))                                                        \
            return fail(MOGE_ERR_UNSUPPORTED, std::string(what) + " is not 4-byte aligned"); \
    } while (0)
#define MOGE_CU(expr, where)                       \
    do {                                           \
        cudaError_t e_ = (expr);                   \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
    } while (0)

// ---------------------------------------------------------------- stage timing
// Optional CUDA-event timing of the five launches of moge_layer_forward
// (router, scan, permute, grouped FFN, combine). Host state for one host
// thread and one device; not for use under stream capture.
constexpr int kTimedStages = 5;
constexpr int kEventSets = 32;
struct StageTimer {
    bool enabled = false;
    cudaEvent_t ev[kEventSets][kTimedStages + 1] = {};
    bool pending[kEventSets] = {};
    int next = 0;
    double total_ms[kTimedStages] = {};
    long long calls = 0;
};
static StageTimer g_timer;

static cudaError_t timer_harvest(int i) {
    if (!g_timer.pending[i]) return cudaSuccess;
    cudaError_t e = cudaEventSynchronize(g_timer.ev[i][kTimedStages]);
    if (e != cudaSuccess) return e;
    for (int s = 0; s < kTimedStages; ++s) {
        float ms = 0.0f;
        e = cudaEventElapsedTime(&ms, g_timer.ev[i][s], g_timer.ev[i][s + 1]);
        if (e != cudaSuccess) return e;
        g_timer.total_ms[s] += ms;
    }
    g_timer.pending[i] = false;
    g_timer.calls += 1;
    return cudaSuccess;
}

// Event set for the next layer call, or nullptr when timing is off.
static cudaEvent_t *timer_slot() {
    if (!g_timer.enabled) return nullptr;
    const int i = g_timer.next;
    g_timer.next = (i + 1) % kEventSets;
    if (timer_harvest(i) != cudaSuccess) return nullptr;
    for (int s = 0; s <= kTimedStages; ++s)
        if (!g_timer.ev[i][s] && cudaEventCreate(&g_timer.ev[i][s]) != cudaSuccess) return nullptr;
    g_timer.pending[i] = true;
    return g_timer.ev[i];
}

}  // namespace moge

using namespace moge;

static int run_ffn(const moge_config &c, const Plan &plan, int n_entries, const FfnOperands &op,
                   cudaStream_t st, cudaEvent_t mid = nullptr) {
    if (c.dtype == MOGE_BF16)
        MOGE_CU(launch_ffn_tc(c, plan, n_entries, op, num_sms(), st, mid),
                "grouped FFN (tcgen05) launch");
    else
        MOGE_CU(launch_ffn_f32(c, plan, n_entries, op, st, mid), "grouped FFN (fp32) launch");
    return MOGE_OK;
}

// The five launches of the layer (router, scan + plan, permute, grouped FFN,
// combine) after the entry point validated its arguments. `op` carries the
// expert weight pointers (and, for fp8, their row scales); the activation
// pointers are filled in here.
// Largest T*K whose permute runs inside the grouped GEMM launch (measured:
// saves ~6 us at T = 456, costs ~30 us at T = 4096).
constexpr long long kFusedPermuteRows = 8192;
// Smallest T*K whose grouped FFN runs on CTA pairs (2-SM MMA): each CTA of a
// pair stages half of the token rows, a third fewer shared-memory bytes per
// MMA flop, and shared-memory bandwidth and the copies' latency are what bound
// the 1-SM kernel on large token tiles. Every batch too large for the permute
// inside the launch takes the pair (measured faster from T*K = 8800 on: 0.78
// vs 0.83 ms at T = 1100 of the prefill layer); decode-sized ones keep the
// 1-SM kernel and its fused permute.
constexpr long long kPairRows = kFusedPermuteRows + 1;

// W8A8 workspace: the forward workspace (its x_perm region holds the routed
// rows' codes, its h region the h codes), then the tokens' codes, the two
// activation scale arrays, h in fp32 and its row amax words and scales.
struct W8Space {
    Workspace fw;
    void *x8;        // [T][d] E4M3 codes
    float *sx;       // [T]
    float *sxp;      // [T*K]
    float *h32;      // [T(K+S)][I]
    uint32_t *hmax;  // [T(K+S)]
    float *sh;       // [T(K+S)]
    size_t total;
};
static W8Space carve_w8a8(const moge_config &c, void *base) {
    W8Space s;
    s.fw = carve_workspace(c, base);
    const size_t K = (size_t)c.M * c.Kp, T = (size_t)c.T, hrows = T * (K + c.S);
    char *p = static_cast<char *>(base);
    size_t off = s.fw.total;
    auto take = [&](size_t bytes) {
        char *r = p ? p + off : nullptr;
        off += align256(bytes > 0 ? bytes : 1);
        return r;
    };
    s.x8 = take(T * c.d);
    s.sx = (float *)take(T * 4);
    s.sxp = (float *)take(T * K * 4);
    s.h32 = (float *)take(hrows * c.I * 4);
    s.hmax = (uint32_t *)take(hrows * 4);
    s.sh = (float *)take(hrows * 4);
    s.total = off;
    return s;
}

// The layer's expert arithmetic: bf16 (or fp32), 8-bit weights, or W8A8.
enum LayerMode { kModeDense = 0, kModeFp8Weights = 1, kModeW8A8 = 2 };

static int layer_run(const moge_config &c, const void *x, const void *w_router,
                     const float *logit_bias, FfnOperands op, LayerMode mode, const void *residual,
                     void *y, void *workspace, cudaStream_t st) {
    const bool fp8 = mode == kModeFp8Weights, w8a8 = mode == kModeW8A8;
    Workspace ws = carve_workspace(c, workspace);
    const int K = c.M * c.Kp;
    cudaEvent_t *ev = timer_slot();
    if (ev) MOGE_CU(cudaEventRecord(ev[0], st), "event");
    MOGE_CU(launch_router(c, x, w_router, logit_bias, ws.topk_idx, ws.topk_w, ws.hist, ws.rank,
                          num_sms(), st), "router launch");
    if (ev) MOGE_CU(cudaEventRecord(ev[1], st), "event");
    MOGE_CU(launch_scan(c, ws.hist, ws.base, ws.counts, ws.offsets, &ws.plan, true, c.S > 0, st),
            "scan launch");
    if (ev) MOGE_CU(cudaEventRecord(ev[2], st), "event");
    // bf16 decode-sized batches: the grouped GEMM launch does the permute itself
    // (its epilogue warps copy the rows while the first, shared-expert items
    // run); larger batches (the copy would hold the epilogue warps long enough to
    // stall the first items), fp8 and fp32: a launch of its own
    const bool fuse_permute = c.dtype == MOGE_BF16 && mode == kModeDense &&
                              (long long)c.T * c.M * c.Kp <= kFusedPermuteRows;
    op.b1 = x;
    if (w8a8) {  // the tokens quantised, their codes permuted
        W8Space w8 = carve_w8a8(c, workspace);
        MOGE_CU(launch_quantize_scatter(c, x, ws.topk_idx, ws.rank, ws.base, ws.offsets,
                                        ws.perm_src, ws.perm_dst, w8.x8, w8.sx, ws.x_perm, w8.sxp,
                                        w8.hmax, st), "quantise + permute launch");
        op.b1 = w8.x8;
        op.cs_b0 = w8.sxp;
        op.cs_b1 = w8.sx;
        op.h32 = w8.h32;
        op.hmax = w8.hmax;
        op.sh = w8.sh;
    } else if (fuse_permute) {
        op.pm_topk_idx = ws.topk_idx; op.pm_rank = ws.rank; op.pm_base = ws.base;
        op.pm_offsets = ws.offsets; op.pm_perm_src = ws.perm_src; op.pm_perm_dst = ws.perm_dst;
    } else {
        MOGE_CU(launch_scatter_rows(c, x, ws.topk_idx, ws.rank, ws.base, ws.offsets, ws.perm_src,
                                    ws.perm_dst, ws.x_perm, st), "permute launch");
    }
    if (ev) MOGE_CU(cudaEventRecord(ev[3], st), "event");
    const int64_t rrows = (int64_t)c.T * K;
    op.b0 = ws.x_perm;
    op.b0_rows = rrows;
    op.b1_rows = c.T;
    op.h = ws.h;
    op.h_rows = rrows + (int64_t)c.T * c.S;
    op.y = ws.y_perm;
    if (fp8) {
        MOGE_CU(launch_ffn_fp8(c, ws.plan, c.N + c.S, op, num_sms(), st), "grouped FFN (fp8) launch");
    } else if (w8a8) {
        MOGE_CU(launch_ffn_w8a8(c, ws.plan, c.N + c.S, op, num_sms(), st),
                "grouped FFN (W8A8) launch");
    } else {
        if (c.dtype == MOGE_BF16 && !fuse_permute && rrows >= kPairRows) {
            MOGE_CU(pair::launch_ffn_tc_pair(c, ws.plan, c.N + c.S, op, num_sms(), st),
                    "grouped FFN (tcgen05 pairs) launch");
        } else {
            int rc = run_ffn(c, ws.plan, c.N + c.S, op, st, nullptr);
            if (rc) return rc;
        }
    }
    if (ev) MOGE_CU(cudaEventRecord(ev[4], st), "event");
    const size_t esz = c.dtype == MOGE_BF16 ? 2 : 4;
    const void *shared_rows = static_cast<const char *>(ws.y_perm) + (size_t)rrows * c.d * esz;
    MOGE_CU(launch_combine(c, ws.y_perm, ws.topk_w, ws.perm_dst, K, shared_rows, c.S, residual, y,
                           st), "combine launch");
    if (ev) MOGE_CU(cudaEventRecord(ev[5], st), "event");
    return MOGE_OK;
}


// Training workspace: the forward workspace, then what the backward pass needs
// beyond it. dgu overwrites gu in place (the SwiGLU backward reads g, u and
// writes dg, du at the same positions, each element by one thread) and dx_perm
// overwrites y_perm (read only by the combine backward, which runs first).
struct TrainSpace {
    Workspace fw;
    void *gu;        // [hrows][2I]
    void *dy_perm;   // [rrows][d]
    float *logits;   // [kMaxLogitSplit][T][N]: partial logits, one per K part
    void *dl;        // [T][N]
    float *dx_r;     // [T][d]
    float *dw;       // [T][K]
    float *part;     // [router_bwd_parts][N]
    size_t total;
};
static TrainSpace carve_train(const moge_config &c, void *base) {
    TrainSpace s;
    s.fw = carve_workspace(c, base);
    const size_t K = (size_t)c.M * c.Kp, T = (size_t)c.T;
    char *p = static_cast<char *>(base);
    size_t off = s.fw.total;
    auto take = [&](size_t bytes) {
        char *r = p ? p + off : nullptr;
        off += align256(bytes > 0 ? bytes : 1);
        return r;
    };
    s.gu = take(T * (K + c.S) * 2 * (size_t)c.I * 2);
    s.dy_perm = take(T * K * c.d * 2);
    s.logits = (float *)take((size_t)kMaxLogitSplit * T * c.N * 4);  // one [T][N] per K part
    s.dl = take(T * c.N * 2);
    s.dx_r = (float *)take(T * c.d * 4);
    s.dw = (float *)take(T * K * 4);
    s.part = (float *)take((size_t)router_bwd_parts(c) * c.N * 4);
    s.total = off;
    return s;
}

static int check_train(const moge_config &c) {
    if (c.dtype != MOGE_BF16) return fail(MOGE_ERR_UNSUPPORTED, "training needs dtype MOGE_BF16");
    if (c.I % 64 != 0) return fail(MOGE_ERR_UNSUPPORTED, "training needs I % 64 == 0");
    if (c.N % 8 != 0) return fail(MOGE_ERR_UNSUPPORTED, "training needs N % 8 == 0");
    if (c.M * c.Kp > 32) return fail(MOGE_ERR_UNSUPPORTED, "training needs M * Kp <= 32");
    return MOGE_OK;
}


// Expert parallelism: rank `rank` of `world` holds the experts of groups
// [rank M/world, (rank+1) M/world) and an I/world slice of every shared
// expert. loc: the routed sub-problem (those experts and groups, all T
// tokens, no shared experts); shr: the shared slice (S experts of I/world,
// no routed experts).
static int ep_configs(const moge_config &c, int rank, int world, moge_config &loc,
                      moge_config &shr) {
    if (world < 1 || rank < 0 || rank >= world)
        return fail(MOGE_ERR_INVALID_ARG, "need 0 <= rank < world");
    if (c.M % world != 0) return fail(MOGE_ERR_UNSUPPORTED, "expert parallelism needs M % world == 0");
    if (c.I % world != 0) return fail(MOGE_ERR_UNSUPPORTED, "expert parallelism needs I % world == 0");
    loc = c;
    loc.N = c.N / world;
    loc.M = c.M / world;
    loc.S = 0;
    shr = c;
    shr.N = 1;
    shr.M = 1;
    shr.Kp = 1;
    shr.I = c.I / world;
    int rc = check_config(&loc, false);
    if (!rc) rc = check_config(&shr, false);
    return rc;
}

struct EpSpace {
    int32_t *hist, *rank, *topk_idx;  // routing of all T tokens over all N experts
    float *topk_w;
    Workspace lw, sw;                 // the routed and the shared sub-problems
    size_t total;
};
static EpSpace carve_ep(const moge_config &c, const moge_config &loc, const moge_config &shr,
                        void *base) {
    EpSpace e;
    const size_t K = (size_t)c.M * c.Kp, T = (size_t)c.T;
    const size_t tiles = (T + kRouterTile - 1) / kRouterTile;
    char *p = static_cast<char *>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *r = p ? p + off : nullptr;
        off += align256(bytes > 0 ? bytes : 1);
        return r;
    };
    e.hist = (int32_t *)take(tiles * c.N * 4);
    e.rank = (int32_t *)take(T * K * 4);
    e.topk_idx = (int32_t *)take(T * K * 4);
    e.topk_w = (float *)take(T * K * 4);
    e.lw = carve_workspace(loc, p ? p + off : nullptr);
    off += e.lw.total;
    e.sw = carve_workspace(shr, p ? p + off : nullptr);
    off += e.sw.total;
    e.total = off;
    return e;
}


// Streams and events of the pipelined host-buffer call, created once per
// device: a host-to-device and a device-to-host copy stream, and per device
// buffer (two) "copied in", "computed" and "copied out" events.
struct HostPipe {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t copied_in[2] = {}, computed[2] = {}, copied_out[2] = {};
    bool ready = false;
};
static int host_pipe(HostPipe *&hp) {
    static HostPipe pipes[64];
    static std::mutex mu;
    int dev = 0;
    MOGE_CU(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(MOGE_ERR_UNSUPPORTED, "device index >= 64");
    std::lock_guard<std::mutex> lock(mu);
    HostPipe &p = pipes[dev];
    if (!p.ready) {
        MOGE_CU(cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking), "copy stream");
        MOGE_CU(cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking), "copy stream");
        for (int b = 0; b < 2; ++b) {
            MOGE_CU(cudaEventCreateWithFlags(&p.copied_in[b], cudaEventDisableTiming), "event");
            MOGE_CU(cudaEventCreateWithFlags(&p.computed[b], cudaEventDisableTiming), "event");
            MOGE_CU(cudaEventCreateWithFlags(&p.copied_out[b], cudaEventDisableTiming), "event");
        }
        p.ready = true;
    }
    hp = &p;
    return MOGE_OK;
}

extern "C" {

size_t moge_workspace_size(const moge_config *cfg) {
    if (check_config(cfg) != MOGE_OK) return 0;
    return carve_workspace(*cfg, nullptr).total;
}

const char *moge_last_error(void) { return g_last_error.c_str(); }

int moge_check_device_errors(void *stream) {
    MOGE_CU(cudaStreamSynchronize((cudaStream_t)stream), "cudaStreamSynchronize");
    uint32_t w = 0, zero = 0;
    MOGE_CU(cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)), "read device error word");
    MOGE_CU(cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)), "clear device error word");
    if (w & ERRBIT_TIMEOUT) return fail(MOGE_ERR_TIMEOUT, "a device-side wait timed out");
    if (w & ERRBIT_INVARIANT) return fail(MOGE_ERR_DEVICE, "a kernel found a violated invariant");
    return MOGE_OK;
}

int moge_route(const moge_config *cfg, const void *x, const void *w_router,
               const float *logit_bias, int32_t *topk_idx, float *topk_w, int32_t *counts,
               int32_t *offsets, int32_t *perm_src, int32_t *perm_dst, void *workspace,
               void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    cudaStream_t st = (cudaStream_t)stream;
    MOGE_NEED4(counts, "counts");
    MOGE_NEED4(offsets, "offsets");
    if (c.T == 0) {
        MOGE_CU(cudaMemsetAsync(counts, 0, sizeof(int32_t) * c.N, st), "memset counts");
        MOGE_CU(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (c.N + 1), st), "memset offsets");
        return MOGE_OK;
    }
    MOGE_NEED(x, "x");
    MOGE_NEED(w_router, "w_router");
    if (logit_bias && !aligned4(logit_bias)) return fail(MOGE_ERR_UNSUPPORTED, "logit_bias misaligned");
    MOGE_NEED4(topk_idx, "topk_idx");
    MOGE_NEED4(topk_w, "topk_w");
    MOGE_NEED4(perm_src, "perm_src");
    MOGE_NEED4(perm_dst, "perm_dst");
    MOGE_NEED(workspace, "workspace");
    Workspace ws = carve_workspace(c, workspace);
    MOGE_CU(launch_router(c, x, w_router, logit_bias, topk_idx, topk_w, ws.hist, ws.rank, num_sms(),
                          st), "router launch");
    MOGE_CU(launch_scan(c, ws.hist, ws.base, counts, offsets, nullptr, false, false, st),
            "scan launch");
    MOGE_CU(launch_finalize(c, topk_idx, ws.rank, ws.base, offsets, perm_src, perm_dst, st),
            "finalize launch");
    return MOGE_OK;
}

int moge_permute(const moge_config *cfg, const void *x, const int32_t *perm_src, void *x_perm,
                 void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOGE_OK;
    MOGE_NEED(x, "x");
    MOGE_NEED4(perm_src, "perm_src");
    MOGE_NEED(x_perm, "x_perm");
    MOGE_CU(launch_gather_rows(*cfg, x, perm_src, x_perm, (cudaStream_t)stream), "permute launch");
    return MOGE_OK;
}


int moge_grouped_ffn(const moge_config *cfg, const void *x_perm, const int32_t *offsets,
                     const void *w_gate, const void *w_up, const void *w_down, void *y_perm,
                     void *workspace, void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    if (c.T == 0) return MOGE_OK;
    MOGE_NEED(x_perm, "x_perm");
    MOGE_NEED4(offsets, "offsets");
    MOGE_NEED(w_gate, "w_gate");
    MOGE_NEED(w_up, "w_up");
    MOGE_NEED(w_down, "w_down");
    MOGE_NEED(y_perm, "y_perm");
    MOGE_NEED(workspace, "workspace");
    cudaStream_t st = (cudaStream_t)stream;
    Workspace ws = carve_workspace(c, workspace);
    MOGE_CU(launch_plan(c, offsets, ws.plan, true, false, st), "plan launch");
    const int64_t rows = (int64_t)c.T * c.M * c.Kp;
    FfnOperands op{x_perm, nullptr, rows, 0, w_gate, w_up, w_down, nullptr, nullptr, nullptr,
                   ws.h, rows, y_perm};
    if (c.dtype == MOGE_BF16 && rows >= kPairRows) {  // prefill-sized: CTA pairs, as the layer does
        MOGE_CU(pair::launch_ffn_tc_pair(c, ws.plan, c.N, op, num_sms(), st),
                "grouped FFN (tcgen05 pairs) launch");
        return MOGE_OK;
    }
    return run_ffn(c, ws.plan, c.N, op, st);
}

int moge_shared_ffn(const moge_config *cfg, const void *x, const void *s_gate, const void *s_up,
                    const void *s_down, void *y_shared, void *workspace, void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    if (c.T == 0) return MOGE_OK;
    cudaStream_t st = (cudaStream_t)stream;
    MOGE_NEED(y_shared, "y_shared");
    const size_t esz = c.dtype == MOGE_BF16 ? 2 : 4;
    if (c.S == 0) {
        MOGE_CU(cudaMemsetAsync(y_shared, 0, (size_t)c.T * c.d * esz, st), "memset y_shared");
        return MOGE_OK;
    }
    MOGE_NEED(x, "x");
    MOGE_NEED(s_gate, "s_gate");
    MOGE_NEED(s_up, "s_up");
    MOGE_NEED(s_down, "s_down");
    MOGE_NEED(workspace, "workspace");
    Workspace ws = carve_workspace(c, workspace);
    MOGE_CU(launch_plan(c, nullptr, ws.plan, false, true, st), "plan launch");
    const int64_t rows = (int64_t)c.T * c.S;
    FfnOperands op{nullptr, x, 0, c.T, nullptr, nullptr, nullptr, s_gate, s_up, s_down,
                   ws.h, rows, ws.y_perm};
    if (c.dtype == MOGE_BF16 && rows >= kPairRows) {  // prefill-sized: CTA pairs, as the layer does
        MOGE_CU(pair::launch_ffn_tc_pair(c, ws.plan, c.S, op, num_sms(), st),
                "grouped FFN (tcgen05 pairs) launch");
    } else {
        rc = run_ffn(c, ws.plan, c.S, op, st);
        if (rc) return rc;
    }
    MOGE_CU(launch_combine(c, nullptr, nullptr, nullptr, 0, ws.y_perm, c.S, nullptr, y_shared, st),
            "shared sum launch");
    return MOGE_OK;
}

int moge_combine(const moge_config *cfg, const void *y_perm, const float *topk_w,
                 const int32_t *perm_dst, const void *y_shared, const void *residual, void *y,
                 void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    if (c.T == 0) return MOGE_OK;
    MOGE_NEED(y_perm, "y_perm");
    MOGE_NEED4(topk_w, "topk_w");
    MOGE_NEED4(perm_dst, "perm_dst");
    MOGE_NEED(y, "y");
    if (y_shared && !aligned16(y_shared)) return fail(MOGE_ERR_UNSUPPORTED, "y_shared misaligned");
    if (residual && !aligned16(residual)) return fail(MOGE_ERR_UNSUPPORTED, "residual misaligned");
    MOGE_CU(launch_combine(c, y_perm, topk_w, perm_dst, c.M * c.Kp, y_shared, y_shared ? 1 : 0,
                           residual, y, (cudaStream_t)stream),
            "combine launch");
    return MOGE_OK;
}

int moge_layer_forward(const moge_config *cfg, const void *x, const void *w_router,
                       const float *logit_bias, const void *w_gate, const void *w_up,
                       const void *w_down, const void *s_gate, const void *s_up,
                       const void *s_down, const void *residual, void *y, void *workspace,
                       void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    if (c.T == 0) return MOGE_OK;
    MOGE_NEED(x, "x");
    MOGE_NEED(w_router, "w_router");
    MOGE_NEED(w_gate, "w_gate");
    MOGE_NEED(w_up, "w_up");
    MOGE_NEED(w_down, "w_down");
    if (c.S > 0) {
        MOGE_NEED(s_gate, "s_gate");
        MOGE_NEED(s_up, "s_up");
        MOGE_NEED(s_down, "s_down");
    }
    if (logit_bias && !aligned4(logit_bias)) return fail(MOGE_ERR_UNSUPPORTED, "logit_bias misaligned");
    if (residual && !aligned16(residual)) return fail(MOGE_ERR_UNSUPPORTED, "residual misaligned");
    MOGE_NEED(y, "y");
    MOGE_NEED(workspace, "workspace");
    if (y == x) return fail(MOGE_ERR_INVALID_ARG, "y must not alias x");
    FfnOperands wts{};
    wts.wg = w_gate; wts.wu = w_up; wts.wd = w_down;
    if (c.S > 0) { wts.sg = s_gate; wts.su = s_up; wts.sd = s_down; }
    return layer_run(c, x, w_router, logit_bias, wts, kModeDense, residual, y, workspace,
                     (cudaStream_t)stream);
}

int moge_layer_forward_host(const moge_config *cfg, const void *x_host, const void *w_router,
                            const float *logit_bias, const void *w_gate, const void *w_up,
                            const void *w_down, const void *s_gate, const void *s_up,
                            const void *s_down, void *y_host, void *x_dev, void *y_dev,
                            void *workspace, void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    if (c.T == 0) return MOGE_OK;
    if (!x_host || !y_host) return fail(MOGE_ERR_INVALID_ARG, "host buffer is NULL");
    MOGE_NEED(x_dev, "x_dev");
    MOGE_NEED(y_dev, "y_dev");
    cudaStream_t st = (cudaStream_t)stream;
    const size_t bytes = (size_t)c.T * c.d * (c.dtype == MOGE_BF16 ? 2 : 4);
    MOGE_CU(cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, st), "copy x in");
    rc = moge_layer_forward(cfg, x_dev, w_router, logit_bias, w_gate, w_up, w_down, s_gate, s_up,
                            s_down, nullptr, y_dev, workspace, stream);
    if (rc) return rc;
    MOGE_CU(cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, st), "copy y out");
    MOGE_CU(cudaStreamSynchronize(st), "cudaStreamSynchronize");
    return MOGE_OK;
}

int moge_layer_forward_host_stream(const moge_config *cfg, int64_t n_batches, const void *x_host,
                                   const void *w_router, const float *logit_bias,
                                   const void *w_gate, const void *w_up, const void *w_down,
                                   const void *s_gate, const void *s_up, const void *s_down,
                                   void *y_host, void *x_dev2, void *y_dev2, void *workspace,
                                   void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    if (n_batches < 0) return fail(MOGE_ERR_INVALID_ARG, "n_batches < 0");
    if (c.T == 0 || n_batches == 0) return MOGE_OK;
    if (!x_host || !y_host) return fail(MOGE_ERR_INVALID_ARG, "host buffer is NULL");
    MOGE_NEED(x_dev2, "x_dev2");
    MOGE_NEED(y_dev2, "y_dev2");
    HostPipe *hp = nullptr;
    if ((rc = host_pipe(hp))) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t bytes = (size_t)c.T * c.d * (c.dtype == MOGE_BF16 ? 2 : 4);
    const char *xh = static_cast<const char *>(x_host);
    char *yh = static_cast<char *>(y_host);
    char *xd = static_cast<char *>(x_dev2), *yd = static_cast<char *>(y_dev2);
    // everything queued on `stream` before this call comes first
    MOGE_CU(cudaEventRecord(hp->computed[1], st), "event");
    MOGE_CU(cudaStreamWaitEvent(hp->in, hp->computed[1], 0), "wait");
    MOGE_CU(cudaStreamWaitEvent(hp->out, hp->computed[1], 0), "wait");
    for (int64_t i = 0; i < n_batches; ++i) {
        const int b = (int)(i & 1);
        // x buffer b: its previous batch (i - 2) has been read by its compute
        if (i >= 2) MOGE_CU(cudaStreamWaitEvent(hp->in, hp->computed[b], 0), "wait");
        MOGE_CU(cudaMemcpyAsync(xd + b * bytes, xh + i * bytes, bytes, cudaMemcpyHostToDevice,
                                hp->in), "copy x in");
        MOGE_CU(cudaEventRecord(hp->copied_in[b], hp->in), "event");
        // y buffer b: its previous batch has been copied out
        MOGE_CU(cudaStreamWaitEvent(st, hp->copied_in[b], 0), "wait");
        if (i >= 2) MOGE_CU(cudaStreamWaitEvent(st, hp->copied_out[b], 0), "wait");
        rc = moge_layer_forward(cfg, xd + b * bytes, w_router, logit_bias, w_gate, w_up, w_down,
                                s_gate, s_up, s_down, nullptr, yd + b * bytes, workspace, stream);
        if (rc) return rc;
        MOGE_CU(cudaEventRecord(hp->computed[b], st), "event");
        MOGE_CU(cudaStreamWaitEvent(hp->out, hp->computed[b], 0), "wait");
        MOGE_CU(cudaMemcpyAsync(yh + i * bytes, yd + b * bytes, bytes, cudaMemcpyDeviceToHost,
                                hp->out), "copy y out");
        MOGE_CU(cudaEventRecord(hp->copied_out[b], hp->out), "event");
    }
    MOGE_CU(cudaStreamSynchronize(hp->out), "cudaStreamSynchronize");
    MOGE_CU(cudaStreamSynchronize(hp->in), "cudaStreamSynchronize");
    MOGE_CU(cudaStreamSynchronize(st), "cudaStreamSynchronize");
    return MOGE_OK;
}

int moge_workspace_routing(const moge_config *cfg, void *workspace, int32_t **topk_idx,
                           float **topk_w, int32_t **counts, int32_t **offsets) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!workspace) return fail(MOGE_ERR_INVALID_ARG, "workspace is NULL");
    Workspace ws = carve_workspace(*cfg, workspace);
    if (topk_idx) *topk_idx = ws.topk_idx;
    if (topk_w) *topk_w = ws.topk_w;
    if (counts) *counts = ws.counts;
    if (offsets) *offsets = ws.offsets;
    return MOGE_OK;
}

int moge_rmsnorm(const moge_config *cfg, const void *x, float eps, void *u, void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (cfg->T == 0) return MOGE_OK;
    MOGE_NEED(x, "x");
    MOGE_NEED(u, "u");
    if (!(eps >= 0.0f)) return fail(MOGE_ERR_INVALID_ARG, "eps must be >= 0");
    MOGE_CU(launch_rmsnorm(*cfg, x, eps, u, (cudaStream_t)stream), "rmsnorm launch");
    return MOGE_OK;
}

int moge_selftest_waits(int64_t limit_us, int32_t *out, void *stream) {
    if (limit_us < 1 || limit_us > 2000000)
        return fail(MOGE_ERR_INVALID_ARG, "limit_us must be in 1 .. 2000000");
    MOGE_NEED4(out, "out");
    MOGE_CU(launch_wait_selftest(out, (uint64_t)limit_us * 1000u, (cudaStream_t)stream),
            "wait self-test launch");
    return MOGE_OK;
}

int moge_quantize_fp8_rows(const void *w, int64_t rows, int64_t cols, void *q, float *scale,
                           void *stream) {
    if (rows < 0 || cols <= 0) return fail(MOGE_ERR_INVALID_ARG, "rows must be >= 0, cols > 0");
    if (cols % 8 != 0) return fail(MOGE_ERR_UNSUPPORTED, "cols must be a multiple of 8");
    if (rows == 0) return MOGE_OK;
    MOGE_NEED(w, "w");
    if (!q) return fail(MOGE_ERR_INVALID_ARG, "q is NULL");
    if (reinterpret_cast<uintptr_t>(q) % 8 != 0)
        return fail(MOGE_ERR_UNSUPPORTED, "q is not 8-byte aligned");
    MOGE_NEED4(scale, "scale");
    MOGE_CU(launch_quantize_fp8(w, rows, cols, q, scale, (cudaStream_t)stream), "quantize launch");
    return MOGE_OK;
}

static int check_fp8_side(const moge_fp8_experts *e, const char *side) {
    if (!e) return fail(MOGE_ERR_INVALID_ARG, std::string(side) + " fp8 experts are NULL");
    MOGE_NEED(e->gate, std::string(side) + ".gate");
    MOGE_NEED(e->up, std::string(side) + ".up");
    MOGE_NEED(e->down, std::string(side) + ".down");
    MOGE_NEED4(e->gate_scale, std::string(side) + ".gate_scale");
    MOGE_NEED4(e->up_scale, std::string(side) + ".up_scale");
    MOGE_NEED4(e->down_scale, std::string(side) + ".down_scale");
    return MOGE_OK;
}

// The two 8-bit layers share their host checks and operands: E4M3 expert
// weights with one fp32 scale per row, bf16 x and y.
static int forward_8bit(const moge_config *cfg, const void *x, const void *w_router,
                        const float *logit_bias, const moge_fp8_experts *routed,
                        const moge_fp8_experts *shared, const void *residual, void *y,
                        void *workspace, void *stream, LayerMode mode) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    const char *what = mode == kModeW8A8 ? "W8A8 needs" : "fp8 experts need";
    if (c.dtype != MOGE_BF16)
        return fail(MOGE_ERR_UNSUPPORTED, std::string(what) + " dtype MOGE_BF16");
    if (c.d % 16 != 0 || c.I % 16 != 0)
        return fail(MOGE_ERR_UNSUPPORTED, std::string(what) + " d % 16 == 0 and I % 16 == 0");
    if (c.T == 0) return MOGE_OK;
    MOGE_NEED(x, "x");
    MOGE_NEED(w_router, "w_router");
    if ((rc = check_fp8_side(routed, "routed"))) return rc;
    if (c.S > 0 && (rc = check_fp8_side(shared, "shared"))) return rc;
    if (logit_bias && !aligned4(logit_bias)) return fail(MOGE_ERR_UNSUPPORTED, "logit_bias misaligned");
    if (residual && !aligned16(residual)) return fail(MOGE_ERR_UNSUPPORTED, "residual misaligned");
    MOGE_NEED(y, "y");
    MOGE_NEED(workspace, "workspace");
    if (y == x) return fail(MOGE_ERR_INVALID_ARG, "y must not alias x");
    FfnOperands op{};
    op.wg = routed->gate; op.wu = routed->up; op.wd = routed->down;
    op.wg_s = routed->gate_scale; op.wu_s = routed->up_scale; op.wd_s = routed->down_scale;
    if (c.S > 0) {
        op.sg = shared->gate; op.su = shared->up; op.sd = shared->down;
        op.sg_s = shared->gate_scale; op.su_s = shared->up_scale; op.sd_s = shared->down_scale;
    }
    return layer_run(c, x, w_router, logit_bias, op, mode, residual, y, workspace,
                     (cudaStream_t)stream);
}

int moge_layer_forward_fp8(const moge_config *cfg, const void *x, const void *w_router,
                           const float *logit_bias, const moge_fp8_experts *routed,
                           const moge_fp8_experts *shared, const void *residual, void *y,
                           void *workspace, void *stream) {
    return forward_8bit(cfg, x, w_router, logit_bias, routed, shared, residual, y, workspace,
                        stream, kModeFp8Weights);
}

size_t moge_w8a8_workspace_size(const moge_config *cfg) {
    if (check_config(cfg) != MOGE_OK) return 0;
    return carve_w8a8(*cfg, nullptr).total;
}

int moge_layer_forward_w8a8(const moge_config *cfg, const void *x, const void *w_router,
                            const float *logit_bias, const moge_fp8_experts *routed,
                            const moge_fp8_experts *shared, const void *residual, void *y,
                            void *workspace, void *stream) {
    return forward_8bit(cfg, x, w_router, logit_bias, routed, shared, residual, y, workspace,
                        stream, kModeW8A8);
}

int moge_stage_timing(int enable) {
    if (enable) {
        for (int i = 0; i < kEventSets; ++i) g_timer.pending[i] = false;
        for (int k = 0; k < kTimedStages; ++k) g_timer.total_ms[k] = 0.0;
        g_timer.calls = 0;
        g_timer.next = 0;
    }
    g_timer.enabled = enable != 0;
    return MOGE_OK;
}

int moge_stage_times(double *ms_total, int64_t *calls) {
    for (int i = 0; i < kEventSets; ++i)
        MOGE_CU(timer_harvest(i), "stage timing events");
    if (ms_total)
        for (int k = 0; k < kTimedStages; ++k) ms_total[k] = g_timer.total_ms[k];
    if (calls) *calls = g_timer.calls;
    return MOGE_OK;
}


size_t moge_train_workspace_size(const moge_config *cfg) {
    if (check_config(cfg) != MOGE_OK || check_train(*cfg) != MOGE_OK) return 0;
    return carve_train(*cfg, nullptr).total;
}

int moge_layer_forward_train(const moge_config *cfg, const void *x, const void *w_router,
                             const float *logit_bias, const void *w_gate, const void *w_up,
                             const void *w_down, const void *s_gate, const void *s_up,
                             const void *s_down, void *y, void *workspace, void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    if ((rc = check_train(c))) return rc;
    if (c.T == 0) return MOGE_OK;
    MOGE_NEED(x, "x");
    MOGE_NEED(w_router, "w_router");
    MOGE_NEED(w_gate, "w_gate");
    MOGE_NEED(w_up, "w_up");
    MOGE_NEED(w_down, "w_down");
    if (c.S > 0) {
        MOGE_NEED(s_gate, "s_gate");
        MOGE_NEED(s_up, "s_up");
        MOGE_NEED(s_down, "s_down");
    }
    if (logit_bias && !aligned4(logit_bias)) return fail(MOGE_ERR_UNSUPPORTED, "logit_bias misaligned");
    MOGE_NEED(y, "y");
    MOGE_NEED(workspace, "workspace");
    if (y == x) return fail(MOGE_ERR_INVALID_ARG, "y must not alias x");
    TrainSpace ts = carve_train(c, workspace);
    FfnOperands wts{};
    wts.wg = w_gate; wts.wu = w_up; wts.wd = w_down;
    if (c.S > 0) { wts.sg = s_gate; wts.su = s_up; wts.sd = s_down; }
    wts.gu = ts.gu;
    return layer_run(c, x, w_router, logit_bias, wts, kModeDense, nullptr, y, workspace,
                     (cudaStream_t)stream);
}

int moge_layer_backward(const moge_config *cfg, float alpha, const void *x, const void *w_router,
                        const float *logit_bias, const void *w_gate, const void *w_up,
                        const void *w_down, const void *s_gate, const void *s_up,
                        const void *s_down, const void *dy, void *dx, void *dw_router,
                        void *dw_gate, void *dw_up, void *dw_down, void *ds_gate, void *ds_up,
                        void *ds_down, float *aux, void *workspace, void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    if ((rc = check_train(c))) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    MOGE_NEED(dw_router, "dw_router");
    MOGE_NEED(dw_gate, "dw_gate");
    MOGE_NEED(dw_up, "dw_up");
    MOGE_NEED(dw_down, "dw_down");
    if (c.S > 0) {
        MOGE_NEED(ds_gate, "ds_gate");
        MOGE_NEED(ds_up, "ds_up");
        MOGE_NEED(ds_down, "ds_down");
    }
    if (aux && !aligned4(aux)) return fail(MOGE_ERR_UNSUPPORTED, "aux misaligned");
    const size_t wsz = (size_t)c.I * c.d * 2;
    if (c.T == 0) {  // no tokens: every gradient is zero
        MOGE_CU(cudaMemsetAsync(dw_router, 0, (size_t)c.N * c.d * 2, st), "memset");
        MOGE_CU(cudaMemsetAsync(dw_gate, 0, c.N * wsz, st), "memset");
        MOGE_CU(cudaMemsetAsync(dw_up, 0, c.N * wsz, st), "memset");
        MOGE_CU(cudaMemsetAsync(dw_down, 0, c.N * wsz, st), "memset");
        if (c.S > 0) {
            MOGE_CU(cudaMemsetAsync(ds_gate, 0, c.S * wsz, st), "memset");
            MOGE_CU(cudaMemsetAsync(ds_up, 0, c.S * wsz, st), "memset");
            MOGE_CU(cudaMemsetAsync(ds_down, 0, c.S * wsz, st), "memset");
        }
        if (aux) MOGE_CU(cudaMemsetAsync(aux, 0, sizeof(float), st), "memset");
        return MOGE_OK;
    }
    MOGE_NEED(x, "x");
    MOGE_NEED(w_router, "w_router");
    MOGE_NEED(w_gate, "w_gate");
    MOGE_NEED(w_up, "w_up");
    MOGE_NEED(w_down, "w_down");
    if (c.S > 0) {
        MOGE_NEED(s_gate, "s_gate");
        MOGE_NEED(s_up, "s_up");
        MOGE_NEED(s_down, "s_down");
    }
    if (logit_bias && !aligned4(logit_bias)) return fail(MOGE_ERR_UNSUPPORTED, "logit_bias misaligned");
    MOGE_NEED(dy, "dy");
    MOGE_NEED(dx, "dx");
    MOGE_NEED(workspace, "workspace");
    if (dx == dy || dx == x) return fail(MOGE_ERR_INVALID_ARG, "dx must not alias x or dy");
    TrainSpace ts = carve_train(c, workspace);
    const Workspace &ws = ts.fw;
    const int E = c.N + c.S;
    BwdTensors b{};
    b.x = x; b.w_router = w_router; b.bias = logit_bias;
    b.wg = w_gate; b.wu = w_up; b.wd = w_down;
    if (c.S > 0) { b.sg = s_gate; b.su = s_up; b.sd = s_down; }
    b.x_perm = ws.x_perm; b.h = ws.h; b.gu = ts.gu;
    b.dy = dy; b.dy_perm = ts.dy_perm;
    b.dgu = ts.gu;          // in place
    b.dx_perm = ws.y_perm;  // y_perm is dead once the combine backward has run
    b.logits = ts.logits; b.dl = ts.dl; b.dx_r = ts.dx_r;
    b.dwg = dw_gate; b.dwu = dw_up; b.dwd = dw_down; b.dwr = dw_router;
    b.dsg = ds_gate; b.dsu = ds_up; b.dsd = ds_down;
    const int sms = num_sms();
    const ExpertWork *ent = ws.plan.up;
    MOGE_CU(launch_combine_bwd(c, dy, ws.y_perm, ws.topk_w, ws.perm_dst, ts.dy_perm, ts.dw, st),
            "combine backward launch");
    MOGE_CU(launch_bwd_gemm(kLOGITS, c, ent, E, b, sms, st), "logits launch");
    MOGE_CU(launch_router_bwd(c, alpha, ts.logits, logits_ksplit(c, sms), ws.topk_idx, ts.dw,
                              ws.counts, ts.dl, ts.part, aux, st), "router backward launch");
    MOGE_CU(launch_bwd_gemm(kDH, c, ent, E, b, sms, st), "dh launch");
    MOGE_CU(launch_bwd_gemm(kDX, c, ent, E, b, sms, st), "dx launch");
    MOGE_CU(launch_bwd_gemm(kDWD, c, ent, E, b, sms, st), "dW_down launch");
    MOGE_CU(launch_bwd_gemm(kDWGU, c, ent, E, b, sms, st), "dW_gate/up launch");
    MOGE_CU(launch_bwd_gemm(kDWR, c, ent, E, b, sms, st), "dW_router launch");
    MOGE_CU(launch_bwd_gemm(kDXR, c, ent, E, b, sms, st), "dx router launch");
    MOGE_CU(launch_unpermute_bwd(c, ws.y_perm, ws.perm_dst, ts.dx_r, dx, st), "un-permute launch");
    return MOGE_OK;
}


size_t moge_ep_workspace_size(const moge_config *cfg, int world) {
    moge_config loc, shr;
    if (check_config(cfg) != MOGE_OK || ep_configs(*cfg, 0, world, loc, shr) != MOGE_OK) return 0;
    return carve_ep(*cfg, loc, shr, nullptr).total;
}

int moge_layer_forward_ep_local(const moge_config *cfg, int rank, int world, const void *x_all,
                                const void *w_router, const float *logit_bias,
                                const void *w_gate, const void *w_up, const void *w_down,
                                const void *s_gate, const void *s_up, const void *s_down,
                                float *y_part, void *workspace, void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    moge_config loc, shr;
    if ((rc = ep_configs(c, rank, world, loc, shr))) return rc;
    MOGE_NEED(y_part, "y_part");
    cudaStream_t st = (cudaStream_t)stream;
    if (c.T == 0) return MOGE_OK;
    MOGE_NEED(x_all, "x_all");
    MOGE_NEED(w_router, "w_router");
    MOGE_NEED(w_gate, "w_gate");
    MOGE_NEED(w_up, "w_up");
    MOGE_NEED(w_down, "w_down");
    if (c.S > 0) {
        MOGE_NEED(s_gate, "s_gate");
        MOGE_NEED(s_up, "s_up");
        MOGE_NEED(s_down, "s_down");
    }
    if (logit_bias && !aligned4(logit_bias)) return fail(MOGE_ERR_UNSUPPORTED, "logit_bias misaligned");
    MOGE_NEED(workspace, "workspace");
    EpSpace es = carve_ep(c, loc, shr, workspace);
    const Workspace &lw = es.lw, &sw = es.sw;
    const int K = c.M * c.Kp, K_loc = loc.M * loc.Kp;
    const int tiles = (c.T + kRouterTile - 1) / kRouterTile;
    MOGE_CU(launch_router(c, x_all, w_router, logit_bias, es.topk_idx, es.topk_w, es.hist, es.rank,
                          num_sms(), st), "router launch");
    MOGE_CU(launch_localize(c.T, c.N, K, rank * K_loc, K_loc, rank * loc.N, loc.N, tiles,
                            es.topk_idx, es.topk_w, es.rank, es.hist, lw.topk_idx, lw.topk_w, lw.rank,
                            lw.hist, st), "localize launch");
    MOGE_CU(launch_scan(loc, lw.hist, lw.base, lw.counts, lw.offsets, &lw.plan, true, false, st),
            "scan launch");
    MOGE_CU(launch_scatter_rows(loc, x_all, lw.topk_idx, lw.rank, lw.base, lw.offsets, lw.perm_src,
                                lw.perm_dst, lw.x_perm, st), "permute launch");
    const int64_t rrows = (int64_t)c.T * K_loc;
    FfnOperands op{};
    op.b0 = lw.x_perm; op.b1 = x_all; op.b0_rows = rrows; op.b1_rows = c.T;
    op.wg = w_gate; op.wu = w_up; op.wd = w_down;
    op.h = lw.h; op.h_rows = rrows; op.y = lw.y_perm;
    rc = run_ffn(loc, lw.plan, loc.N, op, st);
    if (rc) return rc;
    if (c.S > 0) {
        MOGE_CU(launch_plan(shr, nullptr, sw.plan, false, true, st), "plan launch");
        FfnOperands os{};
        os.b1 = x_all; os.b1_rows = c.T;
        os.sg = s_gate; os.su = s_up; os.sd = s_down;
        os.h = sw.h; os.h_rows = (int64_t)c.T * c.S; os.y = sw.y_perm;
        rc = run_ffn(shr, sw.plan, c.S, os, st);
        if (rc) return rc;
    }
    MOGE_CU(launch_combine(loc, lw.y_perm, lw.topk_w, lw.perm_dst, K_loc, c.S ? sw.y_perm : nullptr,
                           c.S, nullptr, y_part, st, true), "combine launch");
    return MOGE_OK;
}

int moge_ep_finish(const moge_config *cfg, int64_t rows, const float *y_sum, const void *residual,
                   void *y, void *stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (rows < 0) return fail(MOGE_ERR_INVALID_ARG, "rows < 0");
    if (rows == 0) return MOGE_OK;
    MOGE_NEED(y_sum, "y_sum");
    MOGE_NEED(y, "y");
    if (residual && !aligned16(residual)) return fail(MOGE_ERR_UNSUPPORTED, "residual misaligned");
    MOGE_CU(launch_ep_finish(cfg->dtype, rows, cfg->d, y_sum, residual, y, (cudaStream_t)stream),
            "finish launch");
    return MOGE_OK;
}

}  // extern "C"
