// moge_route_noalloc: the routing entry point for callers that cannot hand the
// library a workspace. Some callers are not allowed to allocate device memory
// at all on their calling path: a plugin living inside another runtime whose
// device memory is reserved up front by that runtime's own pool, or a
// latency-bound serving loop where cudaMalloc / cudaFree would synchronise the
// device and stall every other stream. moge_route needs scratch memory for
// its per-tile histograms, row bases and ranks; this variant keeps that
// scratch in a fixed array in the library's own device image instead, so the
// caller passes only inputs and outputs and nothing is allocated.
//
// The array (kRouteScratchBytes) is part of the module: every GPU that loads
// the library holds it until the process exits. All calls on a device share
// it, so two calls that overlap on the GPU (different streams, or different
// host threads, without ordering between them) race on it and corrupt each
// other's routing; order such calls on one stream. The array keeps whatever
// the last call left in it; nothing needs clearing, because each call writes
// every scratch word it later reads (each router tile writes its whole
// histogram row, the scan writes every row base, the router writes the rank
// of every (token, pick)).
//
// In host code the array's name is only a host-side shadow, not a device
// address; the device address is taken with cudaGetSymbolAddress on the first
// call made while that device is current, and looked up again whenever the
// device's context is a different one (after a cudaDeviceReset the module is
// loaded anew, possibly at another address).
#include <mutex>

#include "common.cuh"
#include "moge_internal.h"

namespace moge {

constexpr size_t kRouteScratchBytes = size_t(1) << 20;  // 1 MiB
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

static std::mutex g_route_scratch_mu;
static void *g_route_scratch_dev[64] = {nullptr};
static void *g_route_scratch_ctx[64] = {nullptr};  // the context each address belongs to

// The calling thread's current driver context (through the runtime's driver
// entry point: the library does not link libcuda); nullptr if unavailable.
static void *current_context() {
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    static GetCurrentFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetCurrentFn>(ptr);
        tried = true;
    }
    CUcontext ctx = nullptr;
    if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

// Scratch layout: hist [tiles][N] | base [tiles][N] | rank [T][K], each
// region rounded up to 256 bytes.
static size_t route_scratch_layout(const moge_config &c, size_t *off_base, size_t *off_rank) {
    const size_t tiles = ((size_t)c.T + kRouterTile - 1) / kRouterTile;
    const size_t h = align256(tiles * (size_t)c.N * 4);
    const size_t r = align256((size_t)c.T * c.M * c.Kp * 4);
    *off_base = h;
    *off_rank = 2 * h;
    return 2 * h + r;
}

// Device address of the scratch array on the current device (set up once per
// device and context).
static int route_scratch_ptr(unsigned char **out) {
    int dev = -1;
    MOGE_CU(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(MOGE_ERR_UNSUPPORTED, "device index above 63");
    std::lock_guard<std::mutex> lock(g_route_scratch_mu);
    void *ctx = current_context();
    if (!g_route_scratch_dev[dev] || !ctx || ctx != g_route_scratch_ctx[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress(route scratch)");
        g_route_scratch_dev[dev] = p;
        // the runtime creates the context on the lookup above if none was current
        g_route_scratch_ctx[dev] = ctx ? ctx : current_context();
    }
    *out = static_cast<unsigned char *>(g_route_scratch_dev[dev]);
    return MOGE_OK;
}

}  // namespace moge

extern "C" int moge_route_noalloc(const moge_config *cfg, const void *x, const void *w_router,
                                  const float *logit_bias, int32_t *topk_idx, float *topk_w,
                                  int32_t *counts, int32_t *offsets, int32_t *perm_src,
                                  int32_t *perm_dst, void *stream) {
    using namespace moge;
    int rc = check_config(cfg);
    if (rc) return rc;
    const moge_config c = *cfg;
    size_t off_base = 0, off_rank = 0;
    const size_t need = route_scratch_layout(c, &off_base, &off_rank);
    if (need > kRouteScratchBytes)
        return fail(MOGE_ERR_UNSUPPORTED,
                    "moge_route_noalloc: this batch needs " + std::to_string(need) +
                        " bytes of routing scratch, above the fixed 1048576 (1 MiB); use moge_route "
                        "with a workspace");
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
    unsigned char *scratch = nullptr;
    rc = route_scratch_ptr(&scratch);
    if (rc) return rc;
    int32_t *hist = reinterpret_cast<int32_t *>(scratch);
    int32_t *base = reinterpret_cast<int32_t *>(scratch + off_base);
    int32_t *rank = reinterpret_cast<int32_t *>(scratch + off_rank);
    MOGE_CU(launch_router(c, x, w_router, logit_bias, topk_idx, topk_w, hist, rank, num_sms(), st),
            "router launch");
    MOGE_CU(launch_scan(c, hist, base, counts, offsets, nullptr, false, false, st), "scan launch");
    MOGE_CU(launch_finalize(c, topk_idx, rank, base, offsets, perm_src, perm_dst, st),
            "finalize launch");
    return MOGE_OK;
}
