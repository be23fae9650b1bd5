// Router of the MoGE layer: router GEMM, global fp32 softmax over all N
// experts, top-Kp inside every group, per-tile expert histogram and ranks;
// then the scan that turns the histograms into counts / offsets / row bases,
// the grouped-GEMM work plan, and the final permutation indices.
//
// Method: "Huawei releases Pangu Pro MoE" (techwalker.com), section 1: one
// softmax over all experts, then a local top-K' inside each of the M groups,
// which gives every group exactly T*K' assignments.
#include <cooperative_groups.h>

#include "common.cuh"
#include "moge_internal.h"

namespace cg = cooperative_groups;

namespace moge {

constexpr int kRouterWarps = 8;
constexpr int kRouterThreads = kRouterWarps * 32;

// ---------------------------------------------------------------------------
// Shared epilogue: logits [kRouterTile][N] fp32 in smem (bias not yet added)
// -> scores, picks, per-tile histogram, in-tile ranks.
struct RouterSmem {
    float logits[kRouterTile][kMaxExperts];
    float part[kRouterWarps][kRouterTile][64];  // per-warp partial sums (bf16 path)
    int ids[kRouterTile][kMaxExperts];          // picks, [t][k], k < K
};

// Order of candidates inside a group: higher score first, equal scores ->
// lower expert index first.
__device__ __forceinline__ bool ranks_before(float pa, int a, float pb, int b) {
    return pa > pb || (pa == pb && a < b);
}

__device__ void router_epilogue(RouterSmem &sm, const moge_config &c, const float *bias, int t0,
                                int32_t *topk_idx, float *topk_w, int32_t *hist, int32_t *rank) {
    const int N = c.N, M = c.M, Kp = c.Kp, K = M * Kp, G = N / M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntok = min(kRouterTile, c.T - t0);
    // one warp per token: global softmax over all N experts, fp32
    for (int tt = warp; tt < ntok; tt += kRouterWarps) {
        float m = -INFINITY;
        for (int e = lane; e < N; e += 32) {
            float l = sm.logits[tt][e] + (bias ? bias[e] : 0.0f);
            sm.logits[tt][e] = l;
            m = fmaxf(m, l);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float s = 0.0f;
        for (int e = lane; e < N; e += 32) {
            float v = expf(sm.logits[tt][e] - m);
            sm.logits[tt][e] = v;
            s += v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        for (int e = lane; e < N; e += 32) sm.logits[tt][e] = sm.logits[tt][e] / s;
        __syncwarp();
        // per-group top-Kp: the j-th pick is the first candidate (in the order
        // above) that ranks after the (j-1)-th pick
        for (int g = lane; g < M; g += 32) {
            int prev = -1;
            float pprev = 0.0f;
            for (int j = 0; j < Kp; ++j) {
                int best = -1;
                float pb = 0.0f;
                for (int e = g * G; e < (g + 1) * G; ++e) {
                    float pe = sm.logits[tt][e];
                    if (prev >= 0 && !ranks_before(pprev, prev, pe, e)) continue;
                    if (best < 0 || ranks_before(pe, e, pb, best)) { best = e; pb = pe; }
                }
                sm.ids[tt][g * Kp + j] = best;
                const size_t o = (size_t)(t0 + tt) * K + g * Kp + j;
                topk_idx[o] = best;
                topk_w[o] = pb;
                prev = best;
                pprev = pb;
            }
        }
    }
    __syncthreads();
    // histogram of this tile, and the rank of each (t, k) among the tile's
    // earlier tokens that picked the same expert (ascending token order)
    const int tile = t0 / kRouterTile;
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        const int g = e / G;
        int cnt = 0;
        for (int tt = 0; tt < ntok; ++tt)
            for (int j = 0; j < Kp; ++j) cnt += sm.ids[tt][g * Kp + j] == e;
        hist[(size_t)tile * N + e] = cnt;
    }
    for (int s = threadIdx.x; s < ntok * K; s += blockDim.x) {
        const int tt = s / K, k = s % K, g = k / Kp;
        const int e = sm.ids[tt][k];
        int r = 0;
        for (int t2 = 0; t2 < tt; ++t2)
            for (int j = 0; j < Kp; ++j) r += sm.ids[t2][g * Kp + j] == e;
        rank[(size_t)(t0 + tt) * K + k] = r;
    }
}

// ---------------------------------------------------------------------------
// bf16 router GEMM with mma.sync m16n8k16 (the N <= 256 output columns are far
// too narrow for a tcgen05 tile to pay). A cluster of `ks` CTAs splits the
// hidden dimension of one 16-token tile; rank 0 reduces the partial logits
// through distributed shared memory in a fixed order (deterministic).
//
// k-slot mapping: for each 32-wide chunk of the hidden dimension, the thread
// with quad index q loads hidden elements [8q, 8q+8) of its A rows and of its
// B rows, and feeds them to two m16n8k16 steps as the k-slots {2q, 2q+1,
// 2q+8, 2q+9}. A and B use the same mapping, so every product pairs equal
// hidden indices; the sum over the chunk is unchanged.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kRouterThreads) router_bf16_kernel(
    moge_config c, const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr,
    const float *__restrict__ bias, int32_t *topk_idx, float *topk_w, int32_t *hist, int32_t *rank,
    int ks) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RouterSmem &sm = *reinterpret_cast<RouterSmem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int crank = blockIdx.x % ks;
    const int t0 = (blockIdx.x / ks) * kRouterTile;
    const int d = c.d, N = c.N;
    const int nchunk = (d + 31) / 32;
    const int c_begin = (int)((long long)nchunk * crank / ks);
    const int c_end = (int)((long long)nchunk * (crank + 1) / ks);
    const int ra = t0 + g, rb = t0 + g + 8;
    const bool va = ra < c.T, vb = rb < c.T;
    const uint16_t *xa = x + (size_t)(va ? ra : 0) * d;
    const uint16_t *xb = x + (size_t)(vb ? rb : 0) * d;

    for (int n0 = 0; n0 < N; n0 += 64) {  // pass over 64 experts (8 n-tiles)
        const int ntile = min(8, (N - n0) / 8);
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
        for (int ch = c_begin + warp; ch < c_end; ch += kRouterWarps) {
            const int k = ch * 32 + 8 * q;
            const bool kv = k < d;  // d % 8 == 0: a 16-byte vector is all in or all out
            uint4 av = make_uint4(0, 0, 0, 0), bv = make_uint4(0, 0, 0, 0);
            if (kv && va) av = __ldg(reinterpret_cast<const uint4 *>(xa + k));
            if (kv && vb) bv = __ldg(reinterpret_cast<const uint4 *>(xb + k));
            uint4 wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                wv[i] = make_uint4(0, 0, 0, 0);
                if (i < ntile && kv)
                    wv[i] = __ldg(reinterpret_cast<const uint4 *>(wr + (size_t)(n0 + i * 8 + g) * d + k));
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i < ntile) {
                    mma_bf16_16816(acc[i], av.x, bv.x, av.y, bv.y, wv[i].x, wv[i].y);
                    mma_bf16_16816(acc[i], av.z, bv.z, av.w, bv.w, wv[i].z, wv[i].w);
                }
            }
        }
        // per-warp partials -> smem, then a fixed-order sum over warps
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < ntile) {
                sm.part[warp][g][i * 8 + 2 * q] = acc[i][0];
                sm.part[warp][g][i * 8 + 2 * q + 1] = acc[i][1];
                sm.part[warp][g + 8][i * 8 + 2 * q] = acc[i][2];
                sm.part[warp][g + 8][i * 8 + 2 * q + 1] = acc[i][3];
            }
        }
        __syncthreads();
        for (int o = threadIdx.x; o < kRouterTile * ntile * 8; o += blockDim.x) {
            const int tt = o / (ntile * 8), e = o % (ntile * 8);
            float s = 0.0f;
#pragma unroll
            for (int w = 0; w < kRouterWarps; ++w) s += sm.part[w][tt][e];
            sm.logits[tt][n0 + e] = s;
        }
        __syncthreads();
    }

    if (ks > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();  // every CTA's partial logits are complete
        if (crank == 0) {
            for (int o = threadIdx.x; o < kRouterTile * N; o += blockDim.x) {
                const int tt = o / N, e = o % N;
                float s = sm.logits[tt][e];
                for (int r = 1; r < ks; ++r) {
                    const RouterSmem *rs = cluster.map_shared_rank(&sm, r);
                    s += rs->logits[tt][e];
                }
                sm.logits[tt][e] = s;
            }
        }
        cluster.sync();  // peers keep their shared memory until rank 0 has read it
        if (crank != 0) return;
        __syncthreads();
    }
    router_epilogue(sm, c, bias, t0, topk_idx, topk_w, hist, rank);
}

// fp32 router (CUDA cores, sequential sum over the hidden dimension)
__global__ void __launch_bounds__(kRouterThreads) router_f32_kernel(
    moge_config c, const float *__restrict__ x, const float *__restrict__ wr,
    const float *__restrict__ bias, int32_t *topk_idx, float *topk_w, int32_t *hist,
    int32_t *rank) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RouterSmem &sm = *reinterpret_cast<RouterSmem *>(smem_raw);
    const int t0 = blockIdx.x * kRouterTile;
    const int ntok = min(kRouterTile, c.T - t0);
    for (int o = threadIdx.x; o < kRouterTile * c.N; o += blockDim.x) {
        const int tt = o / c.N, e = o % c.N;
        float s = 0.0f;
        if (tt < ntok) {
            const float *xr = x + (size_t)(t0 + tt) * c.d;
            const float *wrow = wr + (size_t)e * c.d;
            for (int k = 0; k < c.d; ++k) s = fmaf(xr[k], wrow[k], s);
        }
        sm.logits[tt][e] = s;
    }
    __syncthreads();
    router_epilogue(sm, c, bias, t0, topk_idx, topk_w, hist, rank);
}

cudaError_t launch_router(const moge_config &c, const void *x, const void *w_router,
                          const float *bias, int32_t *topk_idx, float *topk_w, int32_t *hist,
                          int32_t *rank, int num_sms, cudaStream_t st) {
    const int tiles = (c.T + kRouterTile - 1) / kRouterTile;
    const size_t smem = sizeof(RouterSmem);
    if (c.dtype == MOGE_F32) {
        cudaError_t e = cudaFuncSetAttribute(router_f32_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        router_f32_kernel<<<tiles, kRouterThreads, smem, st>>>(
            c, (const float *)x, (const float *)w_router, bias, topk_idx, topk_w, hist, rank);
        return cudaGetLastError();
    }
    // split the hidden dimension over a cluster when there are few tiles
    int ks = 1;
    while (ks < 8 && tiles * ks * 2 <= 2 * num_sms && (c.d / 32) >= ks * 2 * kRouterWarps) ks *= 2;
    cudaError_t e = cudaFuncSetAttribute(router_bf16_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles * ks);
    cfg.blockDim = dim3(kRouterThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_bf16_kernel, c, (const uint16_t *)x,
                              (const uint16_t *)w_router, bias, topk_idx, topk_w, hist, rank, ks);
}

// ---------------------------------------------------------------------------
// Work plan of the grouped FFN. Entries: routed experts 0..N-1 (if
// with_routed), then shared experts 0..S-1 (if with_shared).
__device__ void build_plan(const moge_config &c, const int32_t *offsets, Plan plan,
                           bool with_routed, bool with_shared, int shared_row_base) {
    const int K = c.M * c.Kp;
    const int fb_up = (c.I + 63) / 64;      // 64 gate + 64 up rows per tile
    const int fb_down = (c.d + 127) / 128;  // 128 output features per tile
    int n = 0, su = 0, sd = 0;
    auto add = [&](int rows, int a_sel, int a_idx, int up_src, int up_bsel, int mid_row) {
        ExpertWork w;
        w.rows = rows;
        w.a_sel = a_sel;
        w.a_idx = a_idx;
        if (rows <= 0) {
            w.bn = 16;
            w.ntb = 0;
        } else if (rows <= kStreamRows) {
            w.bn = (rows + 15) & ~15;
            w.ntb = 1;
        } else {
            const int ntb = (rows + kMaxTileN - 1) / kMaxTileN;
            const int per = (rows + ntb - 1) / ntb;
            w.bn = (per + 15) & ~15;
            w.ntb = (rows + w.bn - 1) / w.bn;
        }
        ExpertWork u = w, dn = w;
        u.src_row0 = up_src;
        u.b_sel = up_bsel;
        u.dst_row0 = mid_row;
        dn.src_row0 = mid_row;
        dn.b_sel = 0;
        dn.dst_row0 = mid_row;
        plan.up[n] = u;
        plan.down[n] = dn;
        plan.up_start[n] = su;
        plan.down_start[n] = sd;
        su += w.ntb * fb_up;
        sd += w.ntb * fb_down;
        ++n;
    };
    (void)K;
    if (with_routed)
        for (int e = 0; e < c.N; ++e)
            add(offsets[e + 1] - offsets[e], 0, e, offsets[e], 0, offsets[e]);
    if (with_shared)
        for (int s = 0; s < c.S; ++s) add(c.T, 1, s, 0, 1, shared_row_base + s * c.T);
    plan.up_start[n] = su;
    plan.down_start[n] = sd;
}

// Column sums of hist over tiles -> base (exclusive), counts, offsets;
// checks the equal group load; optionally writes the layer's GEMM plan.
__global__ void __launch_bounds__(1024) scan_kernel(moge_config c, const int32_t *__restrict__ hist,
                                                     int32_t *base, int32_t *counts,
                                                     int32_t *offsets, Plan plan, int make_plan,
                                                     int with_routed, int with_shared) {
    __shared__ int32_t part[1024];
    __shared__ int32_t cnt_s[kMaxExperts + 1];
    const int N = c.N;
    const int tiles = (c.T + kRouterTile - 1) / kRouterTile;
    const int P = blockDim.x / N;  // chunks of tiles
    const int e = threadIdx.x % N, p = threadIdx.x / N;
    const bool act = p < P;
    const int tb = act ? (int)((long long)tiles * p / P) : 0;
    const int te = act ? (int)((long long)tiles * (p + 1) / P) : 0;
    int s = 0;
    for (int t = tb; t < te; ++t) s += hist[(size_t)t * N + e];
    if (act) part[p * N + e] = s;
    __syncthreads();
    if (threadIdx.x < N) {  // exclusive scan over chunks, per expert
        int run = 0;
        for (int pp = 0; pp < P; ++pp) {
            const int v = part[pp * N + threadIdx.x];
            part[pp * N + threadIdx.x] = run;
            run += v;
        }
        cnt_s[threadIdx.x] = run;
        counts[threadIdx.x] = run;
    }
    __syncthreads();
    if (act) {
        int run = part[p * N + e];
        for (int t = tb; t < te; ++t) {
            base[(size_t)t * N + e] = run;
            run += hist[(size_t)t * N + e];
        }
    }
    if (threadIdx.x == 0) {
        const int G = N / c.M;
        int run = 0;
        for (int i = 0; i < N; ++i) {
            offsets[i] = run;
            run += cnt_s[i];
        }
        offsets[N] = run;
        for (int g = 0; g < c.M; ++g) {  // every group carries exactly T*Kp assignments
            int lg = 0;
            for (int i = g * G; i < (g + 1) * G; ++i) lg += cnt_s[i];
            if (lg != c.T * c.Kp) raise_error(ERRBIT_INVARIANT);
        }
    }
    if (make_plan) {
        __syncthreads();
        if (threadIdx.x == 0)
            build_plan(c, offsets, plan, with_routed != 0, with_shared != 0, c.T * c.M * c.Kp);
    }
}

cudaError_t launch_scan(const moge_config &c, const int32_t *hist, int32_t *base, int32_t *counts,
                        int32_t *offsets, const Plan *plan, bool with_routed, bool with_shared,
                        cudaStream_t st) {
    const int threads = (1024 / c.N) * c.N;
    Plan p = plan ? *plan : Plan{nullptr, nullptr, nullptr, nullptr};
    scan_kernel<<<1, threads, 0, st>>>(c, hist, base, counts, offsets, p, plan ? 1 : 0,
                                        with_routed ? 1 : 0, with_shared ? 1 : 0);
    return cudaGetLastError();
}

__global__ void plan_kernel(moge_config c, const int32_t *offsets, Plan plan, int with_routed,
                            int with_shared) {
    if (threadIdx.x == 0 && blockIdx.x == 0)
        build_plan(c, offsets, plan, with_routed != 0, with_shared != 0,
                   with_routed ? c.T * c.M * c.Kp : 0);
}

cudaError_t launch_plan(const moge_config &c, const int32_t *offsets, const Plan &plan,
                        bool with_routed, bool with_shared, cudaStream_t st) {
    plan_kernel<<<1, 32, 0, st>>>(c, offsets, plan, with_routed ? 1 : 0, with_shared ? 1 : 0);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// perm_dst[t][k] = offsets[e] + base[tile(t)][e] + rank[t][k];  perm_src[that] = t
__global__ void finalize_kernel(moge_config c, const int32_t *__restrict__ topk_idx,
                                const int32_t *__restrict__ rank, const int32_t *__restrict__ base,
                                const int32_t *__restrict__ offsets, int32_t *perm_src,
                                int32_t *perm_dst) {
    const int K = c.M * c.Kp;
    const long long n = (long long)c.T * K;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(i / K);
        const int e = topk_idx[i];
        if (e < 0 || e >= c.N) {
            raise_error(ERRBIT_INVARIANT);
            continue;
        }
        const int row = offsets[e] + base[(size_t)(t / kRouterTile) * c.N + e] + rank[i];
        perm_dst[i] = row;
        perm_src[row] = t;
    }
}

cudaError_t launch_finalize(const moge_config &c, const int32_t *topk_idx, const int32_t *rank,
                            const int32_t *base, const int32_t *offsets, int32_t *perm_src,
                            int32_t *perm_dst, cudaStream_t st) {
    const long long n = (long long)c.T * c.M * c.Kp;
    const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    finalize_kernel<<<blocks > 0 ? blocks : 1, 256, 0, st>>>(c, topk_idx, rank, base, offsets,
                                                             perm_src, perm_dst);
    return cudaGetLastError();
}

}  // namespace moge
