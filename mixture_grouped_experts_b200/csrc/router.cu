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
// Shared epilogue. The CTA's tile of tb tokens has its logits [tb][N] (fp32,
// bias not yet added) in shared memory; this computes the scores, the picks,
// and for every 16-token sub-tile the expert histogram and the in-tile ranks.
struct RouterView {
    float *logits;  // [tb][N]
    int16_t *ids;   // [tb][K] picks
    int tb;
};

// Order of candidates inside a group: higher score first, equal scores ->
// lower expert index first.
__device__ __forceinline__ bool ranks_before(float pa, int a, float pb, int b) {
    return pa > pb || (pa == pb && a < b);
}

// Lane-per-group epilogue (M a power of two <= 32, groups of G = 8, 16 or 32
// experts, Kp <= 2): a token takes M consecutive lanes, lane g of its segment
// holding the G scores of group g in registers, so a warp works on 32 / M
// tokens at once; max and sum need log2(M) shuffle steps, the in-group top-Kp
// is a scan of registers. Histogram and ranks of every 16-token sub-tile then
// come from one warp per (sub-tile, group): its lanes hold the sub-tile's
// picks in that group, __match_any_sync groups equal experts (rank = equal
// picks of earlier tokens, ascending tokens), one ballot per expert counts.
template <int G>
__device__ void router_epilogue_lanes(const RouterView &sm, const moge_config &c, const float *bias,
                                      int t0, int32_t *topk_idx, float *topk_w, int32_t *hist,
                                      int32_t *rank) {
    const int N = c.N, M = c.M, Kp = c.Kp, K = M * Kp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int ntok = min(sm.tb, c.T - t0);
    const int per_warp = 32 / M;  // tokens a warp handles at once
    const int g = lane % M, seg = lane / M;
    for (int tb0 = warp * per_warp; tb0 < ntok; tb0 += nwarps * per_warp) {
        const int tt = tb0 + seg;
        const bool live = tt < ntok;
        float v[G];
        float m = -INFINITY;
        const float *lg = sm.logits + (size_t)(live ? tt : 0) * N + g * G;
#pragma unroll
        for (int j = 0; j < G; ++j) {
            v[j] = lg[j] + (bias ? bias[g * G + j] : 0.0f);
            m = fmaxf(m, v[j]);
        }
        for (int o = M >> 1; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float z = 0.0f;
#pragma unroll
        for (int j = 0; j < G; ++j) {
            v[j] = expf(v[j] - m);
            z += v[j];
        }
        for (int o = M >> 1; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
        for (int j = 0; j < G; ++j) v[j] = v[j] / z;
        int prev = -1;
        for (int k = 0; k < Kp; ++k) {
            int best = -1;
            float pb = 0.0f;
#pragma unroll
            for (int j = 0; j < G; ++j) {  // Kp <= 2: the second pick skips the first
                if (j == prev) continue;
                if (best < 0 || ranks_before(v[j], j, pb, best)) { best = j; pb = v[j]; }
            }
            if (live) {
                const int e = g * G + best;
                const size_t o = (size_t)(t0 + tt) * K + g * Kp + k;
                topk_idx[o] = e;
                topk_w[o] = pb;
                sm.ids[(size_t)tt * K + g * Kp + k] = (int16_t)e;
            }
            prev = best;
        }
    }
    __syncthreads();
    const int nsub = (ntok + kRouterTile - 1) / kRouterTile;
    for (int pr = warp; pr < nsub * M; pr += nwarps) {
        const int sub = pr / M, gg = pr % M;
        const int tl = lane / Kp, j = lane % Kp;       // token in the sub-tile, pick
        const int tt = sub * kRouterTile + tl;
        const bool valid = lane < kRouterTile * Kp && tt < ntok;
        const int e = valid ? (int)sm.ids[(size_t)tt * K + gg * Kp + j] : -1 - lane;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        if (valid) rank[(size_t)(t0 + tt) * K + gg * Kp + j] = __popc(same & ((1u << (tl * Kp)) - 1u));
        int cnt = 0;
        for (int x = 0; x < G; ++x) {
            const int n = __popc(__ballot_sync(0xffffffffu, e == gg * G + x));
            if (lane == x) cnt = n;
        }
        if (lane < G) hist[(size_t)(t0 / kRouterTile + sub) * N + gg * G + lane] = cnt;
    }
}

__device__ void router_epilogue(const RouterView &sm, const moge_config &c, const float *bias,
                                int t0, int32_t *topk_idx, float *topk_w, int32_t *hist,
                                int32_t *rank) {
    const int N = c.N, M = c.M, Kp = c.Kp, K = M * Kp, G = N / M;
    if (M <= 32 && 32 % M == 0 && Kp <= 2) {
        if (G == 8) return router_epilogue_lanes<8>(sm, c, bias, t0, topk_idx, topk_w, hist, rank);
        if (G == 16) return router_epilogue_lanes<16>(sm, c, bias, t0, topk_idx, topk_w, hist, rank);
        if (G == 32) return router_epilogue_lanes<32>(sm, c, bias, t0, topk_idx, topk_w, hist, rank);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int ntok = min(sm.tb, c.T - t0);
    // register path: every lane holds N/32 scores; a group of G (a power of
    // two <= 32) lies inside one 32-lane segment, so its top-Kp is found with
    // xor-shuffles inside G-lane segments
    const bool shuffle = (N % 32 == 0) && G <= 32 && (G & (G - 1)) == 0;
    for (int tt = warp; tt < ntok; tt += nwarps) {
        float *lg = sm.logits + (size_t)tt * N;
        if (shuffle) {
            const int J = N / 32;
            float v[kMaxExperts / 32];
            float m = -INFINITY;
#pragma unroll
            for (int j = 0; j < kMaxExperts / 32; ++j) {
                if (j < J) {
                    const int e = lane + 32 * j;
                    v[j] = lg[e] + (bias ? bias[e] : 0.0f);
                    m = fmaxf(m, v[j]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float z = 0.0f;
#pragma unroll
            for (int j = 0; j < kMaxExperts / 32; ++j)
                if (j < J) {
                    v[j] = expf(v[j] - m);
                    z += v[j];
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
            for (int j = 0; j < kMaxExperts / 32; ++j) {
                if (j >= J) continue;
                float pv = v[j] / z;  // this lane's candidate; -inf once picked
                for (int k = 0; k < Kp; ++k) {
                    float bp = pv;
                    int bi = lane + 32 * j;
                    for (int o = G >> 1; o > 0; o >>= 1) {
                        const float op = __shfl_xor_sync(0xffffffffu, bp, o);
                        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                        if (ranks_before(op, oi, bp, bi)) { bp = op; bi = oi; }
                    }
                    if (bi == lane + 32 * j) pv = -INFINITY;
                    if ((lane & (G - 1)) == 0) {
                        const int g = (lane + 32 * j) / G;
                        const size_t o = (size_t)(t0 + tt) * K + g * Kp + k;
                        topk_idx[o] = bi;
                        topk_w[o] = bp;
                        sm.ids[(size_t)tt * K + g * Kp + k] = (int16_t)bi;
                    }
                }
            }
            continue;
        }
        // shared-memory path (any group size)
        float m = -INFINITY;
        for (int e = lane; e < N; e += 32) {
            float l = lg[e] + (bias ? bias[e] : 0.0f);
            lg[e] = l;
            m = fmaxf(m, l);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float z = 0.0f;
        for (int e = lane; e < N; e += 32) {
            float v = expf(lg[e] - m);
            lg[e] = v;
            z += v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        for (int e = lane; e < N; e += 32) lg[e] = lg[e] / z;
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
                    const float pe = lg[e];
                    if (prev >= 0 && !ranks_before(pprev, prev, pe, e)) continue;
                    if (best < 0 || ranks_before(pe, e, pb, best)) { best = e; pb = pe; }
                }
                sm.ids[(size_t)tt * K + g * Kp + j] = (int16_t)best;
                const size_t o = (size_t)(t0 + tt) * K + g * Kp + j;
                topk_idx[o] = best;
                topk_w[o] = pb;
                prev = best;
                pprev = pb;
            }
        }
    }
    __syncthreads();
    // per 16-token sub-tile: histogram, and the rank of each (t, k) among the
    // sub-tile's earlier tokens that picked the same expert (ascending tokens)
    const int nsub = (ntok + kRouterTile - 1) / kRouterTile;
    for (int i = threadIdx.x; i < nsub * N; i += blockDim.x) {
        const int sub = i / N, e = i % N, g = e / G;
        const int ta = sub * kRouterTile, tz = min(ntok, ta + kRouterTile);
        int cnt = 0;
        for (int tt = ta; tt < tz; ++tt)
            for (int j = 0; j < Kp; ++j) cnt += sm.ids[(size_t)tt * K + g * Kp + j] == e;
        hist[(size_t)(t0 / kRouterTile + sub) * N + e] = cnt;
    }
    for (int i = threadIdx.x; i < ntok * K; i += blockDim.x) {
        const int tt = i / K, k = i % K, g = k / Kp;
        const int e = sm.ids[i];
        int r = 0;
        for (int t2 = (tt / kRouterTile) * kRouterTile; t2 < tt; ++t2)
            for (int j = 0; j < Kp; ++j) r += sm.ids[(size_t)t2 * K + g * Kp + j] == e;
        rank[(size_t)(t0 + tt) * K + k] = r;
    }
}

// ---------------------------------------------------------------------------
// bf16 router GEMM on the tensor cores. One CTA owns a tile of TB = 16*TBM
// tokens and a slice of the hidden dimension; a cluster of `ks` CTAs splits
// the hidden dimension of one tile and the leader adds the partial logits in
// rank order (deterministic). Thread 0 streams the slice through a ring of
// `nst` stages with TMA, one 64-wide K-chunk per stage: a box of TB token rows
// and a box of 128 (or 256) router rows, rows past N arriving as zeros, both
// 128-byte swizzled. Thread 32 issues tcgen05.mma with the router rows as A
// (M = 128 per half) and the token rows as B (N = TB), fp32 accumulation in
// tensor memory, and frees each stage with tcgen05.commit. The accumulator
// D[expert][token] then goes to shared memory as logits [token][expert] for
// the epilogue. (The warp-level mma.sync path it replaces was bound by that
// instruction's low issue rate on this architecture.) Long batches use
// 64-token tiles, which read the router matrix a quarter as often.

constexpr int kRouterChunk = 64;      // hidden elements per stage (128 bytes per row)
constexpr int kRouterMaxStages = 12;

// bytes of one stage: TB token rows and N router rows of 128 bytes (a
// multiple of 1024 since TB % 16 == 0 and N % 8 == 0)
__host__ __device__ inline int router_stage_bytes(int tb, int n) { return (tb + n) * 128; }

template <int TBM>
__global__ void __launch_bounds__(kRouterThreads, TBM == 1 ? 2 : 1) router_bf16_kernel(
    moge_config c, const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
    const float *__restrict__ bias, int32_t *topk_idx, float *topk_w, int32_t *hist, int32_t *rank,
    int ks, int nst) {
    constexpr int TB = kRouterTile * TBM;
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    __shared__ uint64_t full[kRouterMaxStages], empty[kRouterMaxStages], done;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    unsigned char *stage = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const int N = c.N;
    const int mh = N <= 128 ? 1 : 2;                 // 128-row halves of the router matrix
    const int sbytes = router_stage_bytes(TB, 128 * mh);
    RouterView sm;
    sm.logits = reinterpret_cast<float *>(stage + (size_t)nst * sbytes);
    sm.ids = reinterpret_cast<int16_t *>(sm.logits + TB * N);
    sm.tb = TB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int crank = blockIdx.x % ks;
    const int t0 = (blockIdx.x / ks) * TB;
    // this CTA's slice of the hidden dimension, in whole chunks
    const int nck = (c.d + kRouterChunk - 1) / kRouterChunk;
    const int cb = (int)((long long)nck * crank / ks), ce = (int)((long long)nck * (crank + 1) / ks);
    const int nc = ce - cb;
    // accumulator columns: half h at h * hs (hs >= 32, so every 32-column read
    // below stays inside the allocation), allocation a power of two >= 32
    constexpr int hs = TB < 32 ? 32 : TB;
    uint32_t tcols = 32;
    while (tcols < (uint32_t)(hs * mh)) tcols <<= 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);   // the producer's expect_tx arrival (+ the copies' bytes)
            mbar_init(&empty[s], 1);  // the MMA thread's commit
        }
        mbar_init(&done, 1);
        abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    grid_dependency_wait();
    volatile int *abort = &abort_flag;

    // Lane 0 of warp 0 produces and lane 0 of warp 1 issues the MMAs; the other
    // lanes of those two warps wait at __syncwarp (parked, not polling), so the
    // working lane does not share its warp's issue slots with a wait loop.
    if (threadIdx.x == 0) {
        // ---- producer: chunk i of the slice into stage i % nst, a box of TB
        // token rows then the router rows (rows past T and past N come as zeros)
        const uint64_t pol_x = policy_evict_first(), pol_w = policy_evict_last();
        int issued = 0;
        for (; issued < nc; ++issued) {
            const int s = issued % nst;
            if (issued >= nst && !mbar_wait(&empty[s], (uint32_t)(issued / nst - 1) & 1u, abort)) break;
            unsigned char *st = stage + (size_t)s * sbytes;
            mbar_arrive_expect_tx(&full[s], (uint32_t)sbytes);
            tma_load_2d(st, &tmX, &full[s], (cb + issued) * kRouterChunk, t0, pol_x);
            tma_load_2d(st + TB * 128, &tmW, &full[s], (cb + issued) * kRouterChunk, 0, pol_w);
        }
        if (*abort) {  // let the copies in flight land before the stages are reused
            for (int s = 0; s < nst && s < issued; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % nst);
                mbar_wait(&full[s], (uint32_t)(last / nst) & 1u, nullptr);
            }
        }
    } else if (threadIdx.x == 32) {
        // ---- MMA issuer: D[expert][token] += W_chunk * x_chunk^T, M = 128 per half
        const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)TB);
        for (int i = 0; i < nc; ++i) {
            const int s = i % nst;
            if (!mbar_wait(&full[s], (uint32_t)(i / nst) & 1u, abort)) break;
            tc_fence_after();
            const uint32_t sb = smem_u32(stage + (size_t)s * sbytes);
            for (int h = 0; h < mh; ++h)
#pragma unroll
                for (int j = 0; j < kRouterChunk / 16; ++j)  // 16-wide K steps: +32 bytes
                    tc_mma_bf16(tm + (uint32_t)(h * hs), smem_desc_sw128(sb + TB * 128 + h * 16384 + 32 * j),
                                smem_desc_sw128(sb + 32 * j), idesc, (i | j) > 0 ? 1u : 0u);
            tc_commit(&empty[s]);  // the stage may be refilled once these MMAs have read it
        }
        tc_commit(&done);  // every MMA of this CTA has completed after this
    }
    if (warp < 2) __syncwarp();
    // ---- everyone: the accumulator is final; TMEM -> logits [token][expert]
    const bool ok = mbar_wait(&done, 0u, nullptr) && !*abort;
    __syncthreads();
    tc_fence_after();
    {
        const int q4 = warp & 3, wg = warp >> 2;   // TMEM lane quarter, warp group
        const int ncb = (TB + 31) / 32;            // 32-column blocks per half
        for (int idx = wg; idx < mh * ncb; idx += 2) {
            const int h = idx / ncb, c0 = (idx % ncb) * 32;
            uint32_t v[32];
            tmem_ld_32x32b_x32(tm + ((uint32_t)(32 * q4) << 16) + (uint32_t)(h * hs + c0), v);
            tmem_ld_wait();
            const int e = h * 128 + 32 * q4 + lane;
            if (e < N) {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj)
                    if (c0 + jj < TB) sm.logits[(size_t)(c0 + jj) * N + e] = ok ? __uint_as_float(v[jj]) : 0.0f;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, tcols);  // before any CTA of the cluster returns

    if (ks > 1) {
        // peers push their partial logits into the leader's (now idle) stage
        // buffers; the leader adds them in rank order
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();  // all partial logits are final; every CTA is past its K-loop
        float *land = reinterpret_cast<float *>(stage);
        if (crank != 0) {
            float *dst = cluster.map_shared_rank(land, 0) + (size_t)(crank - 1) * TB * N;
            for (int o = threadIdx.x; o < TB * N; o += blockDim.x) dst[o] = sm.logits[o];
        }
        cluster.sync();  // the pushes are visible to the leader
        if (crank != 0) return;
        for (int o = threadIdx.x; o < TB * N; o += blockDim.x) {
            float sum = sm.logits[o];
            for (int r = 1; r < ks; ++r) sum += land[(size_t)(r - 1) * TB * N + o];
            sm.logits[o] = sum;
        }
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
    RouterView sm;
    sm.logits = reinterpret_cast<float *>(smem_raw);
    sm.ids = reinterpret_cast<int16_t *>(sm.logits + kRouterTile * c.N);
    sm.tb = kRouterTile;
    grid_dependency_wait();
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
        sm.logits[o] = s;
    }
    __syncthreads();
    router_epilogue(sm, c, bias, t0, topk_idx, topk_w, hist, rank);
}

template <int TBM>
static cudaError_t launch_router_bf16(const moge_config &c, const void *x, const void *w_router,
                                      const float *bias, int32_t *topk_idx, float *topk_w,
                                      int32_t *hist, int32_t *rank, int num_sms, cudaStream_t st) {
    constexpr int TB = kRouterTile * TBM;
    const int tiles = (c.T + TB - 1) / TB;
    const int per_sm = TBM == 1 ? 2 : 1;
    const int mh = c.N <= 128 ? 1 : 2;  // the router box is 128 (or 256) rows, zero past N
    const int sb = router_stage_bytes(TB, 128 * mh);
    // as many stages as the CTA's shared-memory budget holds (two CTAs per SM
    // with 16-token tiles, one with 64-token tiles)
    const size_t fixed = 1024 + (size_t)TB * c.N * 4 + (size_t)TB * c.M * c.Kp * 2;
    const size_t budget = TBM == 1 ? 100 * 1024 : 200 * 1024;
    int nst = budget > fixed ? (int)((budget - fixed) / sb) : 0;
    nst = nst > kRouterMaxStages ? kRouterMaxStages : nst < 2 ? 2 : nst;
    // Split the hidden dimension over a cluster of up to 8 CTAs while the grid
    // stays within one wave, each CTA keeps >= 2 chunks, and the leader's
    // landing buffer (its stages) holds the (ks - 1) partial tiles.
    const int nck = (c.d + kRouterChunk - 1) / kRouterChunk;
    int ks = 1;
    while (ks < 8 && tiles * 2 * ks <= per_sm * num_sms && nck >= 2 * 2 * ks &&
           (size_t)(2 * ks - 1) * TB * c.N * 4 <= (size_t)nst * sb)
        ks *= 2;
    CUtensorMap mX, mW;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)c.d, (cuuint64_t)c.T};
        const cuuint64_t strides[1] = {(cuuint64_t)c.d * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kRouterChunk, (cuuint32_t)TB};
        if (!encode(&mX, x, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)c.d, (cuuint64_t)c.N};
        const cuuint64_t strides[1] = {(cuuint64_t)c.d * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kRouterChunk, (cuuint32_t)(128 * mh)};
        if (!encode(&mW, w_router, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    const size_t smem = fixed + (size_t)nst * sb;
    auto kern = router_bf16_kernel<TBM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles * ks);
    cfg.blockDim = dim3(kRouterThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, c, mX, mW, bias, topk_idx, topk_w, hist, rank, ks, nst);
}

cudaError_t launch_router(const moge_config &c, const void *x, const void *w_router,
                          const float *bias, int32_t *topk_idx, float *topk_w, int32_t *hist,
                          int32_t *rank, int num_sms, cudaStream_t st) {
    if (c.dtype == MOGE_F32) {
        const int tiles = (c.T + kRouterTile - 1) / kRouterTile;
        const size_t smem = (size_t)kRouterTile * c.N * 4 + (size_t)kRouterTile * c.M * c.Kp * 2;
        cudaError_t e = cudaFuncSetAttribute(router_f32_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(router_f32_kernel, dim3(tiles), dim3(kRouterThreads), smem, st, c,
                          (const float *)x, (const float *)w_router, bias, topk_idx, topk_w, hist,
                          rank);
    }
    // long batches with few experts: 64-token tiles (one CTA per SM);
    // otherwise 16-token tiles (two CTAs per SM, up to 8-CTA clusters over the
    // hidden dimension)
    if (c.N <= 64 && c.T >= 1024)
        return launch_router_bf16<4>(c, x, w_router, bias, topk_idx, topk_w, hist, rank, num_sms, st);
    return launch_router_bf16<1>(c, x, w_router, bias, topk_idx, topk_w, hist, rank, num_sms, st);
}

// ---------------------------------------------------------------------------
// Exclusive prefix sum across a block of exactly 1024 threads: returns the sum
// of v over the threads before this one; *total receives the block sum.
// Every thread must call it (it synchronises the block).
__device__ int block_exclusive_scan_1024(int v, int *wbuf /* [32] */, int *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wbuf[w] = x;
    __syncthreads();
    if (w == 0) {
        int t = wbuf[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        wbuf[lane] = t;
    }
    __syncthreads();
    const int pre = (w > 0 ? wbuf[w - 1] : 0) + x - v;
    *total = wbuf[31];
    __syncthreads();
    return pre;
}

// Work plan of the grouped FFN, one entry per thread: shared experts 0..S-1
// first (if with_shared; T rows each, their h / y rows after shared_row_base),
// then routed experts 0..N-1 (if with_routed, rows from offs[]). The grouped
// FFN hands its work out in this order, so the heavy shared-expert items come
// first. Token-tile width: <= kStreamRows rows -> one streaming tile of
// round16(rows); more -> ceil(rows / max_tile) balanced tiles of round16 width
// (never above max_tile, a multiple of 16).
// Also zeroes the FFN's work-queue counter and per-entry completion counters.
// Called by all 1024 threads of the block.
__device__ void build_plan_block(const moge_config &c, const int32_t *offs, Plan plan,
                                 bool with_routed, bool with_shared, int shared_row_base,
                                 int max_tile, int *wbuf) {
    const int fb_up = (c.I + 63) / 64;      // 64 gate + 64 up rows per tile
    const int fb_down = (c.d + 127) / 128;  // 128 output features per tile
    const int ns = with_shared ? c.S : 0;
    const int n = ns + (with_routed ? c.N : 0);
    const int i = threadIdx.x;
    ExpertWork u = {}, dn = {};
    int items_up = 0, items_down = 0;
    if (i <= n + 1) plan.sync[i] = 0;
    if (i < n) {
        int rows, a_sel, a_idx, up_src, up_bsel, mid;
        if (i >= ns) {
            const int e = i - ns;
            rows = offs[e + 1] - offs[e];
            a_sel = 0; a_idx = e; up_src = offs[e]; up_bsel = 0; mid = offs[e];
        } else {
            rows = c.T;
            a_sel = 1; a_idx = i; up_src = 0; up_bsel = 1; mid = shared_row_base + i * c.T;
        }
    int bn, ntb;
        if (rows <= 0) {
            bn = 16; ntb = 0;
        } else if (rows <= kStreamRows) {
            bn = (rows + 15) & ~15; ntb = 1;
        } else {
            const int nt = (rows + max_tile - 1) / max_tile;
            bn = (((rows + nt - 1) / nt) + 15) & ~15;
            ntb = (rows + bn - 1) / bn;
        }
        u.rows = dn.rows = rows;
        u.a_sel = dn.a_sel = a_sel;
        u.a_idx = dn.a_idx = a_idx;
        u.bn = dn.bn = bn;
        u.ntb = dn.ntb = ntb;
        u.src_row0 = up_src; u.b_sel = up_bsel; u.dst_row0 = mid;
        dn.src_row0 = mid; dn.b_sel = 0; dn.dst_row0 = mid;
        items_up = ntb * fb_up;
        items_down = ntb * fb_down;
    }
    int tot_up, tot_down;
    const int pre_up = block_exclusive_scan_1024(items_up, wbuf, &tot_up);
    const int pre_down = block_exclusive_scan_1024(items_down, wbuf, &tot_down);
    if (i < n) {
        plan.up[i] = u;
        plan.down[i] = dn;
        plan.up_start[i] = pre_up;
        plan.down_start[i] = pre_down;
    }
    if (i == 0) {
        plan.up_start[n] = tot_up;
        plan.down_start[n] = tot_down;
    }
}

// Column sums of hist over tiles -> base (exclusive), counts, offsets;
// checks the equal group load; optionally writes the layer's GEMM plan.
// One block of 1024 threads.
__global__ void __launch_bounds__(1024) scan_kernel(moge_config c, const int32_t *__restrict__ hist,
                                                     int32_t *base, int32_t *counts,
                                                     int32_t *offsets, Plan plan, int make_plan,
                                                     int with_routed, int with_shared,
                                                     int max_tile) {
    __shared__ int32_t part[1024];
    __shared__ int32_t cnt_s[kMaxExperts];
    __shared__ int32_t off_s[kMaxExperts + 1];
    __shared__ int wbuf[32];
    grid_dependency_wait();
    const int N = c.N;
    const int tiles = (c.T + kRouterTile - 1) / kRouterTile;
    const int P = 1024 / N;  // chunks of tiles
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
    }
    __syncthreads();
    if (act) {
        int run = part[p * N + e];
        for (int t = tb; t < te; ++t) {
            base[(size_t)t * N + e] = run;
            run += hist[(size_t)t * N + e];
        }
    }
    const int v = threadIdx.x < N ? cnt_s[threadIdx.x] : 0;
    int total;
    const int pre = block_exclusive_scan_1024(v, wbuf, &total);
    if (threadIdx.x < N) {
        counts[threadIdx.x] = v;
        offsets[threadIdx.x] = pre;
        off_s[threadIdx.x] = pre;
    }
    if (threadIdx.x == 0) {
        offsets[N] = total;
        off_s[N] = total;
    }
    if (threadIdx.x < c.M) {  // every group carries exactly T*Kp assignments
        const int G = N / c.M;
        int lg = 0;
        for (int i = threadIdx.x * G; i < (threadIdx.x + 1) * G; ++i) lg += cnt_s[i];
        if (lg != c.T * c.Kp) raise_error(ERRBIT_INVARIANT);
    }
    if (make_plan) {
        __syncthreads();
        build_plan_block(c, off_s, plan, with_routed != 0, with_shared != 0, c.T * c.M * c.Kp,
                         max_tile, wbuf);
    }
}

cudaError_t launch_scan(const moge_config &c, const int32_t *hist, int32_t *base, int32_t *counts,
                        int32_t *offsets, const Plan *plan, bool with_routed, bool with_shared,
                        cudaStream_t st, int max_tile) {
    Plan p = plan ? *plan : Plan{nullptr, nullptr, nullptr, nullptr};
    return launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, c, hist, base, counts, offsets, p,
                      plan ? 1 : 0, with_routed ? 1 : 0, with_shared ? 1 : 0, max_tile);
}

// Plan from the caller's offsets (routed only) or for the shared experts only.
__global__ void __launch_bounds__(1024) plan_kernel(moge_config c, const int32_t *offsets, Plan plan,
                                                     int with_routed, int with_shared) {
    __shared__ int32_t off_s[kMaxExperts + 1];
    __shared__ int wbuf[32];
    grid_dependency_wait();
    if (with_routed)
        for (int i = threadIdx.x; i <= c.N; i += blockDim.x) off_s[i] = offsets[i];
    __syncthreads();
    build_plan_block(c, off_s, plan, with_routed != 0, with_shared != 0,
                     with_routed ? c.T * c.M * c.Kp : 0, kMaxTileN, wbuf);
}

cudaError_t launch_plan(const moge_config &c, const int32_t *offsets, const Plan &plan,
                        bool with_routed, bool with_shared, cudaStream_t st) {
    return launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, st, c, offsets, plan,
                      with_routed ? 1 : 0, with_shared ? 1 : 0);
}

// ---------------------------------------------------------------------------
// perm_dst[t][k] = offsets[e] + base[tile(t)][e] + rank[t][k];  perm_src[that] = t
__global__ void finalize_kernel(moge_config c, const int32_t *__restrict__ topk_idx,
                                const int32_t *__restrict__ rank, const int32_t *__restrict__ base,
                                const int32_t *__restrict__ offsets, int32_t *perm_src,
                                int32_t *perm_dst) {
    grid_dependency_wait();
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
    return launch_pdl(finalize_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st, c, topk_idx,
                      rank, base, offsets, perm_src, perm_dst);
}

}  // namespace moge
