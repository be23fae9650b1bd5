// Grouped SwiGLU expert FFN on the 5th-generation tensor cores (sm_100a).
//
// One persistent kernel runs both projections of every expert -- the
// up-projection (gate and up, SwiGLU epilogue, h rows out) and the
// down-projection (y rows out) -- one CTA per SM, warp-specialised:
//   warp 0    scheduler + TMA producer: takes work items from a global queue
//             (an atomic counter), publishes them to the other roles through
//             a small shared-memory ring, and streams their operands with TMA
//             (the copies of a stage issued by several lanes at once)
//   warp 1    MMA issuer   (tcgen05.mma kind::f16, M = 128, N = token tile,
//                           fp32 accumulators in TMEM, double-buffered)
//   warps 2-5 epilogue     (tcgen05.ld -> registers -> smem -> coalesced
//                           16-byte global stores, rows masked per expert;
//                           W8: warps 2-9, two per TMEM lane quarter)
//   warps 10-13 (W8 only)  h quantisers, on a queue of their own
//
// The queue hands out every up-projection item before any down-projection
// item, shared experts first (the heaviest items go first, the tail is made
// of small ones). A down-projection item of an expert waits -- bounded -- until
// all up-projection items of that expert have stored their h rows (a per-
// expert counter), so no kernel boundary separates the two phases. Every item
// it waits for was handed out earlier to a running CTA whose pipeline finishes
// it without waiting on anything, so the wait always ends.
//
// Orientation ("swap AB"): the weight tile is the MMA's M = 128 operand and the
// tokens of one expert are its N operand, N = 16 .. 256. A decode-sized expert
// (<= 64 rows) is one "streaming" tile: its weights are the HBM-bound stream,
// and every 48 KB pipeline stage carries two 64-wide K-chunks (32 KB of
// weights). Larger experts are split into token tiles of <= 256 rows
// ("tensor" tiles: one K-chunk per stage). The choice is made per expert from
// its token count, on the device.
//
// The up tile stacks 64 gate rows over the matching 64 up rows, fetched with
// one 16 KB copy from a 4-D tensor map that spans both weight tensors (or two
// 8 KB copies if the tensors overlap), so the accumulator lanes 0-63 hold gate
// and lanes 64-127 hold up for the same 64 features; the epilogue pairs them
// through shared memory. No repacking of the [E][I][d] weights is needed.
//
// W8A8 (the kernel's W8 instantiation): weights and activations are E4M3
// codes, and the MMA is kind::f8f6f4. A K-chunk is still 128 bytes per row (128
// codes), so the stages, boxes and descriptors keep their byte geometry. The
// scales are applied in the epilogue: the weight row's scale per accumulator
// lane and the token's scale per column. Each row of h needs its own scale,
// which depends on all of the row's I features, so the up-projection items
// store h in fp32 and fold each row's amax into a global word. Quantisation
// items -- kQParts row slices per token tile -- come from a second queue and
// run on four quantiser warps per CTA beside the GEMM roles, each once the
// expert's up items are all done, each counting once more on the expert's
// counter; the expert's down-projection items wait for those counts too. (Run
// by the CTA that finished an expert's last up item, quantisation chained:
// that CTA's delayed items made it the last finisher of the next expert, and
// so on; run on the epilogue warps, it stalled the GEMM pipeline.) The 8-bit
// MMA halves an item's time, so the W8 epilogue has eight warps and spreads
// the SwiGLU over all of them.
//
// The grouped expert GEMM ("GroupMatmul") of the Pangu Pro MoE article
// (techwalker.com, section 3) and its SwiftGMM GEMV/GEMM switch (reportify.cn
// product digest) are prior art for Ascend; this is a B200 design of the
// same operation.
#include <cuda_fp8.h>

#include "common.cuh"
#include "moge_internal.h"

namespace moge {

constexpr int kStages = 4;
constexpr int kStageBytes = 48 * 1024;
constexpr int kEpiBytes = 16 * 1024;  // U fp32 [32][64], H and G bf16 [32][64]
constexpr int kTcThreads = 192;
constexpr int kTcThreadsW8 = 448;    // warps 2-9 epilogue (two per TMEM lane quarter), 10-13 the h quantisers
constexpr int kChunkK = 64;          // bf16 elements per K-chunk (128 bytes, one swizzle row)
constexpr int kChunkK8 = 128;        // E4M3 elements per K-chunk (the same 128 bytes)
constexpr int kKSteps = 4;           // MMAs per K-chunk: 32 bytes of K each
constexpr int kBoxRows = 64;         // token rows per TMA box (one 8 KB copy per chunk)
constexpr uint32_t kTmemCols = 512;  // two accumulators of 256 columns
constexpr int kSlots = 8;            // depth of the work-item ring

// How the up-projection's 128-row weight tile is fetched, per weight side
// (routed / shared): one 16 KB copy from a 4-D map over both tensors when
// w_up lies wholly after w_gate (kGateUpFused) or wholly before it
// (kUpGateFused: the tile then holds up rows first), else two 8 KB copies.
enum : int { kGateUpSplit = 0, kGateUpFused = 1, kUpGateFused = 2 };

struct TcParams {
    int gu_mode[2];  // per a_sel
    Plan plan;
    int n_entries;
    int kc_up, kc_down;  // K-chunks of the two projections: ceil(d/64), ceil(I/64)
    int I, d;
    uint16_t *h;         // [rows][I]
    uint16_t *y;         // [rows][d]
    int *sync;           // [0] queue counter, [1 + e] finished up items of entry e
    uint16_t *gu;        // null, or [rows][2I]: the up-projection's g and u (training forward)
    // permute inside this launch (pm_topk_idx non-null): x (b1) -> x_perm (b0)
    const int32_t *pm_topk_idx, *pm_rank, *pm_base, *pm_offsets;
    int32_t *pm_perm_src, *pm_perm_dst;
    const uint4 *pm_x;
    uint4 *pm_x_perm;
    int pm_T, pm_N, pm_K;
};

// The W8A8 instantiation's extra operands (unused by the bf16 one).
struct W8Params {
    const float *sc_g[2], *sc_u[2], *sc_d[2];  // weight row scales, per a_sel
    const float *cs_b0, *cs_b1;  // token scales of the up-projection's B rows (b_sel 0 / 1)
    float *h32;                  // [rows][I] h in fp32, before quantisation
    uint32_t *hmax;              // [rows] amax of each h row (fp32 bits; zeroed beforehand)
    float *sh;                   // [rows] scale of each row of h codes
    uint8_t *h8;                 // [rows][I] h codes: the down-projection's B
};

struct TcItem {
    ExpertWork w;
    int entry, fb, tb, n_valid;
    bool up, stream;
    bool quant;  // W8: quantise part fb of token tile tb's h rows (no GEMM)
};

// W8: every token tile's h rows are quantised by kQParts work items (part p
// takes the tile's rows p, p + kQParts, ...), spread over the grid.
constexpr int kQParts = 16;

// Decode global item q: the up-projection items first, then (W8: tot_q > 0)
// the quantisation items, kQParts per token tile in entry order, then the
// down-projection items.
__device__ __forceinline__ void decode_item(const TcParams &p, int tot_up, int tot_q, int q,
                                            TcItem &it) {
    it.up = q < tot_up;
    it.quant = !it.up && q < tot_up + tot_q;
    const int fb_up = (p.I + 63) / 64;
    // a quantisation item is looked up as the first up item of its tile
    const int local = it.up ? q : it.quant ? ((q - tot_up) / kQParts) * fb_up : q - tot_up - tot_q;
    const int *start = (it.up || it.quant) ? p.plan.up_start : p.plan.down_start;
    int lo = 0, hi = p.n_entries - 1;
    while (lo < hi) {  // last entry whose first item is <= local (entries may be empty)
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(start + mid) <= local) lo = mid; else hi = mid - 1;
    }
    const int *wp =
        reinterpret_cast<const int *>(((it.up || it.quant) ? p.plan.up : p.plan.down) + lo);
    it.w.rows = __ldg(wp + 0);
    it.w.src_row0 = __ldg(wp + 1);
    it.w.dst_row0 = __ldg(wp + 2);
    it.w.a_sel = __ldg(wp + 3);
    it.w.a_idx = __ldg(wp + 4);
    it.w.b_sel = __ldg(wp + 5);
    it.w.bn = __ldg(wp + 6);
    it.w.ntb = __ldg(wp + 7);
    it.entry = lo;
    const int r = local - __ldg(start + lo);
    if (it.quant) {
        it.fb = (q - tot_up) % kQParts;
        it.tb = r / fb_up;
    } else {
        it.fb = r / it.w.ntb;  // feature block major, token tile fastest
        it.tb = r % it.w.ntb;
    }
    it.n_valid = min(it.w.bn, it.w.rows - it.tb * it.w.bn);
    it.stream = it.w.rows <= kStreamRows;
}

// K-chunk processed at step i of an item of feature block fb: items of the
// same expert run side by side and read the same token rows, so each feature
// block starts at a different chunk. The order is fixed per item, so results
// stay deterministic.
__device__ __forceinline__ int chunk_at(int i, int fb, int k_chunks) {
    const int r = (fb * 2 * 5) % k_chunks;  // even start: streaming pairs stay aligned
    const int c = i + r;
    return c >= k_chunks ? c - k_chunks : c;
}

struct TcShared {
    uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], drain;
    uint64_t slot_full[kSlots], slot_empty[kSlots];
    int slot_item[kSlots];
    uint32_t tmem_base;
    int abort;
    int epi_item;
    int pm_rows[kMaxExperts];  // the fused permute: destination rows of the current token
    float cs[kMaxTileN];       // W8: token scales of the current item's columns
    int q_item;                // W8: the quantisers' current item
};

// E4M3 codes of four fp32 values divided by s (IEEE fp32 division, then round
// to nearest even, saturating), packed low byte first.
__device__ __forceinline__ uint32_t e4m3x4_div(float4 f, float s) {
    const uint32_t b0 = __nv_cvt_float_to_fp8(__fdiv_rn(f.x, s), __NV_SATFINITE, __NV_E4M3);
    const uint32_t b1 = __nv_cvt_float_to_fp8(__fdiv_rn(f.y, s), __NV_SATFINITE, __NV_E4M3);
    const uint32_t b2 = __nv_cvt_float_to_fp8(__fdiv_rn(f.z, s), __NV_SATFINITE, __NV_E4M3);
    const uint32_t b3 = __nv_cvt_float_to_fp8(__fdiv_rn(f.w, s), __NV_SATFINITE, __NV_E4M3);
    return b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
}

// W8: quantise rows row0 + first, row0 + first + step, ... (tile-relative
// indices < n) of h (fp32 [.][I], I % 16 == 0), each with its own scale:
// amax / 448 (IEEE fp32 division; 1 for an all-zero row), code = E4M3 of
// fp32(h / scale). The 128 quantiser threads (et) take four rows at a time,
// every thread loading its vectors of all four before converting any. h and
// the amax words were written by other CTAs: read through L2 only.
__device__ void quantize_h_rows(const W8Params &w8, int I, size_t row0, int first, int step, int n,
                                int et) {
    const int nv = I / 4;  // 16-byte vectors per row
    for (int r = first; r < n; r += 4 * step) {
        size_t row[4];
        float sc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            row[j] = row0 + (size_t)(r + j * step);
            sc[j] = 1.0f;
            if (r + j * step < n) {
                const float amax = __uint_as_float(__ldcg(w8.hmax + row[j]));
                if (amax > 0.0f) sc[j] = __fdiv_rn(amax, 448.0f);
                if (et == 0) w8.sh[row[j]] = sc[j];
            }
        }
        for (int v0 = 0; v0 < nv; v0 += 3 * 128) {
            float4 f[4][3];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const int v = v0 + et + 128 * k;
                    if (r + j * step < n && v < nv)
                        f[j][k] = __ldcg(reinterpret_cast<const float4 *>(w8.h32 + row[j] * I) + v);
                }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const int v = v0 + et + 128 * k;
                    if (r + j * step < n && v < nv)
                        reinterpret_cast<uint32_t *>(w8.h8 + row[j] * I)[v] = e4m3x4_div(f[j][k], sc[j]);
                }
        }
    }
}

// smem byte offsets of chunk c of a stage
__device__ __forceinline__ uint32_t a_off(bool stream, int c) { return stream ? c * 24576u : 0u; }
__device__ __forceinline__ uint32_t b_off(bool stream, int c) {
    return stream ? c * 24576u + 16384u : 16384u;
}

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *ctr >= need (an up-projection's h rows of one expert).
// Gives up (records ERRBIT_TIMEOUT, sets *abort) after limit_ns, or at once
// when *abort is set; abort may be NULL.
__device__ bool wait_counter(const int *ctr, int need, volatile int *abort,
                             uint64_t limit_ns = kWaitTimeoutNs, uint32_t sleep_ns = 64) {
    if (ld_acquire(ctr) >= need) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(sleep_ns);
        if (ld_acquire(ctr) >= need) return true;
        if ((it & 63u) == 0) {
            if (abort && *abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                raise_error(ERRBIT_TIMEOUT);
                if (abort) *abort = 1;
                return false;
            }
        }
    }
}

template <bool W8>
__global__ void __launch_bounds__(W8 ? kTcThreadsW8 : kTcThreads, 1) ffn_tc_kernel(
    const __grid_constant__ TcParams p, const __grid_constant__ W8Params w8,
    const __grid_constant__ CUtensorMap tmWg,
    const __grid_constant__ CUtensorMap tmWu, const __grid_constant__ CUtensorMap tmSg,
    const __grid_constant__ CUtensorMap tmSu, const __grid_constant__ CUtensorMap tmX0,
    const __grid_constant__ CUtensorMap tmX1, const __grid_constant__ CUtensorMap tmWd,
    const __grid_constant__ CUtensorMap tmSd, const __grid_constant__ CUtensorMap tmH) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    unsigned char *stages = smem;
    unsigned char *epi = smem + kStages * kStageBytes;
    TcShared &sh = *reinterpret_cast<TcShared *>(epi + kEpiBytes);
    volatile int *abort = &sh.abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh.tfull[a], 1);
            mbar_init(&sh.tempty[a], W8 ? 256 : 128);  // every epilogue thread
        }
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&sh.slot_full[s], 1);
            mbar_init(&sh.slot_empty[s], 2);  // the MMA thread and the epilogue leader
        }
        mbar_init(&sh.drain, 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmWg);
        tma_prefetch_desc(&tmWu);
        tma_prefetch_desc(&tmSg);
        tma_prefetch_desc(&tmSu);
        tma_prefetch_desc(&tmX0);
        tma_prefetch_desc(&tmX1);
        tma_prefetch_desc(&tmWd);
        tma_prefetch_desc(&tmSd);
        tma_prefetch_desc(&tmH);
    }
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sh.tmem_base;
    // everything above overlapped the previous kernel; its results are needed from here on
    grid_dependency_wait();
    const int tot_up = __ldg(p.plan.up_start + p.n_entries);
    const int fb_up = (p.I + 63) / 64;
    // W8: kQParts quantisation items per token tile (every entry's up items
    // are its tiles x fb_up), taken from their own queue by warps 10-13
    const int tot_q = W8 ? kQParts * (tot_up / fb_up) : 0;
    const int total = tot_up + __ldg(p.plan.down_start + p.n_entries);
    constexpr int kCE = W8 ? kChunkK8 : kChunkK;  // elements per K-chunk

    if (warp == 0) {
        // ------------------------------------------------------ scheduler + producer
        // Lane 0 schedules and keeps the stage ring; the copies of a stage are
        // issued by several lanes at once (one copy per lane): a single thread
        // issuing them one after another cannot keep up with the tensor cores.
        const uint64_t pol_w = policy_evict_first();  // weights: read once
        const uint64_t pol_b = policy_evict_last();   // token / h rows: reused across feature blocks
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_par = 0;  // lane 0: per stage, a load issued / its parity
        int next = lane == 0 ? atomicAdd(p.sync, 1) : 0;
        bool permuted = p.pm_topk_idx == nullptr;  // x_perm complete (fused permute)
        for (int s = 0;; ++s) {
            const int slot = s % kSlots;
            int q = 0;
            if (lane == 0) {
                if (mbar_wait(&sh.slot_empty[slot], ((uint32_t)(s / kSlots) & 1u) ^ 1u, abort)) {
                    q = *abort ? total : next;
                    sh.slot_item[slot] = q;
                    mbar_arrive(&sh.slot_full[slot]);
                    if (q < total) next = atomicAdd(p.sync, 1);
                } else {
                    q = -1;
                }
            }
            q = __shfl_sync(0xffffffffu, q, 0);
            if (q < 0 || q >= total) break;
            TcItem it;
            decode_item(p, tot_up, 0, q, it);
            if (!it.up) {  // the h rows of this expert must all be stored (W8: and quantised)
                int ok = 1;
                if (lane == 0)
                    ok = wait_counter(p.sync + 1 + it.entry,
                                      it.w.ntb * (fb_up + (W8 ? kQParts : 0)), abort);
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                fence_proxy_async_global();
            } else if (it.w.b_sel == 0 && !permuted) {  // routed rows: every CTA's permute share
                int ok = 1;
                if (lane == 0) ok = wait_counter(p.sync + 1 + p.n_entries, (int)gridDim.x, abort);
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                fence_proxy_async_global();
                permuted = true;
            }
            const CUtensorMap *ma0, *ma1, *mb;
            if (it.up) {
                ma0 = it.w.a_sel ? &tmSg : &tmWg;
                ma1 = it.w.a_sel ? &tmSu : &tmWu;
                mb = it.w.b_sel ? &tmX1 : &tmX0;
            } else {
                ma0 = ma1 = it.w.a_sel ? &tmSd : &tmWd;
                mb = &tmH;
            }
            const int gu = p.gu_mode[it.w.a_sel];
            const int na = (it.up && gu == kGateUpSplit) ? 2 : 1;  // weight copies per chunk
            const int kcs = it.up ? p.kc_up : p.kc_down;
            const int per = it.stream ? 2 : 1;
            const int nbox = (it.w.bn + kBoxRows - 1) / kBoxRows;
            const int brow0 = it.w.src_row0 + it.tb * it.w.bn;
            const int arow0 = it.up ? it.fb * 64 : it.fb * 128;
            // this lane's copy in every stage: chunk c, copy r of that chunk
            const int ops = na + nbox;
            const int my_c = lane / ops, my_r = lane % ops;
            bool ok = true;
            for (int kc = 0; kc < kcs; kc += per) {
                int got = 1;
                if (lane == 0) got = mbar_wait(&sh.empty[stage], phase ^ 1u, abort);
                if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
                const int nch = min(per, kcs - kc);
                unsigned char *sbase = stages + stage * kStageBytes;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sh.full[stage],
                                          (uint32_t)nch * (16384u + (uint32_t)nbox * kBoxRows * 128u));
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                }
                __syncwarp();
                if (my_c < nch) {
                    const int k = chunk_at(kc + my_c, it.fb, kcs) * kCE;
                    unsigned char *sa = sbase + a_off(it.stream, my_c);
                    unsigned char *sb = sbase + b_off(it.stream, my_c);
                    if (my_r >= na) {
                        const int j = my_r - na;
                        tma_load_2d(sb + j * kBoxRows * 128, mb, &sh.full[stage], k,
                                    brow0 + j * kBoxRows, pol_b);
                    } else if (it.up && gu != kGateUpSplit) {
                        tma_load_4d(sa, ma0, &sh.full[stage], k, arow0, it.w.a_idx, 0, pol_w);
                    } else if (it.up) {
                        tma_load_3d(sa + 8192 * my_r, my_r ? ma1 : ma0, &sh.full[stage], k, arow0,
                                    it.w.a_idx, pol_w);
                    } else {
                        tma_load_3d(sa, ma0, &sh.full[stage], k, arow0, it.w.a_idx, pol_w);
                    }
                }
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
        if (lane == 0 && *abort) {  // let every issued copy land before the CTA can exit
            for (int s = 0; s < kStages; ++s)
                if (armed & (1u << s)) mbar_wait(&sh.full[s], (armed_par >> s) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int s = 0;; ++s) {
                const int slot = s % kSlots;
                if (!mbar_wait(&sh.slot_full[slot], (uint32_t)(s / kSlots) & 1u, abort)) break;
                const int q = sh.slot_item[slot];
                mbar_arrive(&sh.slot_empty[slot]);
                if (q >= total) break;
                TcItem it;
                decode_item(p, tot_up, 0, q, it);
                const int acc = s & 1;
                const uint32_t use = (uint32_t)(s >> 1);
                if (!mbar_wait(&sh.tempty[acc], (use & 1u) ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
                const uint32_t idesc = W8 ? idesc_e4m3_f32(128, (uint32_t)it.w.bn)
                                          : idesc_bf16_f32(128, (uint32_t)it.w.bn);
                const int kcs = it.up ? p.kc_up : p.kc_down;
                const int per = it.stream ? 2 : 1;
                bool ok = true;
                for (int kc = 0; kc < kcs; kc += per) {
                    if (!mbar_wait(&sh.full[stage], phase, abort)) { ok = false; break; }
                    tc_fence_after();
                    const int nch = min(per, kcs - kc);
                    const uint32_t sbase = smem_u32(stages + stage * kStageBytes);
                    for (int c = 0; c < nch; ++c) {
                        const uint32_t sa = sbase + a_off(it.stream, c);
                        const uint32_t sb = sbase + b_off(it.stream, c);
#pragma unroll
                        for (int j = 0; j < kKSteps; ++j) {  // K steps of 32 bytes
                            const uint64_t da = smem_desc_sw128(sa + 32u * j);
                            const uint64_t db = smem_desc_sw128(sb + 32u * j);
                            if constexpr (W8)
                                tc_mma_f8(d_tmem, da, db, idesc, (kc + c + j) > 0 ? 1u : 0u);
                            else
                                tc_mma_bf16(d_tmem, da, db, idesc, (kc + c + j) > 0 ? 1u : 0u);
                        }
                    }
                    tc_commit(&sh.empty[stage]);  // frees the stage once these MMAs have read it
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&sh.tfull[acc]);
            }
            tc_commit(&sh.drain);  // every MMA of this CTA has completed after this
            mbar_wait(&sh.drain, 0, nullptr);
        }
    } else if (W8 && warp >= 10) {
        // ------------------------------------------------------ h quantisers (W8)
        // Items from their own queue (sync[1 + n_entries]: no permute runs in
        // this launch), each once the up items of its expert are all done;
        // they run beside the GEMM roles instead of holding up the epilogue.
        const int qt = threadIdx.x - 10 * 32;  // 0 .. 127
        for (;;) {
            if (qt == 0) {
                int i = atomicAdd(p.sync + 1 + p.n_entries, 1);
                if (i < tot_q) {
                    TcItem lt;
                    decode_item(p, tot_up, tot_q, tot_up + i, lt);
                    // (polled sparsely: up to 148 CTAs may wait here at once)
                    if (!wait_counter(p.sync + 1 + lt.entry, lt.w.ntb * fb_up, abort,
                                      kWaitTimeoutNs, 512))
                        i = tot_q;
                }
                sh.q_item = i;
            }
            named_bar_sync(2, 128);
            const int i = *(volatile int *)&sh.q_item;
            named_bar_sync(2, 128);
            if (i >= tot_q) break;
            TcItem it;
            decode_item(p, tot_up, tot_q, tot_up + i, it);
            // rows fb, fb + kQParts, ... of the tile, then one count for the
            // expert's down-projection items
            quantize_h_rows(w8, p.I, (size_t)it.w.dst_row0 + (size_t)it.tb * it.w.bn, it.fb,
                            kQParts, it.n_valid, qt);
            fence_proxy_async_global();
            __threadfence();
            named_bar_sync(2, 128);
            if (qt == 0) atomicAdd(p.sync + 1 + it.entry, 1);
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int q4 = warp & 3;           // TMEM lane quarter this warp may read
        const int et = threadIdx.x - 64;   // 0 .. kEpi - 1
        // W8: eight epilogue warps, two per lane quarter, each taking 16 of
        // every 32 accumulator columns (the 8-bit MMA halves an item's time)
        constexpr int kEpi = W8 ? 256 : 128;
        const int eh = W8 ? (warp - 2) >> 2 : 0;
        if (p.pm_topk_idx) {
            // The permute, before this CTA's first accumulator exists: tokens
            // blockIdx.x, + gridDim.x, ...; each token's K destination rows
            // (expert offset + earlier tiles' rows + rank in its tile), then its
            // row copied into each. Published with a release for the routed
            // up-projection items, which read x_perm with TMA (async proxy).
            const int K = p.pm_K, nvec = p.d / 8;
            for (int t = blockIdx.x; t < p.pm_T; t += gridDim.x) {
                for (int k = et; k < K; k += 128) {
                    const size_t i = (size_t)t * K + k;
                    const int e = p.pm_topk_idx[i];
                    int row = -1;
                    if (e >= 0 && e < p.pm_N) {
                        row = p.pm_offsets[e] + p.pm_base[(size_t)(t / kRouterTile) * p.pm_N + e] +
                              p.pm_rank[i];
                        p.pm_perm_dst[i] = row;
                        p.pm_perm_src[row] = t;
                    } else {
                        raise_error(ERRBIT_INVARIANT);
                    }
                    sh.pm_rows[k] = row;
                }
                named_bar_sync(1, kEpi);
                for (int v = et; v < nvec; v += 128) {
                    const uint4 val = p.pm_x[(size_t)t * nvec + v];
                    for (int k = 0; k < K; ++k) {
                        const int row = sh.pm_rows[k];
                        if (row >= 0) p.pm_x_perm[(size_t)row * nvec + v] = val;
                    }
                }
                named_bar_sync(1, kEpi);
            }
            fence_proxy_async_global();
            __threadfence();
            named_bar_sync(1, kEpi);
            if (et == 0) atomicAdd(p.sync + 1 + p.n_entries, 1);
        }
        for (int s = 0;; ++s) {
            // the leader takes the next item and waits for its accumulator;
            // all epilogue threads then act on the same decision
            if (et == 0) {
                const int slot = s % kSlots;
                int q = -1;
                if (mbar_wait(&sh.slot_full[slot], (uint32_t)(s / kSlots) & 1u, abort)) {
                    q = sh.slot_item[slot];
                    mbar_arrive(&sh.slot_empty[slot]);
                    if (q < total && !mbar_wait(&sh.tfull[s & 1], (uint32_t)(s >> 1) & 1u, abort))
                        q = -1;
                }
                sh.epi_item = q;
            }
            named_bar_sync(1, kEpi);
            const int q = *(volatile int *)&sh.epi_item;
            named_bar_sync(1, kEpi);
            if (q < 0 || q >= total) break;
            tc_fence_after();
            TcItem it;
            decode_item(p, tot_up, 0, q, it);
            const int acc = s & 1;
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q4) << 16) + (uint32_t)acc * 256u;
            const size_t row0 = (size_t)it.w.dst_row0 + (size_t)it.tb * it.w.bn;
            // W8: the scale of this thread's accumulator row (its weight row)
            // and the token scales of the item's B rows
            float rs = 1.0f;
            const float *cs = nullptr;
            if constexpr (W8) {
                const int m = q4 * 32 + lane;
                if (it.up) {
                    const bool gate_hi = p.gu_mode[it.w.a_sel] == kUpGateFused;
                    const bool is_gate = (q4 < 2) != gate_hi;
                    const int f = it.fb * 64 + (m & 63);
                    const float *sc = is_gate ? w8.sc_g[it.w.a_sel] : w8.sc_u[it.w.a_sel];
                    rs = f < p.I ? __ldg(sc + (size_t)it.w.a_idx * p.I + f) : 0.0f;
                    cs = it.w.b_sel ? w8.cs_b1 : w8.cs_b0;
                } else {
                    const int f = it.fb * 128 + m;
                    rs = f < p.d ? __ldg(w8.sc_d[it.w.a_sel] + (size_t)it.w.a_idx * p.d + f) : 0.0f;
                    cs = w8.sh;
                }
                cs += (size_t)it.w.src_row0 + (size_t)it.tb * it.w.bn;
                // all of the item's token scales at once (h scales were written in
                // this launch: through L2); one load latency per item
                for (int j = et; j < it.n_valid; j += kEpi) sh.cs[j] = __ldcg(cs + j);
                named_bar_sync(1, kEpi);
            }
            for (int c0 = 0; c0 < it.n_valid; c0 += 32) {
                uint32_t v[32];
                if constexpr (W8)
                    tmem_ld_32x32b_x16(tbase + (uint32_t)(c0 + 16 * eh), v);
                else
                    tmem_ld_32x32b_x32(tbase + (uint32_t)c0, v);
                tmem_ld_wait();
                if constexpr (W8) {
                    if (it.up) {
                        // the scaled gate and up accumulators staged side by side,
                        // then every thread forms h for 16 of the block's 2048
                        // (column, feature) pairs (the 8-bit MMA leaves the epilogue
                        // half the time of a bf16 item, so the SwiGLU is spread over
                        // all four warps, with the fast exponential and division)
                        float *G = reinterpret_cast<float *>(epi);           // [32 cols][64 features]
                        float *U = reinterpret_cast<float *>(epi + 8192);    // [32 cols][64 features]
                        const bool gate_hi = p.gu_mode[it.w.a_sel] == kUpGateFused;
                        float *D = ((q4 < 2) != gate_hi) ? G : U;
                        const int f = (q4 & 1) * 32 + lane;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int cj = 16 * eh + j;
                            D[cj * 64 + f] = __uint_as_float(v[j]) * rs * sh.cs[c0 + cj];
                        }
                        named_bar_sync(1, kEpi);
                        // fp32 h rows out, and each row's amax over these 64 features
                        // folded into its global amax word (16 lanes per row)
                        for (int idx = et; idx < 32 * 16; idx += kEpi) {
                            const int r = idx >> 4, vv = idx & 15;
                            const int col = c0 + r, feat = it.fb * 64 + vv * 4;
                            const float4 g = *reinterpret_cast<const float4 *>(G + r * 64 + vv * 4);
                            const float4 u = *reinterpret_cast<const float4 *>(U + r * 64 + vv * 4);
                            float4 hv;
                            hv.x = __fdividef(g.x, 1.0f + __expf(-g.x)) * u.x;
                            hv.y = __fdividef(g.y, 1.0f + __expf(-g.y)) * u.y;
                            hv.z = __fdividef(g.z, 1.0f + __expf(-g.z)) * u.z;
                            hv.w = __fdividef(g.w, 1.0f + __expf(-g.w)) * u.w;
                            float mx = 0.0f;
                            if (col < it.n_valid && feat < p.I) {
                                *reinterpret_cast<float4 *>(w8.h32 + (row0 + col) * p.I + feat) = hv;
                                mx = fmaxf(fmaxf(fabsf(hv.x), fabsf(hv.y)),
                                           fmaxf(fabsf(hv.z), fabsf(hv.w)));
                            }
#pragma unroll
                            for (int o = 8; o > 0; o >>= 1)
                                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                            if (vv == 0 && col < it.n_valid && mx > 0.0f)
                                atomicMax(w8.hmax + row0 + col, __float_as_uint(mx));
                        }
                        named_bar_sync(1, kEpi);
                    } else {
                        uint16_t *Y = reinterpret_cast<uint16_t *>(epi);  // [32 cols][128 features]
                        const int f = q4 * 32 + lane;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int cj = 16 * eh + j;
                            Y[cj * 128 + f] = to_bf16_bits(__uint_as_float(v[j]) * rs * sh.cs[c0 + cj]);
                        }
                        named_bar_sync(1, kEpi);
                        for (int idx = et; idx < 32 * 16; idx += kEpi) {
                            const int r = idx >> 4, vv = idx & 15;
                            const int col = c0 + r, feat = it.fb * 128 + vv * 8;
                            if (col < it.n_valid && feat < p.d)
                                *reinterpret_cast<uint4 *>(p.y + (row0 + col) * p.d + feat) =
                                    *reinterpret_cast<const uint4 *>(Y + r * 128 + vv * 8);
                        }
                        named_bar_sync(1, kEpi);
                    }
                    continue;
                }
                if (it.up) {
                    float *U = reinterpret_cast<float *>(epi);                 // [32 cols][64 features]
                    uint16_t *H = reinterpret_cast<uint16_t *>(epi + 8192);    // [32 cols][64 features]
                    // lanes 0-63 hold gate and 64-127 up, or the reverse for an up-first tile
                    const bool gate_hi = p.gu_mode[it.w.a_sel] == kUpGateFused;
                    const bool is_gate = (q4 < 2) != gate_hi;
                    uint16_t *G = reinterpret_cast<uint16_t *>(epi + 12288);  // [32 cols][64 features]
                    const int f = (q4 & 1) * 32 + lane;
                    if (!is_gate) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) U[j * 64 + f] = __uint_as_float(v[j]);
                    }
                    named_bar_sync(1, kEpi);
                    if (is_gate) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float g = __uint_as_float(v[j]);
                            const float hv = g / (1.0f + expf(-g)) * U[j * 64 + f];
                            H[j * 64 + f] = to_bf16_bits(hv);
                            if (p.gu) G[j * 64 + f] = to_bf16_bits(g);
                        }
                    }
                    named_bar_sync(1, kEpi);
                    for (int idx = et; idx < 32 * 8; idx += kEpi) {
                        const int r = idx >> 3, vv = idx & 7;
                        const int col = c0 + r, feat = it.fb * 64 + vv * 8;
                        if (col < it.n_valid && feat < p.I) {
                            *reinterpret_cast<uint4 *>(p.h + (row0 + col) * p.I + feat) =
                                *reinterpret_cast<const uint4 *>(H + r * 64 + vv * 8);
                            if (p.gu) {  // keep g and u (bf16) for the backward pass
                                uint16_t *dst = p.gu + (row0 + col) * 2 * (size_t)p.I + feat;
                                *reinterpret_cast<uint4 *>(dst) =
                                    *reinterpret_cast<const uint4 *>(G + r * 64 + vv * 8);
                                const float *u8 = U + r * 64 + vv * 8;
                                *reinterpret_cast<uint4 *>(dst + p.I) =
                                    make_uint4(pack_bf16x2(u8[0], u8[1]), pack_bf16x2(u8[2], u8[3]),
                                               pack_bf16x2(u8[4], u8[5]), pack_bf16x2(u8[6], u8[7]));
                            }
                        }
                    }
                    named_bar_sync(1, kEpi);
                } else {
                    uint16_t *Y = reinterpret_cast<uint16_t *>(epi);  // [32 cols][128 features]
                    const int f = q4 * 32 + lane;
#pragma unroll
                    for (int j = 0; j < 32; ++j) Y[j * 128 + f] = to_bf16_bits(__uint_as_float(v[j]));
                    named_bar_sync(1, kEpi);
                    for (int idx = et; idx < 32 * 16; idx += kEpi) {
                        const int r = idx >> 4, vv = idx & 15;
                        const int col = c0 + r, feat = it.fb * 128 + vv * 8;
                        if (col < it.n_valid && feat < p.d)
                            *reinterpret_cast<uint4 *>(p.y + (row0 + col) * p.d + feat) =
                                *reinterpret_cast<const uint4 *>(Y + r * 128 + vv * 8);
                    }
                    named_bar_sync(1, kEpi);
                }
            }
            tc_fence_before();
            mbar_arrive(&sh.tempty[acc]);
            if (it.up) {
                // publish this item's h rows to the down-projection items of the expert
                fence_proxy_async_global();
                __threadfence();
                named_bar_sync(1, kEpi);
                if (et == 0) atomicAdd(p.sync + 1 + it.entry, 1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and the launch. Every map's box is 128 bytes wide:
// 64 bf16 elements, or 128 E4M3 codes (w8).
struct ElemType {
    uint64_t size;
    uint32_t chunk;
    CUtensorMapDataType dt;
};
static ElemType elem_type(bool w8) {
    return w8 ? ElemType{1, (uint32_t)kChunkK8, CU_TENSOR_MAP_DATA_TYPE_UINT8}
              : ElemType{2, (uint32_t)kChunkK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16};
}

// [experts][rows][cols] weights, box = [box_rows][one chunk] of one expert
static bool encode_weights(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                           uint64_t experts, uint32_t box_rows, bool w8 = false) {
    const ElemType et = elem_type(w8);
    const cuuint64_t dims[3] = {cols, rows, experts};
    const cuuint64_t strides[2] = {cols * et.size, cols * rows * et.size};
    const cuuint32_t box[3] = {et.chunk, box_rows, 1};
    return encode(m, base, 3, dims, strides, box, et.dt);
}

// [rows][cols] row matrix, box = [64 rows][one chunk]
static bool encode_rows(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                        bool w8 = false) {
    const ElemType et = elem_type(w8);
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * et.size};
    const cuuint32_t box[2] = {et.chunk, (cuuint32_t)kBoxRows};
    return encode(m, base, 2, dims, strides, box, et.dt);
}

// One map over both the gate and the up tensor ([E][rows][cols] each, dense):
// dims {cols, rows, E, 2}, the last dimension stepping from one tensor to the
// other, so a {64, 64, 1, 2} box is one 16 KB copy of 64 gate rows followed by
// the 64 matching up rows. Strides must increase, so this needs the two
// tensors not to overlap; the tensor at the lower address becomes the first
// half of the tile. Returns kGateUpSplit when they overlap (or on failure),
// and the caller then uses two 3-D maps.
static int encode_gate_up(CUtensorMap *m, const void *gate, const void *up, uint64_t cols,
                          uint64_t rows, uint64_t experts, bool w8 = false) {
    const ElemType et = elem_type(w8);
    const int64_t bytes = (int64_t)(cols * rows * experts * et.size);
    const int64_t delta = static_cast<const char *>(up) - static_cast<const char *>(gate);
    int mode;
    const void *base;
    if (delta >= bytes) {
        mode = kGateUpFused;
        base = gate;
    } else if (-delta >= bytes) {
        mode = kUpGateFused;
        base = up;
    } else {
        return kGateUpSplit;
    }
    const uint64_t step = (uint64_t)(delta >= 0 ? delta : -delta);
    if (step % 16 != 0 || step >= (1ull << 40)) return kGateUpSplit;
    const cuuint64_t dims[4] = {cols, rows, experts, 2};
    const cuuint64_t strides[3] = {cols * et.size, cols * rows * et.size, step};
    const cuuint32_t box[4] = {et.chunk, 64, 1, 2};
    return encode(m, base, 4, dims, strides, box, et.dt) ? mode : kGateUpSplit;
}

static size_t tc_smem_bytes() {
    return 1024 + (size_t)kStages * kStageBytes + kEpiBytes + sizeof(TcShared);
}

// Both instantiations: maps, parameters and the launch. w8: the weights are
// E4M3 codes with row scales (op.*_s), the B rows too (op.cs_b0 / cs_b1 their
// token scales), op.h receives the h codes and op.h32 / hmax / sh the rest.
static cudaError_t launch_ffn_tc_impl(bool w8, const moge_config &c, const Plan &plan,
                                      int n_entries, const FfnOperands &op, int num_sms,
                                      cudaStream_t st) {
    if (n_entries <= 0 || c.T <= 0) return cudaSuccess;
    const int N = c.N, S = c.S, d = c.d, I = c.I;
    // routed / shared weight tensors; a missing side borrows the other's
    // pointer so that its map is valid (no plan entry ever selects it)
    const void *wg = op.wg ? op.wg : op.sg, *wu = op.wu ? op.wu : op.su, *wd = op.wd ? op.wd : op.sd;
    const int ne = op.wg ? N : S;
    const void *sg = op.sg ? op.sg : wg, *su = op.su ? op.su : wu, *sd = op.sd ? op.sd : wd;
    const int ns = op.sg ? S : ne;
    const void *b0 = op.b0 ? op.b0 : op.b1, *b1 = op.b1 ? op.b1 : op.b0;
    const int64_t r0 = op.b0 ? op.b0_rows : op.b1_rows, r1 = op.b1 ? op.b1_rows : op.b0_rows;

    CUtensorMap mWg, mWu, mSg, mSu, mX0, mX1, mWd, mSd, mH;
    TcParams p;
    p.gu_mode[0] = encode_gate_up(&mWg, wg, wu, d, I, ne, w8);
    p.gu_mode[1] = encode_gate_up(&mSg, sg, su, d, I, ns, w8);
    if (p.gu_mode[0] != kGateUpSplit) mWu = mWg;
    else if (!encode_weights(&mWg, wg, d, I, ne, 64, w8) || !encode_weights(&mWu, wu, d, I, ne, 64, w8))
        return cudaErrorInvalidValue;
    if (p.gu_mode[1] != kGateUpSplit) mSu = mSg;
    else if (!encode_weights(&mSg, sg, d, I, ns, 64, w8) || !encode_weights(&mSu, su, d, I, ns, 64, w8))
        return cudaErrorInvalidValue;
    if (!encode_rows(&mX0, b0, d, (uint64_t)r0, w8) || !encode_rows(&mX1, b1, d, (uint64_t)r1, w8) ||
        !encode_weights(&mWd, wd, I, d, ne, 128, w8) || !encode_weights(&mSd, sd, I, d, ns, 128, w8) ||
        !encode_rows(&mH, op.h, I, (uint64_t)op.h_rows, w8))
        return cudaErrorInvalidValue;
    const int ce = w8 ? kChunkK8 : kChunkK;
    p.plan = plan;
    p.n_entries = n_entries;
    p.kc_up = (d + ce - 1) / ce;
    p.kc_down = (I + ce - 1) / ce;
    p.I = I;
    p.d = d;
    p.h = (uint16_t *)op.h;
    p.y = (uint16_t *)op.y;
    p.sync = plan.sync;
    p.gu = (uint16_t *)op.gu;
    p.pm_topk_idx = op.pm_topk_idx;
    p.pm_rank = op.pm_rank;
    p.pm_base = op.pm_base;
    p.pm_offsets = op.pm_offsets;
    p.pm_perm_src = op.pm_perm_src;
    p.pm_perm_dst = op.pm_perm_dst;
    p.pm_x = (const uint4 *)op.b1;
    p.pm_x_perm = (uint4 *)op.b0;
    p.pm_T = c.T;
    p.pm_N = c.N;
    p.pm_K = c.M * c.Kp;
    W8Params q = {};
    if (w8) {
        const float *wgs = op.wg ? op.wg_s : op.sg_s, *wus = op.wg ? op.wu_s : op.su_s,
                    *wds = op.wg ? op.wd_s : op.sd_s;
        q.sc_g[0] = wgs; q.sc_u[0] = wus; q.sc_d[0] = wds;
        q.sc_g[1] = op.sg ? op.sg_s : wgs;
        q.sc_u[1] = op.sg ? op.su_s : wus;
        q.sc_d[1] = op.sg ? op.sd_s : wds;
        q.cs_b0 = op.cs_b0 ? op.cs_b0 : op.cs_b1;
        q.cs_b1 = op.cs_b1 ? op.cs_b1 : op.cs_b0;
        q.h32 = static_cast<float *>(op.h32);
        q.hmax = op.hmax;
        q.sh = op.sh;
        q.h8 = static_cast<uint8_t *>(op.h);
    }

    const size_t smem = tc_smem_bytes();
    auto kern = w8 ? ffn_tc_kernel<true> : ffn_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(num_sms), dim3(w8 ? kTcThreadsW8 : kTcThreads), smem, st, p, q,
                      mWg, mWu, mSg, mSu,
                      mX0, mX1, mWd, mSd, mH);
}

cudaError_t launch_ffn_tc(const moge_config &c, const Plan &plan, int n_entries,
                          const FfnOperands &op, int num_sms, cudaStream_t st, cudaEvent_t mid) {
    (void)mid;
    return launch_ffn_tc_impl(false, c, plan, n_entries, op, num_sms, st);
}

cudaError_t launch_ffn_w8a8(const moge_config &c, const Plan &plan, int n_entries,
                            const FfnOperands &op, int num_sms, cudaStream_t st) {
    return launch_ffn_tc_impl(true, c, plan, n_entries, op, num_sms, st);
}

}  // namespace moge
