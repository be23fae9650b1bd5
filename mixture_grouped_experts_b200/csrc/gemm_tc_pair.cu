// Grouped SwiGLU expert FFN on the 5th-generation tensor cores (sm_100a).
//
// One persistent kernel runs both projections of every expert -- the
// up-projection (gate and up, SwiGLU epilogue, h rows out) and the
// down-projection (y rows out). CTAs work in pairs (clusters of 2) on the
// 2-SM tensor-core MMA (tcgen05.mma.cta_group::2, M = 256): each item is two
// weight tiles of 128 rows (one per CTA) against one token tile of N rows
// (each CTA stages N/2 of them): per CTA, 32 KB staged per 64-wide K-chunk of
// 128 x 256 MMA work, where a single-SM tile stages 48 KB. The up-projection
// can also keep g and u (bf16) for the backward pass. Warp roles in each CTA:
//   warp 0    TMA producer; in the leader CTA also the scheduler, which takes
//             work items from a global queue (an atomic counter) and publishes
//             them to both CTAs through small shared-memory rings
//   warp 1    MMA issuer (leader CTA only; fp32 accumulators in TMEM,
//             double-buffered, each CTA holding its 128 rows)
//   warps 2-5 epilogue (tcgen05.ld -> registers -> smem -> coalesced 16-byte
//             global stores, rows masked per expert)
//
// The queue hands out every up-projection item before any down-projection
// item, shared experts first (the heaviest items go first, the tail is made
// of small ones). A down-projection item of an expert waits -- bounded -- until
// all up-projection items of that expert have stored their h rows (a per-
// expert counter), so no kernel boundary separates the two phases. Every item
// it waits for was handed out earlier to a running CTA whose pipeline finishes
// it without waiting on anything, so the wait always ends.
//
// Orientation ("swap AB"): the weight tiles are the MMA's M operand and the
// tokens of one expert are its N operand, N = 16 .. 256 (token tiles of the
// plan). Every pipeline stage carries one 64-wide K-chunk: 16 KB of weights and
// up to 16 KB of token rows per CTA, six stages deep, which is what keeps the
// MMA fed across the loaded latency of L2 and HBM at 256 x 256 tiles. This
// kernel serves prefill-sized batches; the single-SM kernel, whose stages
// carry two chunks for small experts, serves decode.
//
// The up tile stacks 64 gate rows over the matching 64 up rows, fetched with
// one 16 KB copy from a 4-D tensor map that spans both weight tensors (or two
// 8 KB copies if the tensors overlap), so the accumulator lanes 0-63 hold gate
// and lanes 64-127 hold up for the same 64 features; the epilogue pairs them
// through shared memory. No repacking of the [E][I][d] weights is needed.
//
// The grouped expert GEMM ("GroupMatmul") of the Pangu Pro MoE article
// (techwalker.com, section 3) and its SwiftGMM GEMV/GEMM switch (reportify.cn
// product digest) are prior art for Ascend; this is a B200 design of the
// same operation.
#include "common.cuh"
#include "moge_internal.h"

namespace moge {
namespace pair {

constexpr int kStages = 6;
constexpr int kStageBytes = 32 * 1024;  // one K-chunk: 16 KB of weights, <= 16 KB of token rows
constexpr int kEpiBytes = 16 * 1024;  // G and U fp32 [32][64] (up), Y bf16 [32][128] (down)
constexpr int kTcThreads = 192;
constexpr int kChunkK = 64;          // bf16 elements per K-chunk (128 bytes, one swizzle row)
constexpr int kBoxRows = 64;         // token rows per TMA box (one 8 KB copy per chunk)
constexpr int kSmallBoxRows = 32;    // token rows per box when a CTA holds <= 32 rows
constexpr int kLargeBoxRows = 128;   // token rows per box when a CTA holds > 64 rows
constexpr uint32_t kTmemCols = 512;  // two accumulators of 256 columns
constexpr int kSlots = 8;            // depth of the work-item rings
constexpr uint16_t kPairMask = 0x3;  // both CTAs of the pair

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
    uint16_t *gu;        // [rows][2][I] g and u kept for the backward pass, or null
    int *sync;           // [0] queue counter, [1 + e] finished up-projection halves of entry e
};

struct TcShared {
    uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], drain;
    uint64_t slot_full[kSlots], slot_empty[kSlots];
    int slot_item[kSlots];
    uint32_t tmem_base;
    int abort;
    int epi_item;
    // items of each plan entry before it: up pairs (128 features) and down
    // pairs (256 output features) per token tile, computed by each CTA
    int start_up[2 * kMaxExperts + 1], start_down[2 * kMaxExperts + 1];
};

// A pair item: expert entry, weight-tile pair fp (this CTA's tile: 2 fp + rank),
// token tile tb of bn rows (this CTA stages rows [rank * bn/2, (rank+1) * bn/2)).
struct TcItem {
    ExpertWork w;
    int entry, fp, tb, n_valid;
    bool up;
};

// Decode global item q: the up-projection items first, then the down-projection ones.
__device__ __forceinline__ void decode_item(const TcParams &p, const TcShared &sh, int tot_up, int q,
                                            TcItem &it) {
    it.up = q < tot_up;
    const int local = it.up ? q : q - tot_up;
    const int *start = it.up ? sh.start_up : sh.start_down;
    int lo = 0, hi = p.n_entries - 1;
    while (lo < hi) {  // last entry whose first item is <= local (entries may be empty)
        const int mid = (lo + hi + 1) >> 1;
        if (start[mid] <= local) lo = mid; else hi = mid - 1;
    }
    const int *wp = reinterpret_cast<const int *>((it.up ? p.plan.up : p.plan.down) + lo);
    it.w.rows = __ldg(wp + 0);
    it.w.src_row0 = __ldg(wp + 1);
    it.w.dst_row0 = __ldg(wp + 2);
    it.w.a_sel = __ldg(wp + 3);
    it.w.a_idx = __ldg(wp + 4);
    it.w.b_sel = __ldg(wp + 5);
    it.w.bn = __ldg(wp + 6);
    it.w.ntb = __ldg(wp + 7);
    it.entry = lo;
    const int r = local - start[lo];
    it.fp = r / it.w.ntb;  // weight-tile pair major, token tile fastest
    it.tb = r % it.w.ntb;
    it.n_valid = min(it.w.bn, it.w.rows - it.tb * it.w.bn);
}

// K-chunk processed at step i of an item of weight-tile pair fp: items of the
// same expert run side by side and read the same token rows, so each pair
// starts at a different chunk. The order is fixed per item, so results stay
// deterministic.
__device__ __forceinline__ int chunk_at(int i, int fp, int k_chunks) {
    const int r = (fp * 10) % k_chunks;
    const int c = i + r;
    return c >= k_chunks ? c - k_chunks : c;
}

// Each stage holds one K-chunk per CTA: its 128 weight rows at offset 0, its
// half of the token rows at offset 16 KB.
constexpr uint32_t kBOff = 16384u;

// Token rows this CTA stages per chunk and the one TMA box that carries them
// (32, 64 or 128 rows; rows past the tile are loaded and never used).
__device__ __forceinline__ void b_boxes(int bn, int &half, int &nbox, int &box_rows) {
    half = bn >> 1;
    nbox = 1;
    box_rows = half <= kSmallBoxRows ? kSmallBoxRows : half <= kBoxRows ? kBoxRows : kLargeBoxRows;
}

__global__ void __launch_bounds__(kTcThreads, 1) ffn_tc_pair_kernel(
    const __grid_constant__ TcParams p, const __grid_constant__ CUtensorMap tmWg,
    const __grid_constant__ CUtensorMap tmWu, const __grid_constant__ CUtensorMap tmSg,
    const __grid_constant__ CUtensorMap tmSu, const __grid_constant__ CUtensorMap tmWd,
    const __grid_constant__ CUtensorMap tmSd, const __grid_constant__ CUtensorMap tmX0,
    const __grid_constant__ CUtensorMap tmX0s, const __grid_constant__ CUtensorMap tmX1,
    const __grid_constant__ CUtensorMap tmX1s, const __grid_constant__ CUtensorMap tmH,
    const __grid_constant__ CUtensorMap tmHs, const __grid_constant__ CUtensorMap tmX0l,
    const __grid_constant__ CUtensorMap tmX1l, const __grid_constant__ CUtensorMap tmHl) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    // 1024-byte alignment for the 128-byte swizzle atoms (same offsets in both CTAs)
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    unsigned char *stages = smem;
    unsigned char *epi = smem + kStages * kStageBytes;
    TcShared &sh = *reinterpret_cast<TcShared *>(epi + kEpiBytes);
    volatile int *abort = &sh.abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: leader of the pair, 1: peer
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full[s], 1);   // leader: armed by its producer, both CTAs' bytes
            mbar_init(&sh.empty[s], 1);  // both: the leader's MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh.tfull[a], 1);   // both: the leader's MMA commit
            mbar_init(&sh.tempty[a], 2);  // leader: one arrival per CTA's epilogue
        }
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&sh.slot_full[s], 1);   // both: the leader's scheduler
            mbar_init(&sh.slot_empty[s], 4);  // leader: its MMA + epilogue, the peer's producer + epilogue
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
        tma_prefetch_desc(&tmWd);
        tma_prefetch_desc(&tmSd);
        tma_prefetch_desc(&tmX0);
        tma_prefetch_desc(&tmX0s);
        tma_prefetch_desc(&tmX1);
        tma_prefetch_desc(&tmX1s);
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmHs);
        tma_prefetch_desc(&tmX0l);
        tma_prefetch_desc(&tmX1l);
        tma_prefetch_desc(&tmHl);
    }
    if (warp == 1) {
        tmem_alloc_pair(&sh.tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers are initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = sh.tmem_base;
    // everything above overlapped the previous kernel; its results are needed from here on
    grid_dependency_wait();
    const int up_pairs = (p.I + 127) / 128;   // weight-tile pairs of one up-projection token tile
    const int down_pairs = (p.d + 255) / 256;  // and of one down-projection token tile
    if (warp == 2) {  // prefix sums of the token tiles, 32 entries at a time
        int base = 0;
        for (int e0 = 0; e0 < p.n_entries; e0 += 32) {
            const int e = e0 + lane;
            const int ntb = e < p.n_entries ? __ldg(&p.plan.up[e].ntb) : 0;
            int v = ntb;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += t;
            }
            if (e < p.n_entries) {
                sh.start_up[e] = up_pairs * (base + v - ntb);
                sh.start_down[e] = down_pairs * (base + v - ntb);
            }
            base += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) {
            sh.start_up[p.n_entries] = up_pairs * base;
            sh.start_down[p.n_entries] = down_pairs * base;
        }
    }
    __syncthreads();
    const int tot_up = sh.start_up[p.n_entries];
    const int total = tot_up + sh.start_down[p.n_entries];
    // shared::cluster addresses in the leader CTA
    const uint32_t lead_slot_empty = mapa_shared(&sh.slot_empty[0], 0);
    const uint32_t lead_tempty = mapa_shared(&sh.tempty[0], 0);
    const uint32_t lead_full = mapa_shared(&sh.full[0], 0);

    if (warp == 0) {
        // ------------------------------------------------------ producer (+ scheduler)
        // Lane 0 of the leader schedules; lane 0 keeps the stage ring; the
        // copies of a stage are issued by several lanes at once.
        // weight tiles are read by every token tile of their expert (2 to 16
        // here), token and h rows by every weight-tile pair: both kept in L2
        // (measured: evict_first on the weights re-reads ~1 GB more from DRAM
        // at prefill and costs ~5 % of the kernel's time)
        const uint64_t pol_w = policy_evict_last();
        const uint64_t pol_b = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_par = 0;  // leader lane 0: per stage, armed / its parity
        int next = (leader && lane == 0) ? atomicAdd(p.sync, 1) : 0;
        for (int s = 0;; ++s) {
            const int slot = s % kSlots;
            const uint32_t sp = (uint32_t)(s / kSlots) & 1u;
            int q = 0;
            if (lane == 0) {
                if (leader) {
                    if (mbar_wait_cluster(&sh.slot_empty[slot], sp ^ 1u, abort)) {
                        q = *abort ? total : next;
                        if (q < total) {
                            TcItem it0;
                            decode_item(p, sh, tot_up, q, it0);
                            // a down-projection item needs all h rows of its expert
                            if (!it0.up &&
                                !wait_counter(p.sync + 1 + it0.entry, it0.w.ntb * up_pairs * 2, abort))
                                q = total;
                        }
                        sh.slot_item[slot] = q;
                        st_shared_remote(mapa_shared(&sh.slot_item[slot], 1), q);
                        mbar_arrive(&sh.slot_full[slot]);
                        mbar_arrive_remote(mapa_shared(&sh.slot_full[slot], 1));
                        if (q < total) next = atomicAdd(p.sync, 1);
                    } else {
                        q = -1;
                    }
                } else {
                    if (mbar_wait_cluster(&sh.slot_full[slot], sp, abort)) {
                        q = sh.slot_item[slot];
                        mbar_arrive_remote(lead_slot_empty + 8u * slot);
                    } else {
                        q = -1;
                    }
                }
            }
            q = __shfl_sync(0xffffffffu, q, 0);
            if (q < 0 || q >= total) break;
            TcItem it;
            decode_item(p, sh, tot_up, q, it);
            if (!it.up) fence_proxy_async_global();  // h rows written by other CTAs
            const CUtensorMap *ma0, *ma1, *mb;
            int half, nbox, box_rows;
            b_boxes(it.w.bn, half, nbox, box_rows);
            if (it.up) {
                ma0 = it.w.a_sel ? &tmSg : &tmWg;
                ma1 = it.w.a_sel ? &tmSu : &tmWu;
                mb = it.w.b_sel ? (box_rows == kSmallBoxRows ? &tmX1s : box_rows == kBoxRows ? &tmX1 : &tmX1l)
                                : (box_rows == kSmallBoxRows ? &tmX0s : box_rows == kBoxRows ? &tmX0 : &tmX0l);
            } else {
                ma0 = ma1 = it.w.a_sel ? &tmSd : &tmWd;
                mb = box_rows == kSmallBoxRows ? &tmHs : box_rows == kBoxRows ? &tmH : &tmHl;
            }
            const int gu = p.gu_mode[it.w.a_sel];
            const int na = (it.up && gu == kGateUpSplit) ? 2 : 1;
            const int kcs = it.up ? p.kc_up : p.kc_down;
            const int tile = 2 * it.fp + (int)rank;  // this CTA's weight tile
            const int brow0 = it.w.src_row0 + it.tb * it.w.bn + (int)rank * half;
            const int arow0 = it.up ? tile * 64 : tile * 128;
            const uint32_t bytes_cta = 16384u + (uint32_t)nbox * box_rows * 128u;
            const int ops = na + nbox;
            bool ok = true;
            for (int kc = 0; kc < kcs; ++kc) {
                int got = 1;
                if (lane == 0) got = mbar_wait(&sh.empty[stage], phase ^ 1u, abort);
                if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
                unsigned char *sbase = stages + stage * kStageBytes;
                const uint32_t bar = lead_full + 8u * stage;
                if (leader && lane == 0) {
                    mbar_arrive_expect_tx(&sh.full[stage], 2u * bytes_cta);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                }
                __syncwarp();
                if (lane < ops) {
                    const int my_r = lane;
                    const int k = chunk_at(kc, it.fp, kcs) * kChunkK;
                    unsigned char *sa = sbase;
                    unsigned char *sb = sbase + kBOff;
                    if (my_r >= na) {
                        tma_load_2d_pair(sb, mb, bar, k, brow0, pol_b);
                    } else if (it.up && gu != kGateUpSplit) {
                        tma_load_4d_pair(sa, ma0, bar, k, arow0, it.w.a_idx, 0, pol_w);
                    } else if (it.up) {
                        tma_load_3d_pair(sa + 8192 * my_r, my_r ? ma1 : ma0, bar, k, arow0,
                                         it.w.a_idx, pol_w);
                    } else {
                        tma_load_3d_pair(sa, ma0, bar, k, arow0, it.w.a_idx, pol_w);
                    }
                }
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
        if (leader && lane == 0 && *abort) {  // let every issued copy (both CTAs') land before exit
            for (int s = 0; s < kStages; ++s)
                if (armed & (1u << s)) mbar_wait(&sh.full[s], (armed_par >> s) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            for (int s = 0;; ++s) {
                const int slot = s % kSlots;
                if (!mbar_wait(&sh.slot_full[slot], (uint32_t)(s / kSlots) & 1u, abort)) break;
                const int q = sh.slot_item[slot];
                mbar_arrive(&sh.slot_empty[slot]);
                if (q >= total) break;
                TcItem it;
                decode_item(p, sh, tot_up, q, it);
                const int acc = s & 1;
                const uint32_t use = (uint32_t)(s >> 1);
                if (!mbar_wait_cluster(&sh.tempty[acc], (use & 1u) ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
                const uint32_t idesc = idesc_bf16_f32(256, (uint32_t)it.w.bn);
                const int kcs = it.up ? p.kc_up : p.kc_down;
                bool ok = true;
                for (int kc = 0; kc < kcs; ++kc) {
                    if (!mbar_wait(&sh.full[stage], phase, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(stages + stage * kStageBytes);
                    const uint32_t sb = sa + kBOff;
#pragma unroll
                    for (int j = 0; j < kChunkK / 16; ++j)  // 16-wide K steps: +32 bytes
                        tc_mma_bf16_pair(d_tmem, smem_desc_sw128(sa + 32u * j),
                                         smem_desc_sw128(sb + 32u * j), idesc,
                                         (kc + j) > 0 ? 1u : 0u);
                    tc_commit_pair(&sh.empty[stage], kPairMask);  // frees the stage in both CTAs
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair(&sh.tfull[acc], kPairMask);
            }
            tc_commit_pair(&sh.drain, 0x1);  // every pair MMA of this CTA has completed after this
            mbar_wait(&sh.drain, 0, nullptr);
        }
    } else {
        // ------------------------------------------------------ epilogue (both CTAs)
        const int q4 = warp & 3;           // TMEM lane quarter this warp may read
        const int et = threadIdx.x - 64;   // 0 .. 127
        for (int s = 0;; ++s) {
            // the leader thread takes the next item and waits for its accumulator;
            // all 128 threads then act on the same decision
            if (et == 0) {
                const int slot = s % kSlots;
                int q = -1;
                if (mbar_wait_cluster(&sh.slot_full[slot], (uint32_t)(s / kSlots) & 1u, abort)) {
                    q = sh.slot_item[slot];
                    if (leader) mbar_arrive(&sh.slot_empty[slot]);
                    else mbar_arrive_remote(lead_slot_empty + 8u * slot);
                    if (q < total && !mbar_wait(&sh.tfull[s & 1], (uint32_t)(s >> 1) & 1u, abort))
                        q = -1;
                }
                sh.epi_item = q;
            }
            named_bar_sync(1, 128);
            const int q = *(volatile int *)&sh.epi_item;
            named_bar_sync(1, 128);
            if (q < 0 || q >= total) break;
            tc_fence_after();
            TcItem it;
            decode_item(p, sh, tot_up, q, it);
            const int acc = s & 1;
            const int tile = 2 * it.fp + (int)rank;  // this CTA's 128 accumulator rows
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q4) << 16) + (uint32_t)acc * 256u;
            const size_t row0 = (size_t)it.w.dst_row0 + (size_t)it.tb * it.w.bn;
            for (int c0 = 0; c0 < it.n_valid; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + (uint32_t)c0, v);
                tmem_ld_wait();
                if (it.up) {
                    // the gate and up accumulators staged side by side (fp32), then
                    // every thread forms h for 16 of the block's 2048 (column,
                    // feature) pairs: the SwiGLU spread over all four warps, with the
                    // fast exponential and division (half the warps doing all of it
                    // held the accumulator up: the MMA thread waited for it)
                    float *G = reinterpret_cast<float *>(epi);         // [32 cols][64 features]
                    float *U = reinterpret_cast<float *>(epi + 8192);  // [32 cols][64 features]
                    // lanes 0-63 hold gate and 64-127 up, or the reverse for an up-first tile
                    const bool gate_hi = p.gu_mode[it.w.a_sel] == kUpGateFused;
                    float *D = ((q4 < 2) != gate_hi) ? G : U;
                    const int f = (q4 & 1) * 32 + lane;
#pragma unroll
                    for (int j = 0; j < 32; ++j) D[j * 64 + f] = __uint_as_float(v[j]);
                    named_bar_sync(1, 128);
                    for (int idx = et; idx < 32 * 8; idx += 128) {
                        const int r = idx >> 3, vv = idx & 7;
                        const int col = c0 + r, feat = tile * 64 + vv * 8;
                        if (col < it.n_valid && feat < p.I) {
                            const float4 *g4 = reinterpret_cast<const float4 *>(G + r * 64 + vv * 8);
                            const float4 *u4 = reinterpret_cast<const float4 *>(U + r * 64 + vv * 8);
                            const float4 ga = g4[0], gb = g4[1], ua = u4[0], ub = u4[1];
                            const float g8[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                            const float u8[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
                            float h8[8];
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                h8[k] = __fdividef(g8[k], 1.0f + __expf(-g8[k])) * u8[k];
                            *reinterpret_cast<uint4 *>(p.h + (row0 + col) * p.I + feat) =
                                make_uint4(pack_bf16x2(h8[0], h8[1]), pack_bf16x2(h8[2], h8[3]),
                                           pack_bf16x2(h8[4], h8[5]), pack_bf16x2(h8[6], h8[7]));
                            if (p.gu) {  // keep g and u (bf16) for the backward pass
                                uint16_t *dst = p.gu + (row0 + col) * 2 * (size_t)p.I + feat;
                                *reinterpret_cast<uint4 *>(dst) =
                                    make_uint4(pack_bf16x2(g8[0], g8[1]), pack_bf16x2(g8[2], g8[3]),
                                               pack_bf16x2(g8[4], g8[5]), pack_bf16x2(g8[6], g8[7]));
                                *reinterpret_cast<uint4 *>(dst + p.I) =
                                    make_uint4(pack_bf16x2(u8[0], u8[1]), pack_bf16x2(u8[2], u8[3]),
                                               pack_bf16x2(u8[4], u8[5]), pack_bf16x2(u8[6], u8[7]));
                            }
                        }
                    }
                    named_bar_sync(1, 128);
                } else {
                    uint16_t *Y = reinterpret_cast<uint16_t *>(epi);  // [32 cols][128 features]
                    const int f = q4 * 32 + lane;
#pragma unroll
                    for (int j = 0; j < 32; ++j) Y[j * 128 + f] = to_bf16_bits(__uint_as_float(v[j]));
                    named_bar_sync(1, 128);
                    for (int idx = et; idx < 32 * 16; idx += 128) {
                        const int r = idx >> 4, vv = idx & 15;
                        const int col = c0 + r, feat = tile * 128 + vv * 8;
                        if (col < it.n_valid && feat < p.d)
                            *reinterpret_cast<uint4 *>(p.y + (row0 + col) * p.d + feat) =
                                *reinterpret_cast<const uint4 *>(Y + r * 128 + vv * 8);
                    }
                    named_bar_sync(1, 128);
                }
            }
            // every thread's TMEM reads are complete: give the accumulator back
            tc_fence_before();
            if (it.up) {  // and make this CTA's h rows visible to the down-projection items
                fence_proxy_async_global();
                __threadfence();
            }
            named_bar_sync(1, 128);
            if (et == 0) {
                if (leader) mbar_arrive(&sh.tempty[acc]);
                else mbar_arrive_remote(lead_tempty + 8u * acc);
                if (it.up) atomicAdd(p.sync + 1 + it.entry, 1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no CTA of the pair touches the other's shared memory or TMEM any more
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and the launch. The weight maps (encode_weights,
// encode_gate_up) and the bounded counter wait are the single-SM kernel's;
// token-row maps here take the box height.
// bf16 [rows][cols] row matrix, box = [box_rows][64 cols]
static bool encode_rows(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                        uint32_t box_rows) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kChunkK, box_rows};
    return encode(m, base, 2, dims, strides, box);
}

static size_t tc_smem_bytes() {
    return 1024 + (size_t)kStages * kStageBytes + kEpiBytes + sizeof(TcShared);
}

cudaError_t launch_ffn_tc_pair(const moge_config &c, const Plan &plan, int n_entries,
                               const FfnOperands &op, int num_sms, cudaStream_t st) {
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

    CUtensorMap mWg, mWu, mSg, mSu, mWd, mSd, mX0, mX0s, mX1, mX1s, mH, mHs, mX0l, mX1l, mHl;
    TcParams p;
    p.gu_mode[0] = encode_gate_up(&mWg, wg, wu, d, I, ne);
    p.gu_mode[1] = encode_gate_up(&mSg, sg, su, d, I, ns);
    if (p.gu_mode[0] != kGateUpSplit) mWu = mWg;
    else if (!encode_weights(&mWg, wg, d, I, ne, 64) || !encode_weights(&mWu, wu, d, I, ne, 64))
        return cudaErrorInvalidValue;
    if (p.gu_mode[1] != kGateUpSplit) mSu = mSg;
    else if (!encode_weights(&mSg, sg, d, I, ns, 64) || !encode_weights(&mSu, su, d, I, ns, 64))
        return cudaErrorInvalidValue;
    if (!encode_weights(&mWd, wd, I, d, ne, 128) || !encode_weights(&mSd, sd, I, d, ns, 128) ||
        !encode_rows(&mX0, b0, d, (uint64_t)r0, kBoxRows) ||
        !encode_rows(&mX0s, b0, d, (uint64_t)r0, kSmallBoxRows) ||
        !encode_rows(&mX1, b1, d, (uint64_t)r1, kBoxRows) ||
        !encode_rows(&mX1s, b1, d, (uint64_t)r1, kSmallBoxRows) ||
        !encode_rows(&mH, op.h, I, (uint64_t)op.h_rows, kBoxRows) ||
        !encode_rows(&mHs, op.h, I, (uint64_t)op.h_rows, kSmallBoxRows) ||
        !encode_rows(&mX0l, b0, d, (uint64_t)r0, kLargeBoxRows) ||
        !encode_rows(&mX1l, b1, d, (uint64_t)r1, kLargeBoxRows) ||
        !encode_rows(&mHl, op.h, I, (uint64_t)op.h_rows, kLargeBoxRows))
        return cudaErrorInvalidValue;
    p.plan = plan;
    p.n_entries = n_entries;
    p.kc_up = (d + kChunkK - 1) / kChunkK;
    p.kc_down = (I + kChunkK - 1) / kChunkK;
    p.I = I;
    p.d = d;
    p.h = (uint16_t *)op.h;
    p.y = (uint16_t *)op.y;
    p.gu = (uint16_t *)op.gu;
    p.sync = plan.sync;

    const size_t smem = tc_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(ffn_tc_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM, in pairs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(num_sms / 2 * 2));
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, ffn_tc_pair_kernel, p, mWg, mWu, mSg, mSu, mWd, mSd, mX0, mX0s, mX1,
                              mX1s, mH, mHs, mX0l, mX1l, mHl);
}

}  // namespace pair
}  // namespace moge
