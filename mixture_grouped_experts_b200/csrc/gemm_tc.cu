// Grouped SwiGLU expert FFN on the 5th-generation tensor cores (sm_100a).
//
// One persistent kernel per projection (up: gate+up with the SwiGLU epilogue,
// down: plain), one CTA per SM, warp-specialised:
//   warp 0   TMA producer   (weights: 3-D tensor maps over [E][rows][K],
//                             tokens: 2-D maps over the row matrices)
//   warp 1   MMA issuer     (tcgen05.mma kind::f16, M = 128, N = token tile,
//                             fp32 accumulators in TMEM, double-buffered)
//   warps 2-5 epilogue      (tcgen05.ld -> registers -> smem -> coalesced
//                             16-byte global stores, rows masked per expert)
//
// Orientation ("swap AB"): the weight tile is the MMA's M = 128 operand and the
// tokens of one expert are its N operand, N = 16 .. 256. A decode-sized expert
// (<= 64 rows) is one "streaming" tile: its weight rows are the HBM-bound
// stream, so every pipeline stage carries two 64-wide K-chunks (32 KB of
// weights) to keep more bytes in flight. Larger experts are split into token
// tiles of <= 256 rows ("tensor" tiles: one K-chunk per stage, compute-bound).
// The choice is made per expert from its token count, on the device.
//
// The up tile stacks 64 gate rows over the matching 64 up rows (two TMA boxes
// into one 128-row operand), so the accumulator lanes 0-63 hold gate and lanes
// 64-127 hold up for the same 64 features; the epilogue pairs them through
// shared memory. This needs no repacking of the [E][I][d] weights.
//
// The grouped expert GEMM ("GroupMatmul") of the Pangu Pro MoE article
// (techwalker.com, section 3) and its SwiftGMM GEMV/GEMM switch (reportify.cn
// product digest) are prior art for Ascend; this is a B200 design of the
// same operation.
#include "common.cuh"
#include "moge_internal.h"

namespace moge {

constexpr int kStages = 4;
constexpr int kStageBytes = 48 * 1024;
constexpr int kEpiBytes = 12 * 1024;
constexpr int kTcThreads = 192;
constexpr int kChunkK = 64;          // bf16 elements per K-chunk (128 bytes, one swizzle row)
constexpr int kBoxRows = 64;         // token rows per TMA box (one 8 KB copy per chunk)
constexpr uint32_t kTmemCols = 512;  // two accumulators of 256 columns

// How the up-projection's 128-row weight tile is fetched, per weight side
// (routed / shared): one 16 KB copy from a 4-D map over both tensors when
// w_up lies wholly after w_gate (kGateUpFused) or wholly before it
// (kUpGateFused: the tile then holds up rows first), else two 8 KB copies.
enum : int { kGateUpSplit = 0, kGateUpFused = 1, kUpGateFused = 2 };

struct TcParams {
    int gu_mode[2];  // per a_sel
    const ExpertWork *work;
    const int *item_start;
    int n_entries;
    int k_chunks;  // ceil(K / 64)
    int out_cols;  // I (up) or d (down): valid output features
    uint16_t *out; // h (up) or y_perm (down), row stride out_cols
};

struct TcItem {
    ExpertWork w;
    int fb, tb, n_valid;
    bool stream;
};

__device__ __forceinline__ void decode_item(const TcParams &p, int item, TcItem &it) {
    int lo = 0, hi = p.n_entries - 1;
    while (lo < hi) {  // last entry whose first item is <= item (entries may be empty)
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.item_start + mid) <= item) lo = mid; else hi = mid - 1;
    }
    const int *wp = reinterpret_cast<const int *>(p.work + lo);
    it.w.rows = __ldg(wp + 0);
    it.w.src_row0 = __ldg(wp + 1);
    it.w.dst_row0 = __ldg(wp + 2);
    it.w.a_sel = __ldg(wp + 3);
    it.w.a_idx = __ldg(wp + 4);
    it.w.b_sel = __ldg(wp + 5);
    it.w.bn = __ldg(wp + 6);
    it.w.ntb = __ldg(wp + 7);
    const int local = item - __ldg(p.item_start + lo);
    it.fb = local / it.w.ntb;  // feature block major, token tile fastest
    it.tb = local % it.w.ntb;
    it.n_valid = min(it.w.bn, it.w.rows - it.tb * it.w.bn);
    it.stream = it.w.rows <= kStreamRows;
}

struct TcShared {
    uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    int abort;
    int epi_ok;
};

// K-chunk processed at step i of an item of feature block fb: items of the
// same expert run side by side and read the same token rows, so each feature
// block starts at a different chunk (an L2 hot spot otherwise). The order is
// fixed per item, so results stay deterministic.
__device__ __forceinline__ int chunk_at(int i, int fb, int k_chunks) {
    const int r = (fb * 2 * 5) % k_chunks;  // even start: streaming pairs stay aligned
    const int c = i + r;
    return c >= k_chunks ? c - k_chunks : c;
}

// smem byte offsets of chunk c of a stage
__device__ __forceinline__ uint32_t a_off(bool stream, int c) { return stream ? c * 24576u : 0u; }
__device__ __forceinline__ uint32_t b_off(bool stream, int c) {
    return stream ? c * 24576u + 16384u : 16384u;
}

template <bool UP>
__global__ void __launch_bounds__(kTcThreads, 1) ffn_tc_kernel(
    TcParams p, const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
    const __grid_constant__ CUtensorMap tmS0, const __grid_constant__ CUtensorMap tmS1,
    const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    unsigned char *stages = smem;
    unsigned char *epi = smem + kStages * kStageBytes;
    TcShared &sh = *reinterpret_cast<TcShared *>(epi + kEpiBytes);
    volatile int *abort = &sh.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = __ldg(p.item_start + p.n_entries);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh.tfull[a], 1);
            mbar_init(&sh.tempty[a], 128);
        }
        mbar_init(&sh.drain, 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA0);
        tma_prefetch_desc(&tmS0);
        tma_prefetch_desc(&tmB0);
        if (UP) {
            tma_prefetch_desc(&tmA1);
            tma_prefetch_desc(&tmS1);
            tma_prefetch_desc(&tmB1);
        }
    }
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sh.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();  // weights: read once
            const uint64_t pol_b = policy_evict_last();   // token rows: reused by every feature block
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_par = 0;  // per stage: a load issued / its parity
            for (int item = blockIdx.x; item < total && !*abort; item += gridDim.x) {
                TcItem it;
                decode_item(p, item, it);
                const CUtensorMap *ma0 = it.w.a_sel ? &tmS0 : &tmA0;
                const CUtensorMap *ma1 = it.w.a_sel ? &tmS1 : &tmA1;
                const CUtensorMap *mb = it.w.b_sel ? &tmB1 : &tmB0;
                const int per = it.stream ? 2 : 1;
                const int nbox = (it.w.bn + kBoxRows - 1) / kBoxRows;
                const int brow0 = it.w.src_row0 + it.tb * it.w.bn;
                const int arow0 = UP ? it.fb * 64 : it.fb * 128;
                bool ok = true;
                for (int kc = 0; kc < p.k_chunks; kc += per) {
                    if (!mbar_wait(&sh.empty[stage], phase ^ 1u, abort)) { ok = false; break; }
                    const int nch = min(per, p.k_chunks - kc);
                    unsigned char *sbase = stages + stage * kStageBytes;
                    mbar_arrive_expect_tx(&sh.full[stage],
                                          (uint32_t)nch * (16384u + (uint32_t)nbox * kBoxRows * 128u));
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    for (int c = 0; c < nch; ++c) {
                        const int k = chunk_at(kc + c, it.fb, p.k_chunks) * kChunkK;
                        unsigned char *sa = sbase + a_off(it.stream, c);
                        unsigned char *sb = sbase + b_off(it.stream, c);
                        if (UP) {
                            if (p.gu_mode[it.w.a_sel] != kGateUpSplit) {
                                tma_load_4d(sa, ma0, &sh.full[stage], k, arow0, it.w.a_idx, 0, pol_w);
                            } else {
                                tma_load_3d(sa, ma0, &sh.full[stage], k, arow0, it.w.a_idx, pol_w);
                                tma_load_3d(sa + 8192, ma1, &sh.full[stage], k, arow0, it.w.a_idx, pol_w);
                            }
                        } else {
                            tma_load_3d(sa, ma0, &sh.full[stage], k, arow0, it.w.a_idx, pol_w);
                        }
                        for (int j = 0; j < nbox; ++j)
                            tma_load_2d(sb + j * kBoxRows * 128, mb, &sh.full[stage], k,
                                        brow0 + j * kBoxRows, pol_b);
                    }
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
            if (*abort) {  // let every issued copy land before the CTA can exit
                for (int s = 0; s < kStages; ++s)
                    if (armed & (1u << s)) mbar_wait(&sh.full[s], (armed_par >> s) & 1u, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int li = 0;
            for (int item = blockIdx.x; item < total && !*abort; item += gridDim.x, ++li) {
                TcItem it;
                decode_item(p, item, it);
                const int acc = li & 1;
                const uint32_t use = (uint32_t)(li >> 1);
                if (!mbar_wait(&sh.tempty[acc], (use & 1u) ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
                const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)it.w.bn);
                const int per = it.stream ? 2 : 1;
                bool ok = true;
                for (int kc = 0; kc < p.k_chunks; kc += per) {
                    if (!mbar_wait(&sh.full[stage], phase, abort)) { ok = false; break; }
                    tc_fence_after();
                    const int nch = min(per, p.k_chunks - kc);
                    const uint32_t sbase = smem_u32(stages + stage * kStageBytes);
                    for (int c = 0; c < nch; ++c) {
                        const uint32_t sa = sbase + a_off(it.stream, c);
                        const uint32_t sb = sbase + b_off(it.stream, c);
#pragma unroll
                        for (int j = 0; j < kChunkK / 16; ++j)  // 16-wide K steps: +32 bytes
                            tc_mma_bf16(d_tmem, smem_desc_sw128(sa + 32u * j),
                                        smem_desc_sw128(sb + 32u * j), idesc,
                                        (kc + c + j) > 0 ? 1u : 0u);
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
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;            // TMEM lane quarter this warp may read
        const int et = threadIdx.x - 64;   // 0 .. 127
        int li = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x, ++li) {
            TcItem it;
            decode_item(p, item, it);
            const int acc = li & 1;
            const uint32_t use = (uint32_t)(li >> 1);
            // one thread waits, all 128 take the same decision
            if (et == 0) sh.epi_ok = mbar_wait(&sh.tfull[acc], use & 1u, abort) ? 1 : 0;
            named_bar_sync(1, 128);
            const int ok = *(volatile int *)&sh.epi_ok;
            named_bar_sync(1, 128);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)acc * 256u;
            const size_t row0 = (size_t)it.w.dst_row0 + (size_t)it.tb * it.w.bn;
            for (int c0 = 0; c0 < it.n_valid; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + (uint32_t)c0, v);
                tmem_ld_wait();
                if (UP) {
                    float *U = reinterpret_cast<float *>(epi);                 // [32 cols][64 features]
                    uint16_t *H = reinterpret_cast<uint16_t *>(epi + 8192);    // [32 cols][64 features]
                    // lanes 0-63 hold gate and 64-127 up, or the reverse for an up-first tile
                    const bool gate_hi = p.gu_mode[it.w.a_sel] == kUpGateFused;
                    const bool is_gate = (q < 2) != gate_hi;
                    const int f = (q & 1) * 32 + lane;
                    if (!is_gate) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) U[j * 64 + f] = __uint_as_float(v[j]);
                    }
                    named_bar_sync(1, 128);
                    if (is_gate) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float g = __uint_as_float(v[j]);
                            const float hv = g / (1.0f + expf(-g)) * U[j * 64 + f];
                            H[j * 64 + f] = to_bf16_bits(hv);
                        }
                    }
                    named_bar_sync(1, 128);
                    for (int idx = et; idx < 32 * 8; idx += 128) {
                        const int r = idx >> 3, vv = idx & 7;
                        const int col = c0 + r, feat = it.fb * 64 + vv * 8;
                        if (col < it.n_valid && feat < p.out_cols)
                            *reinterpret_cast<uint4 *>(p.out + (row0 + col) * p.out_cols + feat) =
                                *reinterpret_cast<const uint4 *>(H + r * 64 + vv * 8);
                    }
                    named_bar_sync(1, 128);
                } else {
                    uint16_t *Y = reinterpret_cast<uint16_t *>(epi);  // [32 cols][128 features]
                    const int f = q * 32 + lane;
#pragma unroll
                    for (int j = 0; j < 32; ++j) Y[j * 128 + f] = to_bf16_bits(__uint_as_float(v[j]));
                    named_bar_sync(1, 128);
                    for (int idx = et; idx < 32 * 16; idx += 128) {
                        const int r = idx >> 4, vv = idx & 15;
                        const int col = c0 + r, feat = it.fb * 128 + vv * 8;
                        if (col < it.n_valid && feat < p.out_cols)
                            *reinterpret_cast<uint4 *>(p.out + (row0 + col) * p.out_cols + feat) =
                                *reinterpret_cast<const uint4 *>(Y + r * 128 + vv * 8);
                    }
                    named_bar_sync(1, 128);
                }
            }
            tc_fence_before();
            mbar_arrive(&sh.tempty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// bf16 map over a row-major [outer][rows][cols] tensor (outer = 1 for 2-D),
// box = [box_rows][64 cols], 128-byte swizzle, zero fill out of bounds.
static bool encode_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                       uint64_t outer, uint32_t box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {cols, rows, outer};
    const cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kChunkK, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const cuuint32_t rank = outer > 1 ? 3 : 2;
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
static bool encode_weights(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                           uint64_t experts, uint32_t box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {cols, rows, experts};
    const cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kChunkK, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// One map over both the gate and the up tensor ([E][rows][cols] each, dense):
// dims {cols, rows, E, 2}, the last dimension stepping from one tensor to the
// other, so a {64, 64, 1, 2} box is one 16 KB copy of 64 gate rows followed by
// the 64 matching up rows. Strides must increase, so this needs the two
// tensors not to overlap; the tensor at the lower address becomes the first
// half of the tile. Returns kGateUpSplit when they overlap (or on failure),
// and the caller then uses two 3-D maps.
static int encode_gate_up(CUtensorMap *m, const void *gate, const void *up, uint64_t cols,
                          uint64_t rows, uint64_t experts) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return kGateUpSplit;
    const int64_t bytes = (int64_t)(cols * rows * experts * 2);
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
    const cuuint64_t strides[3] = {cols * 2, cols * rows * 2, step};
    const cuuint32_t box[4] = {(cuuint32_t)kChunkK, 64, 1, 2};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? mode : kGateUpSplit;
}

static bool encode_rows(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows) {
    return encode_map(m, base, cols, rows, 1, kBoxRows);
}

static size_t tc_smem_bytes() {
    return 1024 + (size_t)kStages * kStageBytes + kEpiBytes + sizeof(TcShared);
}

cudaError_t launch_ffn_tc(const moge_config &c, const Plan &plan, int n_entries,
                          const FfnOperands &op, int num_sms, cudaStream_t st, cudaEvent_t mid) {
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
    int gu_mode[2];
    gu_mode[0] = encode_gate_up(&mWg, wg, wu, d, I, ne);
    gu_mode[1] = encode_gate_up(&mSg, sg, su, d, I, ns);
    if (gu_mode[0] != kGateUpSplit) mWu = mWg;
    else if (!encode_weights(&mWg, wg, d, I, ne, 64) || !encode_weights(&mWu, wu, d, I, ne, 64))
        return cudaErrorInvalidValue;
    if (gu_mode[1] != kGateUpSplit) mSu = mSg;
    else if (!encode_weights(&mSg, sg, d, I, ns, 64) || !encode_weights(&mSu, su, d, I, ns, 64))
        return cudaErrorInvalidValue;
    if (!encode_rows(&mX0, b0, d, (uint64_t)r0) || !encode_rows(&mX1, b1, d, (uint64_t)r1) ||
        !encode_weights(&mWd, wd, I, d, ne, 128) || !encode_weights(&mSd, sd, I, d, ns, 128) ||
        !encode_rows(&mH, op.h, I, (uint64_t)op.h_rows))
        return cudaErrorInvalidValue;

    const size_t smem = tc_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(ffn_tc_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ffn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;

    TcParams pu{{gu_mode[0], gu_mode[1]}, plan.up, plan.up_start, n_entries,
                (d + kChunkK - 1) / kChunkK, I, (uint16_t *)op.h};
    ffn_tc_kernel<true><<<num_sms, kTcThreads, smem, st>>>(pu, mWg, mWu, mSg, mSu, mX0, mX1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (mid && (e = cudaEventRecord(mid, st)) != cudaSuccess) return e;
    TcParams pd{{kGateUpSplit, kGateUpSplit}, plan.down, plan.down_start, n_entries,
                (I + kChunkK - 1) / kChunkK, d, (uint16_t *)op.y};
    ffn_tc_kernel<false><<<num_sms, kTcThreads, smem, st>>>(pd, mWd, mWd, mSd, mSd, mH, mH);
    return cudaGetLastError();
}

}  // namespace moge
