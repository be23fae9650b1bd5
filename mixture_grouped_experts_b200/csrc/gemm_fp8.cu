// Grouped SwiGLU expert FFN with 8-bit expert weights (weights-only FP8).
//
// Weights are OCP E4M3 codes with one fp32 scale per weight row (output
// channel); activations, h and y stay bf16. The pages report 8-bit weight
// quantisation (hwcomputing.csdn.net news piece, deployment section) and an
// expert-aware quantisation method (techwalker.com article, section 3) but
// give no format; this is the reading taken.
//
// The kernel is the persistent work-queue kernel of gemm_tc.cu (same plan,
// same item order, same per-expert completion counters) with a different
// operand path for the weights:
//   warp 0     scheduler + TMA producer: the codes of a stage land in the
//              upper half of its weight areas (a streaming stage's two
//              K-chunks as one copy of 128 rows x 128 bytes, a tensor stage's
//              chunk as 128 rows x 64 bytes), plus the token rows. It alone
//              decodes each work item and hands it to the other roles
//              through a shared-memory ring
//   warps 6-9  converters: load the stage's codes into registers, then write
//              them back widened to bf16 (every E4M3 value is a bf16 value)
//              over the whole 16 KB area, 128-byte swizzled for the MMA --
//              in place, so a stage is the same 48 KB as in the bf16 kernel
//   warp 1     MMA issuer: tcgen05.mma as in the bf16 kernel once a stage is
//              widened, fp32 accumulators in TMEM (double-buffered)
//   warps 2-5  epilogue: the row scale of each accumulator row (its weight
//              row) multiplies the accumulator, then SwiGLU / stores as in
//              the bf16 kernel
// The tensor cores see exactly the dequantised weights up to the one fp32
// rounding of the scale product in the epilogue, and the weights take half
// the HBM of bf16 ones. The widening moves about 6 bytes of shared memory
// per code and lies on each stage's critical path with the MMA, so at decode
// this kernel runs about as fast as the bf16 one rather than twice as fast
// (measured alternatives: widening into tensor memory with the MMA reading A
// from there, more converter warps, L2 prefetch of codes, fewer and wider
// copies, deeper rings -- none faster).
#include <cuda_fp8.h>

#include "common.cuh"
#include "moge_internal.h"

namespace moge {

// ---------------------------------------------------------------- quantisation
// One CTA per row: amax over the row (exact in fp32), scale = amax / 448 with
// one IEEE fp32 division, then each code = E4M3 round-to-nearest-even,
// saturating, of fp32(w / scale) (another IEEE division).
__global__ void __launch_bounds__(256) quantize_fp8_kernel(const uint4 *__restrict__ w,
                                                           int64_t rows, int64_t cols,
                                                           uint2 *__restrict__ q,
                                                           float *__restrict__ scale) {
    __shared__ float red[8];
    grid_dependency_wait();
    const int64_t nv = cols / 8;  // 8 bf16 per 16-byte vector
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const uint4 *wr = w + r * nv;
        float amax = 0.0f;
        for (int64_t i = threadIdx.x; i < nv; i += blockDim.x) {
            const uint4 v = wr[i];
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                amax = fmaxf(amax, fabsf(__uint_as_float(u[k] << 16)));
                amax = fmaxf(amax, fabsf(__uint_as_float(u[k] & 0xFFFF0000u)));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
        __syncthreads();
        amax = red[0];
        for (int k = 1; k < (int)(blockDim.x >> 5); ++k) amax = fmaxf(amax, red[k]);
        __syncthreads();
        const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        if (threadIdx.x == 0) scale[r] = s;
        uint2 *qr = q + r * nv;
        for (int64_t i = threadIdx.x; i < nv; i += blockDim.x) {
            const uint4 v = wr[i];
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            uint32_t out[2] = {0u, 0u};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float lo = __fdiv_rn(__uint_as_float(u[k] << 16), s);
                const float hi = __fdiv_rn(__uint_as_float(u[k] & 0xFFFF0000u), s);
                const uint32_t b0 = __nv_cvt_float_to_fp8(lo, __NV_SATFINITE, __NV_E4M3);
                const uint32_t b1 = __nv_cvt_float_to_fp8(hi, __NV_SATFINITE, __NV_E4M3);
                out[k >> 1] |= (b0 | (b1 << 8)) << (16 * (k & 1));
            }
            qr[i] = make_uint2(out[0], out[1]);
        }
    }
}

cudaError_t launch_quantize_fp8(const void *w, int64_t rows, int64_t cols, void *q, float *scale,
                                cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const int64_t blocks = rows < 65535 * 8 ? rows : 65535 * 8;
    return launch_pdl(quantize_fp8_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                      static_cast<const uint4 *>(w), rows, cols, static_cast<uint2 *>(q), scale);
}


// ---------------------------------------------------------------- FFN kernel
constexpr int kF8Stages = 4;
constexpr int kF8StageBytes = 48 * 1024;  // stream: 2 x 16 KB weights + 2 x 8 KB tokens;
                                          // tensor: 16 KB weights + up to 32 KB tokens
constexpr int kF8EpiBytes = 12 * 1024;
constexpr int kF8Threads = 320;           // 10 warps
constexpr int kF8CvtThreads = 128;        // warps 6-9
constexpr uint32_t kF8CodeOff = 8192;     // codes land in the upper half of a weight area

struct F8Params {
    TcParams t;
    const float *sc_g[2], *sc_u[2], *sc_d[2];  // per a_sel (routed / shared)
};

constexpr int kF8MaxEntries = 2 * kMaxExperts;  // routed + shared experts of a plan

struct F8Shared {
    uint64_t full[kF8Stages], wide[kF8Stages], empty[kF8Stages];
    uint64_t tfull[2], tempty[2], drain;
    uint64_t slot_full[kSlots], slot_empty[kSlots];
    int slot_item[kSlots];
    TcItem slot_it[kSlots];       // the producer's decoded items
    TcItem epi_it, cvt_it;        // a role leader's copy for its threads
    uint32_t tmem_base;
    int abort;
    int epi_item, cvt_item;
    int st_up[kF8MaxEntries + 1], st_down[kF8MaxEntries + 1];  // the plan's item starts
};

// Decode global item q (up-projection items first) against the plan's item
// starts held in shared memory: a binary search there plus one read of the
// entry. Only the producer decodes; the other roles get the decoded item
// through the slot ring.
__device__ __forceinline__ void decode_item_smem(const TcParams &p, const int *st_up,
                                                 const int *st_down, int tot_up, int q, TcItem &it) {
    it.up = q < tot_up;
    const int local = it.up ? q : q - tot_up;
    const int *start = it.up ? st_up : st_down;
    int lo = 0, hi = p.n_entries - 1;
    while (lo < hi) {  // last entry whose first item is <= local (entries may be empty)
        const int mid = (lo + hi + 1) >> 1;
        if (start[mid] <= local) lo = mid; else hi = mid - 1;
    }
    const int4 *wp = reinterpret_cast<const int4 *>((it.up ? p.plan.up : p.plan.down) + lo);
    const int4 a = __ldg(wp), b = __ldg(wp + 1);
    it.w.rows = a.x;
    it.w.src_row0 = a.y;
    it.w.dst_row0 = a.z;
    it.w.a_sel = a.w;
    it.w.a_idx = b.x;
    it.w.b_sel = b.y;
    it.w.bn = b.z;
    it.w.ntb = b.w;
    it.entry = lo;
    const int r = local - start[lo];
    it.fb = r / it.w.ntb;  // feature block major, token tile fastest
    it.tb = r % it.w.ntb;
    it.n_valid = min(it.w.bn, it.w.rows - it.tb * it.w.bn);
    it.stream = it.w.rows <= kStreamRows;
}

// byte offsets inside a stage of chunk c's (widened) weights and token rows
__device__ __forceinline__ uint32_t f8_a_off(bool stream, int c) { return stream ? c * 16384u : 0u; }
__device__ __forceinline__ uint32_t f8_b_off(bool stream, int c) {
    return stream ? 32768u + c * 8192u : 16384u;
}

// Named barrier over the converter threads that also ANDs a predicate: every
// converter learns whether all of them got past their (bounded) waits.
__device__ __forceinline__ bool cvt_bar_and(bool ok) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 2, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "n"(kF8CvtThreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Two E4M3 codes (low byte first) -> two bf16 values packed low-first. Every
// E4M3 value is exactly representable in f16, f32 and bf16, so each step is exact.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two_codes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two_codes, __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<const uint32_t *>(&b);
}

// In-place widening of a stage's weight chunks. Chunk c's codes (128 rows x
// 64 bytes, row-major) sit at area + 8192; the widened bf16 tile (row r at
// r * 128, 16-byte unit j at (j ^ (r & 7)) * 16: 128-byte swizzle, K-major)
// covers the whole 16 KB area, so it overwrites codes: every converter loads
// all its codes into registers, the converters synchronise, and only then
// write. The synchronisation also ANDs `ok` (each converter's wait for the
// stage): if any wait failed, nobody writes and all return false. Converter
// thread ct handles, in pass p, row p * 16 + (ct / 32) * 4 + (ct % 32) / 8
// and unit ct % 8 (conflict-free loads and stores).
template <int NCH>
__device__ __forceinline__ bool widen_in_place(unsigned char *stage, bool stream, int ct, bool ok) {
    const int cw = ct >> 5, lane = ct & 31;
    const int j = lane & 7;
    uint2 v[NCH][8];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        // a pair of chunks came as one box of 128-byte rows at +8192 (chunk c at
        // byte 64 c of a row); a single chunk as 64-byte rows at its area + 8192
        const unsigned char *codes = NCH == 2 ? stage + kF8CodeOff + c * 64
                                              : stage + f8_a_off(stream, c) + kF8CodeOff;
        const int rstride = NCH == 2 ? 128 : 64;
#pragma unroll
        for (int pass = 0; pass < 8; ++pass) {
            const int r = pass * 16 + cw * 4 + (lane >> 3);
            v[c][pass] = *reinterpret_cast<const uint2 *>(codes + r * rstride + j * 8);
        }
    }
    if (!cvt_bar_and(ok)) return false;  // every code of the stage is in registers
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        unsigned char *tile = stage + f8_a_off(stream, c);
#pragma unroll
        for (int pass = 0; pass < 8; ++pass) {
            const int r = pass * 16 + cw * 4 + (lane >> 3);
            uint4 o;
            o.x = e4m3x2_to_bf16x2(v[c][pass].x & 0xFFFFu);
            o.y = e4m3x2_to_bf16x2(v[c][pass].x >> 16);
            o.z = e4m3x2_to_bf16x2(v[c][pass].y & 0xFFFFu);
            o.w = e4m3x2_to_bf16x2(v[c][pass].y >> 16);
            *reinterpret_cast<uint4 *>(tile + r * 128 + ((j ^ (r & 7)) << 4)) = o;
        }
    }
    return true;
}

__global__ void __launch_bounds__(kF8Threads, 1) ffn_fp8_kernel(
    const __grid_constant__ F8Params p, const __grid_constant__ CUtensorMap tmWg,
    const __grid_constant__ CUtensorMap tmWu, const __grid_constant__ CUtensorMap tmSg,
    const __grid_constant__ CUtensorMap tmSu, const __grid_constant__ CUtensorMap tmX0,
    const __grid_constant__ CUtensorMap tmX1, const __grid_constant__ CUtensorMap tmWd,
    const __grid_constant__ CUtensorMap tmSd, const __grid_constant__ CUtensorMap tmH,
    const __grid_constant__ CUtensorMap tmWg2, const __grid_constant__ CUtensorMap tmWu2,
    const __grid_constant__ CUtensorMap tmSg2, const __grid_constant__ CUtensorMap tmSu2,
    const __grid_constant__ CUtensorMap tmWd2, const __grid_constant__ CUtensorMap tmSd2) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    unsigned char *stages = smem;                              // kF8Stages x 48 KB
    unsigned char *epi = smem + kF8Stages * kF8StageBytes;     // 12 KB
    F8Shared &sh = *reinterpret_cast<F8Shared *>(epi + kF8EpiBytes);
    volatile int *abort = &sh.abort;
    const TcParams &tp = p.t;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kF8Stages; ++s) {
            mbar_init(&sh.full[s], 1);   // the producer's expect_tx arrival (+ the copies' bytes)
            mbar_init(&sh.wide[s], 1);   // the converter leader: weights widened
            mbar_init(&sh.empty[s], 1);  // the MMA commit: stage consumed
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh.tfull[a], 1);
            mbar_init(&sh.tempty[a], 128);
        }
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&sh.slot_full[s], 1);
            mbar_init(&sh.slot_empty[s], 3);  // MMA thread, epilogue leader, converter leader
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
    grid_dependency_wait();
    for (int i = threadIdx.x; i <= tp.n_entries; i += blockDim.x) {
        sh.st_up[i] = __ldg(tp.plan.up_start + i);
        sh.st_down[i] = __ldg(tp.plan.down_start + i);
    }
    __syncthreads();
    const int tot_up = sh.st_up[tp.n_entries];
    const int total = tot_up + sh.st_down[tp.n_entries];
    const int fb_up = (tp.I + 63) / 64;

    if (warp == 0) {
        // ------------------------------------------------------ scheduler + producer
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_b = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_par = 0;
        int next = lane == 0 ? atomicAdd(tp.sync, 1) : 0;
        for (int s = 0;; ++s) {
            const int slot = s % kSlots;
            int q = 0;
            if (lane == 0) {
                if (mbar_wait(&sh.slot_empty[slot], ((uint32_t)(s / kSlots) & 1u) ^ 1u, abort)) {
                    q = *abort ? total : next;
                    if (q < total) {
                        TcItem d;
                        decode_item_smem(tp, sh.st_up, sh.st_down, tot_up, q, d);
                        sh.slot_it[slot] = d;
                    }
                    sh.slot_item[slot] = q;
                    mbar_arrive(&sh.slot_full[slot]);
                    if (q < total) next = atomicAdd(tp.sync, 1);
                } else {
                    q = -1;
                }
            }
            __syncwarp();
            q = __shfl_sync(0xffffffffu, q, 0);
            if (q < 0 || q >= total) break;
            const TcItem it = sh.slot_it[slot];
            if (!it.up) {  // the h rows of this expert must all be stored
                int ok = 1;
                if (lane == 0) ok = wait_counter(tp.sync + 1 + it.entry, it.w.ntb * fb_up, abort);
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                fence_proxy_async_global();
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
            const int gu = tp.gu_mode[it.w.a_sel];
            const int na = (it.up && gu == kGateUpSplit) ? 2 : 1;  // code copies per chunk
            const int kcs = it.up ? tp.kc_up : tp.kc_down;
            const int per = it.stream ? 2 : 1;
            const int nbox = (it.w.bn + kBoxRows - 1) / kBoxRows;
            const int brow0 = it.w.src_row0 + it.tb * it.w.bn;
            const int arow0 = it.up ? it.fb * 64 : it.fb * 128;
            const int ops = na + nbox;
            const int my_c = lane / ops, my_r = lane % ops;
            const CUtensorMap *ma0w, *ma1w;
            if (it.up) {
                ma0w = it.w.a_sel ? &tmSg2 : &tmWg2;
                ma1w = it.w.a_sel ? &tmSu2 : &tmWu2;
            } else {
                ma0w = ma1w = it.w.a_sel ? &tmSd2 : &tmWd2;
            }
            bool ok = true;
            for (int kc = 0; kc < kcs; kc += per) {
                int got = 1;
                if (lane == 0) got = mbar_wait(&sh.empty[stage], phase ^ 1u, abort);
                if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
                const int nch = min(per, kcs - kc);
                unsigned char *sbase = stages + stage * kF8StageBytes;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sh.full[stage],
                                          (uint32_t)nch * (8192u + (uint32_t)nbox * kBoxRows * 128u));
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                }
                __syncwarp();
                if (nch == 2) {
                    // a streaming pair: one wide copy of codes (or two, gate and up
                    // apart) and the token boxes of both chunks
                    const int k = kc * kChunkK;
                    if (lane < na) {
                        unsigned char *sa = sbase + kF8CodeOff;
                        if (it.up && gu != kGateUpSplit)
                            tma_load_4d(sa, ma0w, &sh.full[stage], k, arow0, it.w.a_idx, 0, pol_w);
                        else if (it.up)
                            tma_load_3d(sa + 8192 * lane, lane ? ma1w : ma0w, &sh.full[stage], k,
                                        arow0, it.w.a_idx, pol_w);
                        else
                            tma_load_3d(sa, ma0w, &sh.full[stage], k, arow0, it.w.a_idx, pol_w);
                    } else if (lane < na + 2 * nbox) {
                        const int c = (lane - na) / nbox, j = (lane - na) % nbox;
                        tma_load_2d(sbase + f8_b_off(true, c) + j * kBoxRows * 128, mb,
                                    &sh.full[stage], k + c * kChunkK, brow0 + j * kBoxRows, pol_b);
                    }
                    if (++stage == kF8Stages) { stage = 0; phase ^= 1u; }
                    continue;
                }
                if (my_c < nch) {
                    const int k = (kc + my_c) * kChunkK;
                    unsigned char *sa = sbase + f8_a_off(it.stream, my_c) + kF8CodeOff;
                    unsigned char *sb = sbase + f8_b_off(it.stream, my_c);
                    if (my_r >= na) {
                        const int j = my_r - na;
                        tma_load_2d(sb + j * kBoxRows * 128, mb, &sh.full[stage], k,
                                    brow0 + j * kBoxRows, pol_b);
                    } else if (it.up && gu != kGateUpSplit) {
                        tma_load_4d(sa, ma0, &sh.full[stage], k, arow0, it.w.a_idx, 0, pol_w);
                    } else if (it.up) {  // gate rows, then up rows: 64 rows x 64 bytes each
                        tma_load_3d(sa + 4096 * my_r, my_r ? ma1 : ma0, &sh.full[stage], k, arow0,
                                    it.w.a_idx, pol_w);
                    } else {
                        tma_load_3d(sa, ma0, &sh.full[stage], k, arow0, it.w.a_idx, pol_w);
                    }
                }
                if (++stage == kF8Stages) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
        if (lane == 0 && *abort) {  // let every issued copy land before the CTA can exit
            for (int s = 0; s < kF8Stages; ++s)
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
                TcItem it;
                if (q < total) it = sh.slot_it[slot];
                mbar_arrive(&sh.slot_empty[slot]);
                if (q >= total) break;
                const int acc = s & 1;
                const uint32_t use = (uint32_t)(s >> 1);
                if (!mbar_wait(&sh.tempty[acc], (use & 1u) ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
                const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)it.w.bn);
                const int kcs = it.up ? tp.kc_up : tp.kc_down;
                const int per = it.stream ? 2 : 1;
                bool ok = true;
                for (int kc = 0; kc < kcs; kc += per) {
                    // the stage's copies have landed and its weights are widened
                    if (!mbar_wait(&sh.full[stage], phase, abort) ||
                        !mbar_wait(&sh.wide[stage], phase, abort)) { ok = false; break; }
                    tc_fence_after();
                    const int nch = min(per, kcs - kc);
                    const uint32_t sbase = smem_u32(stages + stage * kF8StageBytes);
                    for (int c = 0; c < nch; ++c) {
                        const uint32_t sa = sbase + f8_a_off(it.stream, c);
                        const uint32_t sb = sbase + f8_b_off(it.stream, c);
#pragma unroll
                        for (int j = 0; j < kChunkK / 16; ++j)
                            tc_mma_bf16(d_tmem, smem_desc_sw128(sa + 32u * j),
                                        smem_desc_sw128(sb + 32u * j), idesc,
                                        (kc + c + j) > 0 ? 1u : 0u);
                    }
                    tc_commit(&sh.empty[stage]);
                    if (++stage == kF8Stages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&sh.tfull[acc]);
            }
            tc_commit(&sh.drain);
            mbar_wait(&sh.drain, 0, nullptr);
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------ converters
        const int ct = threadIdx.x - 192;  // 0 .. 127
        int stage = 0;
        uint32_t phase = 0;
        for (int s = 0;; ++s) {
            if (ct == 0) {
                const int slot = s % kSlots;
                int q = -1;
                if (mbar_wait(&sh.slot_full[slot], (uint32_t)(s / kSlots) & 1u, abort)) {
                    q = sh.slot_item[slot];
                    if (q < total) sh.cvt_it = sh.slot_it[slot];
                    mbar_arrive(&sh.slot_empty[slot]);
                }
                sh.cvt_item = q;
            }
            named_bar_sync(2, kF8CvtThreads);
            const int q = *(volatile int *)&sh.cvt_item;
            if (q < 0 || q >= total) break;
            const TcItem it = sh.cvt_it;
            named_bar_sync(2, kF8CvtThreads);
            const int kcs = it.up ? tp.kc_up : tp.kc_down;
            const int per = it.stream ? 2 : 1;
            bool ok = true;
            for (int kc = 0; kc < kcs; kc += per) {
                const int nch = min(per, kcs - kc);
                const bool mine = mbar_wait(&sh.full[stage], phase, abort);
                unsigned char *sbase = stages + stage * kF8StageBytes;
                ok = nch == 2 ? widen_in_place<2>(sbase, it.stream, ct, mine)
                              : widen_in_place<1>(sbase, it.stream, ct, mine);
                if (!ok) break;  // every converter takes the same decision
                fence_proxy_async_smem();  // generic-proxy writes -> the MMA's async reads
                named_bar_sync(2, kF8CvtThreads);
                if (ct == 0) mbar_arrive(&sh.wide[stage]);
                if (++stage == kF8Stages) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------ epilogue (warps 2-5)
        const int q4 = warp & 3;
        const int et = threadIdx.x - 64;  // 0 .. 127
        for (int s = 0;; ++s) {
            if (et == 0) {
                const int slot = s % kSlots;
                int q = -1;
                if (mbar_wait(&sh.slot_full[slot], (uint32_t)(s / kSlots) & 1u, abort)) {
                    q = sh.slot_item[slot];
                    if (q < total) sh.epi_it = sh.slot_it[slot];
                    mbar_arrive(&sh.slot_empty[slot]);
                    if (q < total && !mbar_wait(&sh.tfull[s & 1], (uint32_t)(s >> 1) & 1u, abort))
                        q = -1;
                }
                sh.epi_item = q;
            }
            named_bar_sync(1, 128);
            const int q = *(volatile int *)&sh.epi_item;
            if (q < 0 || q >= total) break;
            const TcItem it = sh.epi_it;
            named_bar_sync(1, 128);
            tc_fence_after();
            const int acc = s & 1;
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q4) << 16) + (uint32_t)acc * 256u;
            const size_t row0 = (size_t)it.w.dst_row0 + (size_t)it.tb * it.w.bn;
            // the row scale of this thread's accumulator row (its weight row)
            const int m = q4 * 32 + lane;
            const bool gate_hi = tp.gu_mode[it.w.a_sel] == kUpGateFused;
            const bool is_gate = (q4 < 2) != gate_hi;
            float rs = 0.0f;
            if (it.up) {
                const int f = it.fb * 64 + (m & 63);
                const float *sc = is_gate ? p.sc_g[it.w.a_sel] : p.sc_u[it.w.a_sel];
                if (f < tp.I) rs = __ldg(sc + (size_t)it.w.a_idx * tp.I + f);
            } else {
                const int f = it.fb * 128 + m;
                if (f < tp.d) rs = __ldg(p.sc_d[it.w.a_sel] + (size_t)it.w.a_idx * tp.d + f);
            }
            for (int c0 = 0; c0 < it.n_valid; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + (uint32_t)c0, v);
                tmem_ld_wait();
                if (it.up) {
                    float *U = reinterpret_cast<float *>(epi);               // [32 cols][64 features]
                    uint16_t *H = reinterpret_cast<uint16_t *>(epi + 8192);  // [32 cols][64 features]
                    const int f = (q4 & 1) * 32 + lane;
                    if (!is_gate) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) U[j * 64 + f] = __uint_as_float(v[j]) * rs;
                    }
                    named_bar_sync(1, 128);
                    if (is_gate) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float g = __uint_as_float(v[j]) * rs;
                            const float hv = g / (1.0f + expf(-g)) * U[j * 64 + f];
                            H[j * 64 + f] = to_bf16_bits(hv);
                        }
                    }
                    named_bar_sync(1, 128);
                    for (int idx = et; idx < 32 * 8; idx += 128) {
                        const int r = idx >> 3, vv = idx & 7;
                        const int col = c0 + r, feat = it.fb * 64 + vv * 8;
                        if (col < it.n_valid && feat < tp.I)
                            *reinterpret_cast<uint4 *>(tp.h + (row0 + col) * tp.I + feat) =
                                *reinterpret_cast<const uint4 *>(H + r * 64 + vv * 8);
                    }
                    named_bar_sync(1, 128);
                } else {
                    uint16_t *Y = reinterpret_cast<uint16_t *>(epi);  // [32 cols][128 features]
                    const int f = q4 * 32 + lane;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        Y[j * 128 + f] = to_bf16_bits(__uint_as_float(v[j]) * rs);
                    named_bar_sync(1, 128);
                    for (int idx = et; idx < 32 * 16; idx += 128) {
                        const int r = idx >> 4, vv = idx & 15;
                        const int col = c0 + r, feat = it.fb * 128 + vv * 8;
                        if (col < it.n_valid && feat < tp.d)
                            *reinterpret_cast<uint4 *>(tp.y + (row0 + col) * tp.d + feat) =
                                *reinterpret_cast<const uint4 *>(Y + r * 128 + vv * 8);
                    }
                    named_bar_sync(1, 128);
                }
            }
            tc_fence_before();
            mbar_arrive(&sh.tempty[acc]);
            if (it.up) {
                fence_proxy_async_global();
                __threadfence();
                named_bar_sync(1, 128);
                if (et == 0) atomicAdd(tp.sync + 1 + it.entry, 1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side.
static bool encode_u8(CUtensorMap *m, const void *base, cuuint32_t rank, const cuuint64_t *dims,
                      const cuuint64_t *strides, const cuuint32_t *box) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// codes [experts][rows][cols], box = [box_rows][64 codes] of one expert
static bool encode_codes(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                         uint64_t experts, uint32_t box_rows) {
    const cuuint64_t dims[3] = {cols, rows, experts};
    const cuuint64_t strides[2] = {cols, cols * rows};
    const cuuint32_t box[3] = {(cuuint32_t)kChunkK, box_rows, 1};
    return encode_u8(m, base, 3, dims, strides, box);
}

// gate + up codes in one 4-D map (as encode_gate_up in gemm_tc.cu, 1-byte elements)
static int encode_codes_gate_up(CUtensorMap *m, const void *gate, const void *up, uint64_t cols,
                                uint64_t rows, uint64_t experts) {
    const int64_t bytes = (int64_t)(cols * rows * experts);
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
    const cuuint64_t strides[3] = {cols, cols * rows, step};
    const cuuint32_t box[4] = {(cuuint32_t)kChunkK, 64, 1, 2};
    return encode_u8(m, base, 4, dims, strides, box) ? mode : kGateUpSplit;
}

// Streaming stages fetch both K-chunks' codes of a weight row as one 128-byte
// segment (boxes of 128 codes x rows); rows of the box keep the global layout
// (no swizzle), chunk c being bytes 64 c .. 64 c + 63 of each row.
static bool encode_codes_wide(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                              uint64_t experts, uint32_t box_rows) {
    const cuuint64_t dims[3] = {cols, rows, experts};
    const cuuint64_t strides[2] = {cols, cols * rows};
    const cuuint32_t box[3] = {(cuuint32_t)(2 * kChunkK), box_rows, 1};
    return encode_u8(m, base, 3, dims, strides, box);
}
static bool encode_codes_gate_up_wide(CUtensorMap *m, const void *base, uint64_t cols,
                                      uint64_t rows, uint64_t experts, uint64_t step) {
    const cuuint64_t dims[4] = {cols, rows, experts, 2};
    const cuuint64_t strides[3] = {cols, cols * rows, step};
    const cuuint32_t box[4] = {(cuuint32_t)(2 * kChunkK), 64, 1, 2};
    return encode_u8(m, base, 4, dims, strides, box);
}

static size_t f8_smem_bytes() {
    return 1024 + (size_t)kF8Stages * kF8StageBytes + kF8EpiBytes + sizeof(F8Shared);
}

cudaError_t launch_ffn_fp8(const moge_config &c, const Plan &plan, int n_entries,
                           const FfnOperands &op, int num_sms, cudaStream_t st) {
    if (n_entries <= 0 || c.T <= 0) return cudaSuccess;
    const int N = c.N, S = c.S, d = c.d, I = c.I;
    // a missing side borrows the other's pointers so that its maps are valid
    // (no plan entry ever selects it)
    const void *wg = op.wg ? op.wg : op.sg, *wu = op.wu ? op.wu : op.su, *wd = op.wd ? op.wd : op.sd;
    const float *wgs = op.wg ? op.wg_s : op.sg_s, *wus = op.wu ? op.wu_s : op.su_s,
                *wds = op.wd ? op.wd_s : op.sd_s;
    const int ne = op.wg ? N : S;
    const void *sg = op.sg ? op.sg : wg, *su = op.su ? op.su : wu, *sd = op.sd ? op.sd : wd;
    const float *sgs = op.sg ? op.sg_s : wgs, *sus = op.su ? op.su_s : wus,
                *sds = op.sd ? op.sd_s : wds;
    const int ns = op.sg ? S : ne;
    const void *b0 = op.b0 ? op.b0 : op.b1, *b1 = op.b1 ? op.b1 : op.b0;
    const int64_t r0 = op.b0 ? op.b0_rows : op.b1_rows, r1 = op.b1 ? op.b1_rows : op.b0_rows;

    CUtensorMap mWg, mWu, mSg, mSu, mX0, mX1, mWd, mSd, mH;
    F8Params p;
    TcParams &t = p.t;
    t.gu_mode[0] = encode_codes_gate_up(&mWg, wg, wu, d, I, ne);
    t.gu_mode[1] = encode_codes_gate_up(&mSg, sg, su, d, I, ns);
    if (t.gu_mode[0] != kGateUpSplit) mWu = mWg;
    else if (!encode_codes(&mWg, wg, d, I, ne, 64) || !encode_codes(&mWu, wu, d, I, ne, 64))
        return cudaErrorInvalidValue;
    if (t.gu_mode[1] != kGateUpSplit) mSu = mSg;
    else if (!encode_codes(&mSg, sg, d, I, ns, 64) || !encode_codes(&mSu, su, d, I, ns, 64))
        return cudaErrorInvalidValue;
    if (!encode_rows(&mX0, b0, d, (uint64_t)r0) || !encode_rows(&mX1, b1, d, (uint64_t)r1) ||
        !encode_codes(&mWd, wd, I, d, ne, 128) || !encode_codes(&mSd, sd, I, d, ns, 128) ||
        !encode_rows(&mH, op.h, I, (uint64_t)op.h_rows))
        return cudaErrorInvalidValue;
    t.plan = plan;
    t.n_entries = n_entries;
    t.kc_up = (d + kChunkK - 1) / kChunkK;
    t.kc_down = (I + kChunkK - 1) / kChunkK;
    t.I = I;
    t.d = d;
    t.h = (uint16_t *)op.h;
    t.y = (uint16_t *)op.y;
    t.sync = plan.sync;
    p.sc_g[0] = wgs; p.sc_u[0] = wus; p.sc_d[0] = wds;
    p.sc_g[1] = sgs; p.sc_u[1] = sus; p.sc_d[1] = sds;

    // maps of the streaming stages: two K-chunks of codes per weight row
    CUtensorMap mWg2, mWu2, mSg2, mSu2, mWd2, mSd2;
    auto wide_gu = [&](CUtensorMap *g2, CUtensorMap *u2, int mode, const void *g, const void *u,
                       int ex) -> bool {
        if (mode == kGateUpSplit)
            return encode_codes_wide(g2, g, d, I, ex, 64) && encode_codes_wide(u2, u, d, I, ex, 64);
        const char *lo = static_cast<const char *>(mode == kGateUpFused ? g : u);
        const char *hi = static_cast<const char *>(mode == kGateUpFused ? u : g);
        if (!encode_codes_gate_up_wide(g2, lo, d, I, ex, (uint64_t)(hi - lo))) return false;
        *u2 = *g2;
        return true;
    };
    if (!wide_gu(&mWg2, &mWu2, t.gu_mode[0], wg, wu, ne) ||
        !wide_gu(&mSg2, &mSu2, t.gu_mode[1], sg, su, ns) ||
        !encode_codes_wide(&mWd2, wd, I, d, ne, 128) || !encode_codes_wide(&mSd2, sd, I, d, ns, 128))
        return cudaErrorInvalidValue;
    const size_t smem = f8_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(ffn_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(ffn_fp8_kernel, dim3(num_sms), dim3(kF8Threads), smem, st, p, mWg, mWu, mSg,
                      mSu, mX0, mX1, mWd, mSd, mH, mWg2, mWu2, mSg2, mSu2, mWd2, mSd2);
}

}  // namespace moge
