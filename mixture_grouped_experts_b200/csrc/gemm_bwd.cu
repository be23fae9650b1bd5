// Backward pass of the MoGE layer: its grouped GEMMs on the 5th-generation
// tensor cores (sm_100a).
//
// One persistent kernel serves seven GEMM kinds; a launch runs one kind over
// every expert entry of the forward's plan (shared experts first, then the
// routed ones, rows in the forward's permuted order). With x, x_perm, h, the
// saved SwiGLU pre-activations gu = [g | u] and dy_perm = w * dy (routed rows)
// or dy (shared rows), for expert e:
//   kDH     dh^T  = Wd^T dy^T      -> SwiGLU backward in the epilogue: dgu = [dg | du]
//   kDX     dx^T  = Wg^T dg^T + Wu^T du^T   (K runs over [g | u]: 2I)
//   kDWD    dWd   = dy^T h         (K = the expert's rows)
//   kDWGU   dWg   = dg^T x,  dWu = du^T x   (K = the expert's rows)
// and for the router (one entry, all T tokens):
//   kLOGITS l     = x Wr^T + bias  (recomputed logits, fp32)
//   kDWR    dWr   = dl^T x         (K = T)
//   kDXR    dx_r  = dl Wr          (K = N, fp32)
// D = A B^T with the MMA's M = 128 rows of A in TMEM lanes and N <= 256
// columns. Operands are staged by TMA with the 128-byte swizzle; a row-major
// matrix read along its rows is a "K-major" operand, read across them an
// "MN-major" one (tcgen05 descriptor: 8-row groups 1024 bytes apart,
// 64-element blocks 8 KB apart). Few, large copies: a copy's issue cost, not
// its bytes, bounded these GEMMs with 8 KB boxes. So a K-major operand comes
// in 128-row boxes, and an MN-major one -- whose 128-byte swizzle row holds
// only 64 of its MN elements -- through a view of the matrix whose outermost
// dimension steps over its 64-column blocks ({64 columns, rows, column
// blocks}, the blocks 128 bytes apart): one copy lands several 64-wide blocks
// one after another, 8 KB apart, which is the descriptor's layout. Gradients over an expert's rows have a
// ragged last K-chunk: its rows past the expert are zeroed in shared memory in
// the A operand (they belong to the next expert) and the MMAs past them are
// skipped.
//
// Roles per CTA (one per SM, 192 threads): warp 0 TMA producer, warp 1 MMA
// issuer (one thread; the warp zeroes ragged rows), warps 2-5 epilogue. Items
// are dealt out statically (item blockIdx.x + i * gridDim.x), all three roles
// walk the same sequence; two 256-column accumulators let the epilogue of one
// item overlap the MMAs of the next. Every wait is bounded.
#include "common.cuh"
#include "moge_internal.h"

namespace moge {

constexpr int kGStages = 4;
constexpr int kGStageBytes = 48 * 1024;  // A: 2 boxes (16 KB), B: up to 4 boxes (32 KB)
constexpr int kGThreads = 192;
constexpr uint32_t kGTmemCols = 512;
constexpr int kGMaxEntries = kMaxExperts + 64;
constexpr int kGEpiBytes = 4 * 2 * 2048;  // per epilogue warp: two [32][32] bf16 staging tiles

// m[0..5]: operand maps (per kind); m[6..9]: weight-gradient outputs, stored
// by TMA from a staging tile ([32 rows][32 cols] bf16 per epilogue warp)
struct GMaps {
    CUtensorMap m[10];
};

struct GParams {
    int kind;
    const ExpertWork *ent;  // forward plan entries (token and weight-gradient kinds)
    int n_entries;
    int T, d, I, N;
    int m_tiles;            // M tiles per entry (per part for kDWGU)
    int n_tiles, bn;        // weight-gradient and router kinds: N tiles and their width
    int kc;                 // K chunks of the fixed-K kinds
    int ksplit;             // kLOGITS: K split into this many parts, partial logits per part
    int nst;                // pipeline stages in use (3 for the weight-gradient kinds, whose
                            // freed stage holds the epilogue's store staging tiles)
    void *out[4];
    const uint16_t *gu;     // kDH: [rows][2I]
    const float *bias;      // kLOGITS, nullable
    int a_wide, b_wide;     // A: one 128-column copy; B: one 256-column copy (MN-major views)
};

// One work item, with its plan entry's fields held in registers (the copy
// issue and the epilogues read them every chunk)
struct GItem {
    int entry, mt, nt, bn, n_valid, nck, kv_last;
    int a_sel, a_idx, b_sel, src_row0, dst_row0;
    int ks, kc0;  // kLOGITS: K part and its first chunk
};

struct GShared {
    uint64_t full[kGStages], empty[kGStages], tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    int abort;
    int total;
    int epi_ok;  // the epilogue leader's wait result, shared with the other epilogue threads
    int start[kGMaxEntries + 1];  // token kinds: prefix sum of items per entry
};

__device__ __forceinline__ bool g_token_kind(int kind) { return kind == kDH || kind == kDX; }
__device__ __forceinline__ bool g_wgrad_kind(int kind) { return kind == kDWD || kind == kDWGU; }
// (A, B) is MN-major?
__device__ __forceinline__ bool g_a_mn(int kind) { return kind != kLOGITS; }
__device__ __forceinline__ bool g_b_mn(int kind) {
    return kind == kDWD || kind == kDWGU || kind == kDWR;
}

__device__ void g_decode(const GParams &p, const GShared &sh, int q, GItem &it) {
    it.kv_last = 64;
    it.a_sel = it.a_idx = it.b_sel = it.src_row0 = it.dst_row0 = 0;
    it.ks = it.kc0 = 0;
    if (g_token_kind(p.kind)) {
        int lo = 0, hi = p.n_entries - 1;
        while (lo < hi) {  // last entry whose first item is <= q
            const int mid = (lo + hi + 1) >> 1;
            if (sh.start[mid] <= q) lo = mid; else hi = mid - 1;
        }
        const ExpertWork &w = p.ent[lo];
        const int r = q - sh.start[lo];
        it.entry = lo;
        it.a_sel = w.a_sel; it.a_idx = w.a_idx; it.b_sel = w.b_sel;
        it.src_row0 = w.src_row0; it.dst_row0 = w.dst_row0;
        it.mt = r / w.ntb;
        it.nt = r % w.ntb;
        it.bn = w.bn;
        it.n_valid = min(w.bn, w.rows - it.nt * w.bn);
        it.nck = p.kc;
    } else if (g_wgrad_kind(p.kind)) {
        const int mt_all = p.kind == kDWGU ? 2 * p.m_tiles : p.m_tiles;
        const int per = mt_all * p.n_tiles;
        it.entry = q / per;
        const int r = q % per;
        it.mt = r / p.n_tiles;
        it.nt = r % p.n_tiles;
        it.bn = p.bn;
        it.n_valid = p.bn;
        const ExpertWork &w = p.ent[it.entry];
        const int rows = w.rows;
        it.a_sel = w.a_sel; it.a_idx = w.a_idx; it.b_sel = w.b_sel;
        it.src_row0 = w.src_row0; it.dst_row0 = w.dst_row0;
        it.nck = (rows + 63) / 64;
        it.kv_last = rows - 64 * (it.nck - 1);
    } else {
        it.entry = 0;
        const int ksp = p.kind == kLOGITS ? p.ksplit : 1;
        it.ks = q % ksp;
        q /= ksp;
        it.mt = q / p.n_tiles;
        it.nt = q % p.n_tiles;
        it.bn = p.bn;
        const int ncols = p.kind == kDWR ? p.d : p.T;
        it.n_valid = min(p.bn, ncols - it.nt * p.bn);
        it.nck = p.kind == kDWR ? (p.T + 63) / 64 : p.kc;
        if (ksp > 1) {  // chunks [kc0, kc0 + nck) of this part
            it.kc0 = it.ks * it.nck / ksp;
            it.nck = (it.ks + 1) * it.nck / ksp - it.kc0;
        }
    }
}

// Copies of one chunk: A in na copies, B in nb (g_copies); lane j issues
// copy j (A's first). A wide copy (p.a_wide / p.b_wide) is one copy of a
// column-block view (see the file comment); otherwise 64 x 64 boxes, or
// 128-row boxes for the K-major B rows of the token kinds.
__device__ __forceinline__ void g_copies(const GParams &p, const GItem &it, int &na, int &nb,
                                         uint32_t &bytes) {
    na = p.a_wide ? 1 : 2;
    if (p.b_wide) nb = 1;
    else if (g_token_kind(p.kind)) nb = (it.bn + 127) / 128;
    else nb = (it.bn + 63) / 64;
    const uint32_t bbox = p.b_wide ? (uint32_t)p.bn * 128u : g_token_kind(p.kind) ? 16384u : 8192u;
    bytes = 16384u + bbox * (uint32_t)nb;
}

__device__ __forceinline__ void g_load(const GParams &p, const GMaps &mp, const GItem &it, int kc,
                                       int j, int na, unsigned char *stage, uint64_t *bar,
                                       uint64_t pol_a, uint64_t pol_b) {
    const int k = 64 * (kc + it.kc0);
    if (j < na) {
        unsigned char *dst = stage + 8192 * j;
        const int mn = it.mt * 128 + 64 * j;
        switch (p.kind) {
            case kDH:  // Wd[e] as [d][I]: rows are K
                if (p.a_wide) tma_load_4d(dst, &mp.m[it.a_sel], bar, 0, k, mn / 64, it.a_idx, pol_a);
                else tma_load_3d(dst, &mp.m[it.a_sel], bar, mn, k, it.a_idx, pol_a);
                break;
            case kDX: {  // Wg[e] then Wu[e], as [I][d]: rows are K
                const int kh = p.I / 64;
                const int sel = (kc < kh ? 0 : 2) + it.a_sel;
                const int kk = kc < kh ? k : k - p.I;
                if (p.a_wide) tma_load_4d(dst, &mp.m[sel], bar, 0, kk, mn / 64, it.a_idx, pol_a);
                else tma_load_3d(dst, &mp.m[sel], bar, mn, kk, it.a_idx, pol_a);
                break;
            }
            case kDWD:  // dy rows (dy_perm / dy) read across: rows are K
                if (p.a_wide) tma_load_3d(dst, &mp.m[it.b_sel], bar, 0, it.src_row0 + k, mn / 64, pol_a);
                else tma_load_2d(dst, &mp.m[it.b_sel], bar, mn, it.src_row0 + k, pol_a);
                break;
            case kDWGU: {  // [g | u] rows read across
                const int part = it.mt / p.m_tiles;
                const int m0 = (it.mt - part * p.m_tiles) * 128 + 64 * j + part * p.I;
                if (p.a_wide) tma_load_3d(dst, &mp.m[0], bar, 0, it.dst_row0 + k, m0 / 64, pol_a);
                else tma_load_2d(dst, &mp.m[0], bar, m0, it.dst_row0 + k, pol_a);
                break;
            }
            case kLOGITS:  // Wr rows, K-major
                tma_load_2d(dst, &mp.m[0], bar, k, mn, pol_a);
                break;
            default:  // kDWR: dl read across (rows are tokens = K); kDXR: Wr read across
                tma_load_2d(dst, &mp.m[0], bar, mn, k, pol_a);
                break;
        }
    } else {
        const int jb = j - na;
        const int brows = p.b_wide ? 256 : g_token_kind(p.kind) ? 128 : 64;
        unsigned char *dst = stage + 16384 + brows * 128 * jb;
        const int r0 = it.nt * it.bn + brows * jb;  // first N element of the copy
        switch (p.kind) {
            case kDH:  // dy rows, K-major
                tma_load_2d(dst, &mp.m[2 + it.b_sel], bar, k, it.src_row0 + r0, pol_b);
                break;
            case kDX:  // [dg | du] rows, K-major
                tma_load_2d(dst, &mp.m[4], bar, k, it.dst_row0 + r0, pol_b);
                break;
            case kDWD:  // h rows read across
                if (p.b_wide) tma_load_3d(dst, &mp.m[2], bar, 0, it.dst_row0 + k, r0 / 64, pol_b);
                else tma_load_2d(dst, &mp.m[2], bar, r0, it.dst_row0 + k, pol_b);
                break;
            case kDWGU:  // x rows (x_perm / x) read across
                if (p.b_wide) tma_load_3d(dst, &mp.m[2 + it.b_sel], bar, 0, it.src_row0 + k, r0 / 64, pol_b);
                else tma_load_2d(dst, &mp.m[2 + it.b_sel], bar, r0, it.src_row0 + k, pol_b);
                break;
            case kDWR:  // x read across
                tma_load_2d(dst, &mp.m[1], bar, r0, k, pol_b);
                break;
            default:  // kLOGITS: x rows; kDXR: dl rows (K-major)
                tma_load_2d(dst, &mp.m[1], bar, k, r0, pol_b);
                break;
        }
    }
}

// Instruction descriptor of kind::f16 with the operands' majors (bit 15: A
// MN-major, bit 16: B MN-major).
__device__ __forceinline__ uint32_t g_idesc(int kind, uint32_t n) {
    return idesc_bf16_f32(128, n) | (g_a_mn(kind) ? (1u << 15) : 0u) |
           (g_b_mn(kind) ? (1u << 16) : 0u);
}

// Shared-memory descriptor of a 128-byte-swizzled operand: K-major (8-row
// groups 1024 bytes apart) or MN-major (64-element blocks 8 KB apart, 8-row K
// groups 1024 bytes apart).
__device__ __forceinline__ uint64_t g_sdesc(uint32_t saddr, bool mn) {
    uint64_t dsc = 0;
    dsc |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    dsc |= (uint64_t)((mn ? 8192u : 16u) >> 4) << 16;
    dsc |= (uint64_t)(1024u >> 4) << 32;
    dsc |= (uint64_t)1u << 46;
    dsc |= (uint64_t)2u << 61;
    return dsc;
}


__device__ __forceinline__ float bits_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Epilogue of the token kinds for one 32-column chunk (32 rows of the expert):
// every epilogue thread stages its feature's 32 values in S (row-major
// [32 rows][128 features], fp32), then each thread takes 16-byte vectors of
// 8 features of one row. kDH: dg, du from dh and the saved g, u (read as
// vectors before any store: dgu overwrites gu in place); kDX: dx_perm rows.
__device__ __forceinline__ void g_store_rows(const GParams &p, const GItem &it, int m, int et,
                                             int c0, const uint32_t (&v)[32], float *S) {
#pragma unroll
    for (int j = 0; j < 32; ++j) S[j * 128 + m] = __uint_as_float(v[j]);
    named_bar_sync(1, 128);
    const size_t row_base = (size_t)it.dst_row0 + (size_t)it.nt * it.bn + c0;
    const int f0 = it.mt * 128;
    if (p.kind == kDH) {
        const size_t ld = 2 * (size_t)p.I;
        uint4 gv[4], uv[4];
        bool ok[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int idx = et + 128 * q, j = idx >> 4, fv = (idx & 15) * 8;
            ok[q] = c0 + j < it.n_valid && f0 + fv < p.I;
            if (ok[q]) {
                const uint16_t *src = p.gu + (row_base + j) * ld + f0 + fv;
                gv[q] = *reinterpret_cast<const uint4 *>(src);
                uv[q] = *reinterpret_cast<const uint4 *>(src + p.I);
            }
        }
        uint16_t *dgu = static_cast<uint16_t *>(p.out[0]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (!ok[q]) continue;
            const int idx = et + 128 * q, j = idx >> 4, fv = (idx & 15) * 8;
            const float4 d0 = *reinterpret_cast<const float4 *>(S + j * 128 + fv);
            const float4 d1 = *reinterpret_cast<const float4 *>(S + j * 128 + fv + 4);
            const float dh[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
            const uint32_t gw[4] = {gv[q].x, gv[q].y, gv[q].z, gv[q].w};
            const uint32_t uw[4] = {uv[q].x, uv[q].y, uv[q].z, uv[q].w};
            uint32_t og[4], ou[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float dg2[2], du2[2];
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const float g = b ? bf16_hi(gw[h]) : bf16_lo(gw[h]);
                    const float u = b ? bf16_hi(uw[h]) : bf16_lo(uw[h]);
                    const float sg = 1.0f / (1.0f + expf(-g));
                    const float x = dh[2 * h + b];
                    dg2[b] = x * u * sg * (1.0f + g * (1.0f - sg));
                    du2[b] = x * g * sg;
                }
                og[h] = pack_bf16x2(dg2[0], dg2[1]);
                ou[h] = pack_bf16x2(du2[0], du2[1]);
            }
            uint16_t *dst = dgu + (row_base + j) * ld + f0 + fv;
            *reinterpret_cast<uint4 *>(dst) = make_uint4(og[0], og[1], og[2], og[3]);
            *reinterpret_cast<uint4 *>(dst + p.I) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
        }
    } else {  // kDX
        uint16_t *dxp = static_cast<uint16_t *>(p.out[0]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int idx = et + 128 * q, j = idx >> 4, fv = (idx & 15) * 8;
            if (c0 + j >= it.n_valid || f0 + fv >= p.d) continue;
            const float4 a = *reinterpret_cast<const float4 *>(S + j * 128 + fv);
            const float4 b = *reinterpret_cast<const float4 *>(S + j * 128 + fv + 4);
            *reinterpret_cast<uint4 *>(dxp + (row_base + j) * p.d + f0 + fv) =
                make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                           pack_bf16x2(b.z, b.w));
        }
    }
    named_bar_sync(1, 128);  // S is rewritten by the next chunk
}

// Epilogue of one item: 32 accumulator columns (c0 ...) of TMEM lane `m`
// (M row m of the tile) in v; `zero`: the item had no K (an expert no token
// chose: its weight gradient is zero).
__device__ __forceinline__ void g_store(const GParams &p, const GItem &it, int m, int c0,
                                        const uint32_t (&v)[32], bool zero) {
    switch (p.kind) {
        case kLOGITS: {
            const int e = it.mt * 128 + m;
            if (e >= p.N) return;
            float *l = static_cast<float *>(p.out[0]) + (size_t)it.ks * p.T * p.N;
            const float b = (p.bias && it.ks == 0) ? p.bias[e] : 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int c = c0 + j;
                if (c >= it.n_valid) continue;
                l[(size_t)(it.nt * it.bn + c) * p.N + e] = __uint_as_float(v[j]) + b;
            }
            break;
        }
        case kDXR: {
            const int jf = it.mt * 128 + m;
            if (jf >= p.d) return;
            float *o = static_cast<float *>(p.out[0]);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int c = c0 + j;
                if (c >= it.n_valid) continue;
                o[(size_t)(it.nt * it.bn + c) * p.d + jf] = __uint_as_float(v[j]);
            }
            break;
        }
        default:  // weight gradients: staged and stored by TMA (g_store_wgrad)
            break;
    }
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap *m, const void *src, int c0, int c1,
                                             int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_3() {
    asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Weight-gradient epilogue of 64 columns (two 32-column chunks: va, and vb
// when `two`) for one warp: lane r holds row (32 q4 + r) of the tile; the warp
// writes its two [32][32] bf16 blocks into a pair of staging tiles (a ring of
// 4 pairs per warp; 64-byte swizzle, the output maps') and lane 0 stores them
// with TMA as one bulk group. Blocks wholly past the tensor are skipped; rows
// and columns partly past it are clipped by the copy.
__device__ __forceinline__ void g_stage_block(unsigned char *tile, int lane, const uint32_t (&v)[32]) {
    uint4 *dst = reinterpret_cast<uint4 *>(tile + lane * 64);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 o;
        o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
        o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
        o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
        o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
        dst[q ^ ((lane >> 1) & 3)] = o;  // 16-byte chunk q of row r at q ^ ((r >> 1) & 3)
    }
}

__device__ __forceinline__ void g_store_wgrad(const GParams &p, const GMaps &mp, const GItem &it,
                                              int q4, int lane, int c0, const uint32_t (&va)[32],
                                              const uint32_t (&vb)[32], bool two,
                                              unsigned char *pair) {
    const CUtensorMap *map;
    int row0, e, rows, cols;
    if (p.kind == kDWR) {
        map = &mp.m[6]; row0 = it.mt * 128; e = 0; rows = p.N; cols = p.d;
    } else {
        e = it.a_idx;
        if (p.kind == kDWD) {
            map = &mp.m[6 + it.a_sel]; row0 = it.mt * 128; rows = p.d; cols = p.I;
        } else {
            const int part = it.mt / p.m_tiles;
            map = &mp.m[6 + 2 * part + it.a_sel]; row0 = (it.mt - part * p.m_tiles) * 128;
            rows = p.I; cols = p.d;
        }
    }
    row0 += 32 * q4;
    const int col0 = it.nt * it.bn + c0;
    if (row0 >= rows || col0 >= cols) return;  // wholly past the tensor: nothing to store
    const bool second = two && col0 + 32 < cols;
    if (lane == 0) bulk_wait_read_3();  // this pair's previous stores have read it
    __syncwarp();
    g_stage_block(pair, lane, va);
    if (second) g_stage_block(pair + 2048, lane, vb);
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
        tma_store_3d(map, pair, col0, row0, e);
        if (second) tma_store_3d(map, pair + 2048, col0 + 32, row0, e);
        bulk_commit();
    }
}

__global__ void __launch_bounds__(kGThreads, 1) bwd_gemm_kernel(const __grid_constant__ GParams p,
                                                                 const __grid_constant__ GMaps mp) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    unsigned char *stages = smem;
    unsigned char *epi = smem + kGStages * kGStageBytes;
    GShared &sh = *reinterpret_cast<GShared *>(epi + kGEpiBytes);
    volatile int *abort = &sh.abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
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
    if (warp == 0 && lane == 0)
        for (int i = 0; i < 10; ++i) tma_prefetch_desc(&mp.m[i]);
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, kGTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sh.tmem_base;
    grid_dependency_wait();
    // item count (token kinds: from the plan's token tiles)
    if (threadIdx.x == 0) {
        int tot;
        if (g_token_kind(p.kind)) {
            tot = 0;
            for (int e = 0; e < p.n_entries; ++e) {
                sh.start[e] = tot;
                tot += p.m_tiles * p.ent[e].ntb;
            }
            sh.start[p.n_entries] = tot;
        } else if (g_wgrad_kind(p.kind)) {
            tot = p.n_entries * (p.kind == kDWGU ? 2 : 1) * p.m_tiles * p.n_tiles;
        } else {
            tot = p.m_tiles * p.n_tiles * (p.kind == kLOGITS ? p.ksplit : 1);
        }
        sh.total = tot;
    }
    __syncthreads();
    const int total = sh.total;
    const bool a_mn = g_a_mn(p.kind), b_mn = g_b_mn(p.kind);
    const int nst = p.nst;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        const uint64_t pol_a = policy_evict_first();
        const uint64_t pol_b = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_par = 0;
        bool ok = true;
        for (int q = blockIdx.x; q < total && ok; q += gridDim.x) {
            GItem it;
            g_decode(p, sh, q, it);
            int na, nb;
            uint32_t bytes;
            g_copies(p, it, na, nb, bytes);
            for (int kc = 0; kc < it.nck; ++kc) {
                int got = 1;
                if (lane == 0) got = mbar_wait(&sh.empty[stage], phase ^ 1u, abort);
                if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
                unsigned char *sbase = stages + stage * kGStageBytes;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sh.full[stage], bytes);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                }
                __syncwarp();
                if (lane < na + nb)
                    g_load(p, mp, it, kc, lane, na, sbase, &sh.full[stage], pol_a, pol_b);
                if (++stage == nst) { stage = 0; phase ^= 1u; }
            }
        }
        if (lane == 0 && *abort) {  // let every issued copy land before the CTA can exit
            for (int s = 0; s < kGStages; ++s)
                if (armed & (1u << s)) mbar_wait(&sh.full[s], (armed_par >> s) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        int stage = 0;
        uint32_t phase = 0;
        int i = 0;
        bool ok = true;
        for (int q = blockIdx.x; q < total && ok; q += gridDim.x, ++i) {
            GItem it;
            g_decode(p, sh, q, it);
            const int acc = i & 1;
            int got = 1;
            if (lane == 0) got = mbar_wait(&sh.tempty[acc], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort);
            if (!__shfl_sync(0xffffffffu, got, 0)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
            const uint32_t idesc = g_idesc(p.kind, (uint32_t)it.bn);
            for (int kc = 0; kc < it.nck; ++kc) {
                got = 1;
                if (lane == 0) got = mbar_wait(&sh.full[stage], phase, abort);
                if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
                unsigned char *sbase = stages + stage * kGStageBytes;
                int steps = 4;
                if (kc == it.nck - 1 && it.kv_last < 64) {
                    // ragged K: rows kv_last .. (next multiple of 16) of A hold the
                    // next expert's rows; zero them, skip the MMAs past them
                    __syncwarp();  // order the lanes after lane 0's wait (TMA has landed)
                    const int kv = it.kv_last;
                    steps = (kv + 15) / 16;
                    const int nz = 16 * steps - kv;  // rows to clear in each of A's two boxes
                    for (int z = lane; z < 2 * nz * 8; z += 32) {
                        const int box = z / (nz * 8), r = (z / 8) % nz, c16 = z % 8;
                        *reinterpret_cast<uint4 *>(sbase + 8192 * box + (kv + r) * 128 + 16 * c16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async();
                    __syncwarp();
                }
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t sa = smem_u32(sbase), sb = sa + 16384u;
                    for (int j = 0; j < steps; ++j) {
                        const uint32_t adv_a = a_mn ? 2048u * j : 32u * j;
                        const uint32_t adv_b = b_mn ? 2048u * j : 32u * j;
                        tc_mma_bf16(d_tmem, g_sdesc(sa + adv_a, a_mn), g_sdesc(sb + adv_b, b_mn), idesc,
                                    (kc + j) > 0 ? 1u : 0u);
                    }
                    tc_commit(&sh.empty[stage]);
                }
                __syncwarp();
                if (++stage == nst) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (lane == 0) tc_commit(&sh.tfull[acc]);  // (no MMA: arrives at once)
            __syncwarp();
        }
        if (lane == 0) {
            tc_commit(&sh.drain);
            mbar_wait(&sh.drain, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int q4 = warp & 3;
        const int m = 32 * q4 + lane;
        const bool wgrad = g_wgrad_kind(p.kind) || p.kind == kDWR;
        const bool rowk = g_token_kind(p.kind);
        const int et = threadIdx.x - 64;
        // weight-gradient staging (these kinds run 3 stages): the freed 4th stage and
        // the epilogue area, 64 KB, 16 KB per warp = 4 pairs of [32][32] bf16 tiles
        unsigned char *wstage = stages + (size_t)(kGStages - 1) * kGStageBytes + q4 * 16384;
        int i = 0, pairs = 0;
        for (int q = blockIdx.x; q < total; q += gridDim.x, ++i) {
            GItem it;
            g_decode(p, sh, q, it);
            const int acc = i & 1;
            // one thread waits and all 128 act on its result (the row epilogues meet
            // at named barriers, so they must all take or all skip an item)
            if (et == 0) sh.epi_ok = mbar_wait(&sh.tfull[acc], (uint32_t)(i >> 1) & 1u, abort) ? 1 : 0;
            named_bar_sync(1, 128);
            const int ok_item = *(volatile int *)&sh.epi_ok;
            named_bar_sync(1, 128);
            if (!ok_item) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q4) << 16) + (uint32_t)acc * 256u;
            const bool zero = it.nck == 0;
            if (wgrad) {  // 64 columns per TMEM wait, two staging tiles, one store group
                for (int c0 = 0; c0 < it.n_valid; c0 += 64) {
                    const bool two = c0 + 32 < it.n_valid;
                    uint32_t va[32], vb[32];
                    if (!zero) {
                        tmem_ld_32x32b_x32(tbase + (uint32_t)c0, va);
                        if (two) tmem_ld_32x32b_x32(tbase + (uint32_t)c0 + 32u, vb);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) va[j] = vb[j] = 0u;
                    }
                    g_store_wgrad(p, mp, it, q4, lane, c0, va, vb, two,
                                  wstage + (size_t)(pairs & 3) * 4096);
                    ++pairs;
                }
            }
            for (int c0 = 0; !wgrad && c0 < it.n_valid; c0 += 32) {
                uint32_t v[32];
                if (!zero) {
                    tmem_ld_32x32b_x32(tbase + (uint32_t)c0, v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = 0u;
                }
                if (rowk) {
                    g_store_rows(p, it, m, et, c0, v, reinterpret_cast<float *>(epi));
                } else {
                    g_store(p, it, m, c0, v, zero);
                }
            }
            tc_fence_before();
            mbar_arrive(&sh.tempty[acc]);
        }
        if (lane == 0) bulk_wait_all();  // every gradient store has completed
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kGTmemCols);
}

// ---------------------------------------------------------------------------
// Host side.
static bool g_rows(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                   uint32_t box_rows = 64) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    return encode(m, base, 2, dims, strides, box);
}
// MN-major view of a row-major bf16 [rows][cols] matrix (cols % 64 == 0):
// {64 columns, rows, cols / 64 column blocks}, the blocks 128 bytes apart; a
// {64, 64, nblk} box lands nblk 64-column blocks of 64 rows one after
// another, 8 KB apart
static bool g_rows_mn(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                      uint32_t nblk) {
    const cuuint64_t dims[3] = {64, rows, cols / 64};
    const cuuint64_t strides[2] = {cols * 2, 128};
    const cuuint32_t box[3] = {64, 64, nblk};
    return encode(m, base, 3, dims, strides, box);
}
// the same view of [E][rows][cols] expert matrices: {64, rows, cols / 64, E}
static bool g_experts_mn(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                         uint64_t E, uint32_t nblk) {
    const cuuint64_t dims[4] = {64, rows, cols / 64, E};
    const cuuint64_t strides[3] = {cols * 2, 128, cols * rows * 2};
    const cuuint32_t box[4] = {64, 64, nblk, 1};
    return encode(m, base, 4, dims, strides, box);
}
static bool g_experts(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t E) {
    const cuuint64_t dims[3] = {cols, rows, E};
    const cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
    const cuuint32_t box[3] = {64, 64, 1};
    return encode(m, base, 3, dims, strides, box);
}
// N tiles of at most 256 columns over n columns, each a multiple of 16 wide
static void g_ntiles(int n, int &tiles, int &bn, int align = 16) {
    tiles = (n + 255) / 256;
    if (tiles < 1) tiles = 1;
    bn = (((n + tiles - 1) / tiles) + align - 1) / align * align;
    if (bn < align) bn = align;
}
// N tiles of 64-column blocks (a wide B copy starts on a block): the width
// out of 256, 192, 128, 64 that covers n with the fewest columns (the widest
// on a tie)
static void g_ntiles64(int n, int &tiles, int &bn) {
    int best = 0;
    for (int w = 256; w >= 64; w -= 64) {
        const int t = (n + w - 1) / w;
        if (best == 0 || t * w < tiles * bn) { tiles = t; bn = w; best = 1; }
    }
}
// bf16 [E][rows][cols] gradient written in [32 rows][32 cols] boxes (64-byte swizzle)
static bool g_out(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t E) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {cols, rows, E};
    const cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K parts of the recomputed router logits: enough items for the SMs (the
// GEMM is small: one or two 128-row tiles of experts), at most kMaxLogitSplit
int logits_ksplit(const moge_config &c, int num_sms) {
    const int tiles = ((c.N + 127) / 128) * ((c.T + 255) / 256);
    const int kc = (c.d + 63) / 64;
    int ks = num_sms / (tiles > 0 ? tiles : 1);
    ks = ks < kMaxLogitSplit ? ks : kMaxLogitSplit;
    ks = ks < kc / 2 ? ks : kc / 2;
    return ks > 1 ? ks : 1;
}

static size_t g_smem_bytes() {
    return 1024 + (size_t)kGStages * kGStageBytes + kGEpiBytes + sizeof(GShared);
}

cudaError_t launch_bwd_gemm(int kind, const moge_config &c, const ExpertWork *ent, int n_entries,
                            const BwdTensors &b, int num_sms, cudaStream_t st) {
    const int T = c.T, d = c.d, I = c.I, N = c.N, S = c.S;
    const int K = c.M * c.Kp;
    const uint64_t rrows = (uint64_t)T * K, hrows = (uint64_t)T * (K + S);
    // a missing shared side borrows the routed tensors (no entry selects it)
    const void *sg = S ? b.sg : b.wg, *su = S ? b.su : b.wu, *sd = S ? b.sd : b.wd;
    const int ns = S ? S : N;
    GMaps mp;
    GParams p = {};
    p.kind = kind;
    p.ent = ent;
    p.n_entries = n_entries;
    p.T = T; p.d = d; p.I = I; p.N = N;
    bool ok = true;
    int total = -1;  // unknown on the host (token kinds)
    switch (kind) {
        case kDH:
            p.a_wide = I % 64 == 0;
            ok = (p.a_wide ? g_experts_mn(&mp.m[0], b.wd, I, d, N, 2) &&
                                 g_experts_mn(&mp.m[1], sd, I, d, ns, 2)
                           : g_experts(&mp.m[0], b.wd, I, d, N) && g_experts(&mp.m[1], sd, I, d, ns)) &&
                 g_rows(&mp.m[2], b.dy_perm, d, rrows, 128) && g_rows(&mp.m[3], b.dy, d, T, 128);
            mp.m[4] = mp.m[5] = mp.m[0];
            p.m_tiles = (I + 127) / 128;
            p.kc = (d + 63) / 64;
            p.out[0] = b.dgu;
            p.gu = (const uint16_t *)b.gu;
            break;
        case kDX:
            p.a_wide = d % 64 == 0;
            ok = (p.a_wide ? g_experts_mn(&mp.m[0], b.wg, d, I, N, 2) &&
                                 g_experts_mn(&mp.m[1], sg, d, I, ns, 2) &&
                                 g_experts_mn(&mp.m[2], b.wu, d, I, N, 2) &&
                                 g_experts_mn(&mp.m[3], su, d, I, ns, 2)
                           : g_experts(&mp.m[0], b.wg, d, I, N) && g_experts(&mp.m[1], sg, d, I, ns) &&
                                 g_experts(&mp.m[2], b.wu, d, I, N) &&
                                 g_experts(&mp.m[3], su, d, I, ns)) &&
                 g_rows(&mp.m[4], b.dgu, 2 * (uint64_t)I, hrows, 128);
            mp.m[5] = mp.m[0];
            p.m_tiles = (d + 127) / 128;
            p.kc = 2 * I / 64;
            p.out[0] = b.dx_perm;
            break;
        case kDWD:
            p.a_wide = d % 64 == 0;
            p.b_wide = I % 64 == 0;
            if (p.b_wide) g_ntiles64(I, p.n_tiles, p.bn);
            else g_ntiles(I, p.n_tiles, p.bn, 32);
            ok = (p.a_wide ? g_rows_mn(&mp.m[0], b.dy_perm, d, rrows, 2) &&
                                 g_rows_mn(&mp.m[1], b.dy, d, T, 2)
                           : g_rows(&mp.m[0], b.dy_perm, d, rrows) && g_rows(&mp.m[1], b.dy, d, T)) &&
                 (p.b_wide ? g_rows_mn(&mp.m[2], b.h, I, hrows, (uint32_t)p.bn / 64)
                           : g_rows(&mp.m[2], b.h, I, hrows));
            ok = ok && g_out(&mp.m[6], b.dwd, I, d, N) && g_out(&mp.m[7], S ? b.dsd : b.dwd, I, d, ns);
            mp.m[3] = mp.m[4] = mp.m[5] = mp.m[0];
            mp.m[8] = mp.m[9] = mp.m[6];
            p.m_tiles = (d + 127) / 128;
            p.out[0] = b.dwd; p.out[1] = b.dsd;
            total = n_entries * p.m_tiles * p.n_tiles;
            break;
        case kDWGU:
            p.a_wide = I % 64 == 0;
            p.b_wide = d % 64 == 0;
            if (p.b_wide) g_ntiles64(d, p.n_tiles, p.bn);
            else g_ntiles(d, p.n_tiles, p.bn, 32);
            ok = (p.a_wide ? g_rows_mn(&mp.m[0], b.dgu, 2 * (uint64_t)I, hrows, 2)
                           : g_rows(&mp.m[0], b.dgu, 2 * (uint64_t)I, hrows)) &&
                 (p.b_wide ? g_rows_mn(&mp.m[2], b.x_perm, d, rrows, (uint32_t)p.bn / 64) &&
                                 g_rows_mn(&mp.m[3], b.x, d, T, (uint32_t)p.bn / 64)
                           : g_rows(&mp.m[2], b.x_perm, d, rrows) && g_rows(&mp.m[3], b.x, d, T));
            ok = ok && g_out(&mp.m[6], b.dwg, d, I, N) && g_out(&mp.m[7], S ? b.dsg : b.dwg, d, I, ns) &&
                 g_out(&mp.m[8], b.dwu, d, I, N) && g_out(&mp.m[9], S ? b.dsu : b.dwu, d, I, ns);
            mp.m[1] = mp.m[4] = mp.m[5] = mp.m[0];
            p.m_tiles = (I + 127) / 128;
            p.out[0] = b.dwg; p.out[1] = b.dsg; p.out[2] = b.dwu; p.out[3] = b.dsu;
            total = n_entries * 2 * p.m_tiles * p.n_tiles;
            break;
        case kLOGITS:
            ok = g_rows(&mp.m[0], b.w_router, d, N) && g_rows(&mp.m[1], b.x, d, T);
            mp.m[2] = mp.m[3] = mp.m[4] = mp.m[5] = mp.m[0];
            p.m_tiles = (N + 127) / 128;
            p.kc = (d + 63) / 64;
            g_ntiles(T, p.n_tiles, p.bn);
            p.out[0] = b.logits;
            p.bias = b.bias;
            p.ksplit = logits_ksplit(c, num_sms);
            total = p.m_tiles * p.n_tiles * p.ksplit;
            break;
        case kDWR:
            ok = g_rows(&mp.m[0], b.dl, N, T) && g_rows(&mp.m[1], b.x, d, T) &&
                 g_out(&mp.m[6], b.dwr, d, N, 1);
            mp.m[2] = mp.m[3] = mp.m[4] = mp.m[5] = mp.m[0];
            mp.m[7] = mp.m[8] = mp.m[9] = mp.m[6];
            p.m_tiles = (N + 127) / 128;
            g_ntiles(d, p.n_tiles, p.bn, 32);
            p.out[0] = b.dwr;
            total = p.m_tiles * p.n_tiles;
            break;
        case kDXR:
            ok = g_rows(&mp.m[0], b.w_router, d, N) && g_rows(&mp.m[1], b.dl, N, T);
            mp.m[2] = mp.m[3] = mp.m[4] = mp.m[5] = mp.m[0];
            p.m_tiles = (d + 127) / 128;
            p.kc = (N + 63) / 64;
            g_ntiles(T, p.n_tiles, p.bn);
            p.out[0] = b.dx_r;
            total = p.m_tiles * p.n_tiles;
            break;
        default:
            return cudaErrorInvalidValue;
    }
    if (!ok) return cudaErrorInvalidValue;
    p.nst = (kind == kDWD || kind == kDWGU || kind == kDWR) ? 3 : kGStages;
    if (kind == kDH || kind == kDX || kind == kLOGITS || kind == kDXR)
        mp.m[6] = mp.m[7] = mp.m[8] = mp.m[9] = mp.m[0];  // no gradient output (never stored to)
    if (total == 0) return cudaSuccess;
    const int grid = total < 0 ? num_sms : (total < num_sms ? total : num_sms);
    const size_t smem = g_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(bwd_gemm_kernel, dim3(grid), dim3(kGThreads), smem, st, p, mp);
}

}  // namespace moge
