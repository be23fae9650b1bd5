// Internal declarations shared by the MoGE CUDA sources: the grouped-GEMM
// work plan, the workspace layout and the kernel launchers used by api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/moge.h"

namespace moge {

// Tokens handled by one router tile (one CTA, or one cluster of CTAs that
// split the hidden dimension).
constexpr int kRouterTile = 16;
constexpr int kMaxExperts = 256;

// One expert's block of rows in a grouped GEMM launch.
//   rows      rows of this expert (routed: counts[e]; shared: T)
//   src_row0  first row in the B-operand matrix (x_perm / x / h)
//   dst_row0  first row in the output matrix (h / y_perm)
//   a_sel     0: routed weight tensors, 1: shared weight tensors
//   a_idx     expert index inside the selected weight tensor
//   b_sel     0: first B matrix (x_perm, or h), 1: second (x)
//   bn        token-tile width (multiple of 16, <= 256)
//   ntb       token tiles of this expert (ceil(rows / bn)), 0 if rows == 0
struct ExpertWork {
    int rows, src_row0, dst_row0, a_sel, a_idx, b_sel, bn, ntb;
};

// Token-tile widths: an expert with at most kStreamRows rows is one
// "streaming" tile (two K-chunks per pipeline stage, weights are the
// bandwidth-bound stream); larger experts use tensor tiles of up to 256 rows.
constexpr int kStreamRows = 64;
constexpr int kMaxTileN = 256;

// Work plan of one layer call: an up-projection list and a down-projection list.
struct Plan {
    ExpertWork *up;     // [n_entries]
    ExpertWork *down;   // [n_entries]
    int *up_start;      // [n_entries + 1] prefix sum of items (ntb * feature blocks)
    int *down_start;    // [n_entries + 1]
    int *sync;          // [n_entries + 2] work-queue counter, per-entry finished
                        // up-projection items, and the CTAs done with a permute done
                        // inside the grouped GEMM ([n_entries + 1]); zeroed by the
                        // kernel that writes the plan
};

// Workspace carve-up (all regions 256-byte aligned).
struct Workspace {
    int32_t *hist;      // [tiles][N] per-tile expert counts
    int32_t *base;      // [tiles][N] rows of expert e taken by earlier tiles
    int32_t *rank;      // [T][K]     rank of (t, k) among its tile's tokens of that expert
    int32_t *topk_idx;  // [T][K]
    float *topk_w;      // [T][K]
    int32_t *counts;    // [N]
    int32_t *offsets;   // [N+1]
    int32_t *perm_src;  // [T*K]
    int32_t *perm_dst;  // [T][K]
    Plan plan;          // N + S entries per list
    void *x_perm;       // [T*K][d]      dtype
    void *h;            // [T*(K+S)][I]  dtype
    void *y_perm;       // [T*(K+S)][d]  dtype
    size_t total;
};
Workspace carve_workspace(const moge_config &c, void *base);

// Launch with programmatic stream serialisation (the kernel starts its
// prologue while the previous kernel on the stream drains; every kernel of
// this library calls grid_dependency_wait() before its first global access),
// optionally as clusters of `cluster` CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- launchers
// Each returns a cudaError_t of the launch.
cudaError_t launch_router(const moge_config &c, const void *x, const void *w_router,
                          const float *bias, int32_t *topk_idx, float *topk_w, int32_t *hist,
                          int32_t *rank, int num_sms, cudaStream_t st);
// counts/offsets/base from hist; when plan_* are given also the layer's GEMM plan
// (token tiles of the plan: at most max_tile rows each)
cudaError_t launch_scan(const moge_config &c, const int32_t *hist, int32_t *base, int32_t *counts,
                        int32_t *offsets, const Plan *plan, bool with_routed, bool with_shared,
                        cudaStream_t st, int max_tile = kMaxTileN);
// plan from caller offsets (routed only) or for shared experts only
cudaError_t launch_plan(const moge_config &c, const int32_t *offsets, const Plan &plan,
                        bool with_routed, bool with_shared, cudaStream_t st);
cudaError_t launch_finalize(const moge_config &c, const int32_t *topk_idx, const int32_t *rank,
                            const int32_t *base, const int32_t *offsets, int32_t *perm_src,
                            int32_t *perm_dst, cudaStream_t st);
cudaError_t launch_scatter_rows(const moge_config &c, const void *x, const int32_t *topk_idx,
                                const int32_t *rank, const int32_t *base, const int32_t *offsets,
                                int32_t *perm_src, int32_t *perm_dst, void *x_perm,
                                cudaStream_t st);
cudaError_t launch_gather_rows(const moge_config &c, const void *x, const int32_t *perm_src,
                               void *x_perm, cudaStream_t st);
cudaError_t launch_combine(const moge_config &c, const void *y_perm, const float *topk_w,
                           const int32_t *perm_dst, int K, const void *shared_rows,
                           int n_shared_blocks, const void *residual, void *y, cudaStream_t st,
                           bool out_f32 = false);
cudaError_t launch_rmsnorm(const moge_config &c, const void *x, float eps, void *u,
                           cudaStream_t st);

// Grouped SwiGLU FFN over a plan list (n_entries experts).
struct FfnOperands {
    const void *b0;          // up: x_perm (routed rows) ; down: h
    const void *b1;          // up: x (shared rows)      ; down: unused
    int64_t b0_rows, b1_rows;
    const void *wg, *wu, *wd;  // routed weights [N][I][d], [N][I][d], [N][d][I]
    const void *sg, *su, *sd;  // shared weights [S][I][d], [S][I][d], [S][d][I]
    void *h;                 // [h_rows][I]
    int64_t h_rows;
    void *y;                 // [h_rows][d]
    // Optional (bf16 tensor-core FFN only, training forward): the
    // up-projection's pre-activations, [h_rows][2I] = [g | u] per row.
    void *gu;
    // Optional (bf16 tensor-core FFN only): the permute done inside the grouped
    // GEMM launch -- x_perm (b0) is written from x (b1) by the kernel's epilogue
    // warps before their first item, with the indices below (as the scatter
    // kernel computes them); the routed up-projection items wait for it.
    const int32_t *pm_topk_idx, *pm_rank, *pm_base, *pm_offsets;
    int32_t *pm_perm_src, *pm_perm_dst;
    // FP8 weights only (launch_ffn_fp8): the w*/s* pointers above are E4M3
    // codes and these their per-row fp32 scales ([E][I], [E][I], [E][d])
    const float *wg_s, *wu_s, *wd_s;
    const float *sg_s, *su_s, *sd_s;
    // W8A8 only (launch_ffn_w8a8): b0 / b1 are E4M3 token rows with these
    // per-row scales, h receives the h codes ([h_rows][I] bytes); h32
    // ([h_rows][I] fp32), hmax ([h_rows], zeroed beforehand) and sh ([h_rows])
    // hold h before quantisation, its row amax and its row scales
    const float *cs_b0, *cs_b1;
    void *h32;
    uint32_t *hmax;
    float *sh;
};
// `mid` (may be null) is recorded on the stream between the up- and the
// down-projection launches.
cudaError_t launch_ffn_tc(const moge_config &c, const Plan &plan, int n_entries,
                          const FfnOperands &op, int num_sms, cudaStream_t st, cudaEvent_t mid);
cudaError_t launch_ffn_w8a8(const moge_config &c, const Plan &plan, int n_entries,
                            const FfnOperands &op, int num_sms, cudaStream_t st);
// W8A8 activations: per token t, scale sx[t] = amax / 448 of x's bf16 row
// (fp32; 1 for a zero row) and the row's E4M3 codes into x8[t] and into each
// of its K routed rows of x8p (sxp the same scale), with perm_src / perm_dst
// as launch_scatter_rows; zeroes the amax word of each of the token's h rows
// (hmax [T (K + S)]).
cudaError_t launch_quantize_scatter(const moge_config &c, const void *x, const int32_t *topk_idx,
                                    const int32_t *rank, const int32_t *base,
                                    const int32_t *offsets, int32_t *perm_src, int32_t *perm_dst,
                                    void *x8, float *sx, void *x8p, float *sxp, uint32_t *hmax,
                                    cudaStream_t st);
cudaError_t launch_ffn_f32(const moge_config &c, const Plan &plan, int n_entries,
                           const FfnOperands &op, cudaStream_t st, cudaEvent_t mid);
namespace pair {
// The same grouped FFN on CTA pairs (2-SM tcgen05 MMA, M = 256): bf16, no
// permute inside the launch (g/u kept when op.gu is set); used for
// prefill-sized batches.
cudaError_t launch_ffn_tc_pair(const moge_config &c, const Plan &plan, int n_entries,
                               const FfnOperands &op, int num_sms, cudaStream_t st);
}  // namespace pair
// grouped FFN with FP8 (E4M3, per-row scale) weights and bf16 activations
cudaError_t launch_ffn_fp8(const moge_config &c, const Plan &plan, int n_entries,
                           const FfnOperands &op, int num_sms, cudaStream_t st);

// ---------------------------------------------------------------- backward
// Tensors of the backward pass (bf16 unless noted; rows as in the forward:
// rrows = T*K routed rows in permuted order, hrows = T*(K+S) with the shared
// experts' rows after the routed ones).
struct BwdTensors {
    const void *x, *w_router;            // [T][d], [N][d]
    const float *bias;                   // [N] or null
    const void *wg, *wu, *wd;            // routed weights [N][I][d], [N][I][d], [N][d][I]
    const void *sg, *su, *sd;            // shared weights (null when S == 0)
    const void *x_perm, *h;              // [rrows][d], [hrows][I]   (forward)
    const void *gu;                      // [hrows][2I] pre-activations [g | u] (forward)
    const void *dy, *dy_perm;            // [T][d], [rrows][d]
    void *dgu;                           // [hrows][2I] (may alias gu)
    void *dx_perm;                       // [hrows][d]
    float *logits;                       // [T][N] fp32
    void *dl;                            // [T][N]
    float *dx_r;                         // [T][d] fp32
    void *dwg, *dwu, *dwd, *dsg, *dsu, *dsd, *dwr;  // weight gradients (layouts of the weights)
};
// GEMM kinds of the backward pass: dh (with the SwiGLU backward), dx, dW_down,
// dW_gate / dW_up, the router's logits, dW_router, the router's share of dx
enum : int { kDH = 0, kDX = 1, kDWD = 2, kDWGU = 3, kLOGITS = 4, kDWR = 5, kDXR = 6 };
cudaError_t launch_bwd_gemm(int kind, const moge_config &c, const ExpertWork *ent, int n_entries,
                            const BwdTensors &b, int num_sms, cudaStream_t st);
// K parts of the backward's router-logit GEMM (each writes its own [T][N]
// partial, summed in order by the router backward); at most kMaxLogitSplit
constexpr int kMaxLogitSplit = 16;
int logits_ksplit(const moge_config &c, int num_sms);
cudaError_t launch_combine_bwd(const moge_config &c, const void *dy, const void *y_perm,
                               const float *topk_w, const int32_t *perm_dst, void *dy_perm,
                               float *dw, cudaStream_t st);
int router_bwd_parts(const moge_config &c);
cudaError_t launch_router_bwd(const moge_config &c, float alpha, const float *logits, int ksplit,
                              const int32_t *topk_idx, const float *dw, const int32_t *counts,
                              void *dl, float *part, float *aux, cudaStream_t st);
cudaError_t launch_unpermute_bwd(const moge_config &c, const void *dx_perm, const int32_t *perm_dst,
                                 const float *dx_r, void *dx, cudaStream_t st);

// kernel whose bounded waits run out after limit_ns (failure-path check)
cudaError_t launch_wait_selftest(int32_t *out, uint64_t limit_ns, cudaStream_t st);
// per-row FP8 quantisation of bf16 rows
cudaError_t launch_quantize_fp8(const void *w, int64_t rows, int64_t cols, void *q, float *scale,
                                cudaStream_t st);

// ---------------------------------------------------------------- expert parallelism
cudaError_t launch_localize(int T, int N, int K, int k0, int K_loc, int e0, int N_loc, int tiles,
                            const int32_t *topk_idx, const float *topk_w, const int32_t *rank,
                            const int32_t *hist, int32_t *idx_loc, float *w_loc, int32_t *rank_loc,
                            int32_t *hist_loc, cudaStream_t st);
cudaError_t launch_ep_finish(int dtype, long long rows, int d, const float *y_sum,
                             const void *residual, void *y, cudaStream_t st);

}  // namespace moge
