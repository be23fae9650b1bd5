/*
 * moge.h -- C ABI of the MoGE (Mixture of Grouped Experts) FFN layer forward
 * pass for NVIDIA B200 (sm_100a).
 *
 * The operation (restated from "Huawei releases Pangu Pro MoE: the first 72B
 * sparse language model, designed for Ascend NPUs", techwalker.com,
 * section 1 "Innovative architecture", and section 2 for the shared experts):
 *
 *   for every token t, with x_t its hidden vector (length d):
 *     l_e   = x_t . w_router[e] (+ logit_bias[e])          e = 0 .. N-1
 *     p     = softmax(l) over ALL N experts (global softmax, before selection)
 *     group g holds experts [g*G, (g+1)*G), G = N/M; inside EVERY group the
 *     Kp = K/M experts with the largest p are picked (ties: lower index)
 *     y_t   = sum_{picked e} p_e * FFN_e(x_t)  +  sum_{s<S} FFN_s(x_t)
 *     FFN(x) = W_down (silu(W_gate x) * (W_up x)),  silu(z) = z / (1 + e^-z)
 *
 * Every group receives exactly T*Kp (token, expert) assignments, so the
 * per-group load is equal by construction (imbalance score 0). The picked
 * weights are NOT renormalised; shared experts enter with weight 1.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are caller-owned DEVICE pointers on the current CUDA
 *    device, 16-byte aligned, row-major, densely packed. The library never
 *    allocates device memory in these calls and never synchronises the host
 *    (except moge_check_device_errors).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it.
 *  - dtype MOGE_BF16: x, weights and every activation are bf16 (bit patterns,
 *    2 bytes); router logits, softmax, SwiGLU epilogue and all sums are fp32.
 *    dtype MOGE_F32: everything is fp32 (CUDA-core arithmetic, no TF32).
 *    Scores (topk_w) and logit_bias are always fp32; indices are int32.
 *  - Return value: MOGE_OK or an error code; nothing is enqueued when a host
 *    check fails. moge_last_error() gives a message (thread-local).
 *    Errors found by the kernels (a bounded wait that timed out, a violated
 *    routing invariant) are recorded in a device-side word and reported by
 *    moge_check_device_errors().
 *
 * Weight layouts follow the nn.Linear [out][in] convention:
 *   w_router [N][d]; w_gate, w_up [N][I][d]; w_down [N][d][I]
 *   s_gate, s_up [S][I][d]; s_down [S][d][I]
 * Size limits: 1 <= N <= 256, 0 <= S <= 256, N % M == 0, 1 <= Kp <= N/M, d % 8 == 0,
 * I % 8 == 0, T*(M*Kp+S) < 2^31 (else MOGE_ERR_UNSUPPORTED).
 */
#ifndef MOGE_H
#define MOGE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOGE_API __attribute__((visibility("default")))
#else
#define MOGE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOGE_OK 0
#define MOGE_ERR_INVALID_ARG 1 /* null pointer, negative size, bad dtype */
#define MOGE_ERR_UNSUPPORTED 2 /* a size limit above, or a misaligned pointer */
#define MOGE_ERR_CUDA 3        /* a CUDA runtime/driver call failed */
#define MOGE_ERR_TIMEOUT 4     /* a bounded device wait gave up (device word) */
#define MOGE_ERR_DEVICE 5      /* a kernel found a violated invariant (device word) */

#define MOGE_F32 0
#define MOGE_BF16 1

typedef struct moge_config {
    int T;     /* tokens in the batch (>= 0) */
    int d;     /* hidden size */
    int N;     /* routed experts */
    int M;     /* groups (N/M experts each) */
    int Kp;    /* experts picked per group per token (K = M*Kp per token) */
    int S;     /* always-on shared experts (>= 0) */
    int I;     /* SwiGLU intermediate size of every expert */
    int dtype; /* MOGE_BF16 or MOGE_F32 */
} moge_config;

/* Bytes of device workspace the calls below need for this configuration
 * (0 for an invalid one). The caller allocates it once (256-byte aligned) and
 * may reuse it across calls on the same stream. */
MOGE_API size_t moge_workspace_size(const moge_config *cfg);

/* Message of the last failing call on this host thread ("" if none). */
MOGE_API const char *moge_last_error(void);

/* Synchronises `stream`, reads and clears the device error word of the
 * current device: MOGE_OK, MOGE_ERR_TIMEOUT or MOGE_ERR_DEVICE. */
MOGE_API int moge_check_device_errors(void *stream);

/* Routing: router GEMM, global fp32 softmax, per-group top-Kp, per-expert
 * counts and the expert-major permutation (section 1 of the article above;
 * equal per-group load from the reportify "mixture of grouped experts" page).
 *   x [T][d] dtype, w_router [N][d] dtype, logit_bias [N] fp32 or NULL
 *   out topk_idx [T][K] int32  picks, group-major, descending score inside a group
 *   out topk_w   [T][K] fp32   the picks' global softmax scores (no renorm)
 *   out counts   [N]    int32  assignments per expert
 *   out offsets  [N+1]  int32  exclusive prefix sum of counts (offsets[N] = T*K)
 *   out perm_src [T*K]  int32  token held by each expert-major row
 *   out perm_dst [T][K] int32  expert-major row of each (token, pick)
 * Rows of one expert keep ascending token order. */
MOGE_API int moge_route(const moge_config *cfg, const void *x, const void *w_router,
               const float *logit_bias, int32_t *topk_idx, float *topk_w, int32_t *counts,
               int32_t *offsets, int32_t *perm_src, int32_t *perm_dst, void *workspace,
               void *stream);

/* Permute: x_perm[r] = x[perm_src[r]] for r < T*K (rows of d, dtype).
 * The dispatch of every token to the K' picked experts of each group
 * (techwalker.com article, section 1: every group receives the tokens routed
 * to its experts), laid out expert by expert as the grouped matmul of
 * section 3 reads it. Rows of one expert in ascending token order. */
MOGE_API int moge_permute(const moge_config *cfg, const void *x, const int32_t *perm_src, void *x_perm,
                 void *stream);

/* Grouped routed-expert FFN over expert-major rows: for every expert e and
 * row r in [offsets[e], offsets[e+1]):
 *   y_perm[r] = W_down[e] (silu(W_gate[e] x_perm[r]) * (W_up[e] x_perm[r]))
 * The grouped expert matmul ("GroupMatmul", whose SwiftGMM kernel picks a
 * GEMV- or GEMM-like path by load: techwalker.com article, section 3, and the
 * reportify.cn product digest); the pages do not give the expert's internals,
 * the SwiGLU form is this library's reading.
 * x_perm, y_perm [T*K][d] dtype; offsets [N+1] int32 on the device.
 * bf16: tcgen05 tensor-core GEMMs (TMA-fed, TMEM accumulators), the SwiGLU
 * product rounded to bf16 between the two GEMMs; above 8192 rows (T*K) on CTA
 * pairs (2-SM MMA), as in moge_layer_forward. */
MOGE_API int moge_grouped_ffn(const moge_config *cfg, const void *x_perm, const int32_t *offsets,
                     const void *w_gate, const void *w_up, const void *w_down, void *y_perm,
                     void *workspace, void *stream);

/* Shared experts: y_shared[t] = sum_{s<S} FFN_s(x[t]); x, y_shared [T][d].
 * The always-on shared experts (techwalker.com article, section 2: 4 shared
 * beside the 64 routed experts; mokono.cn news page, item 1), each an FFN of
 * the routed experts' form, entering with weight 1. Above 8192 rows (T*S) on
 * CTA pairs. */
MOGE_API int moge_shared_ffn(const moge_config *cfg, const void *x, const void *s_gate,
                    const void *s_up, const void *s_down, void *y_shared, void *workspace,
                    void *stream);

/* Combine: y[t] = residual[t] + sum_{k<K} topk_w[t][k] * y_perm[perm_dst[t][k]]
 *                 + y_shared[t]
 * The picked experts' outputs weighted by their global softmax scores
 * (techwalker.com article, section 1; no renormalisation) plus the shared
 * experts' (section 2). Summed in fp32 in this order (k ascending); residual
 * and y_shared may be NULL (treated as zero). y may alias residual. */
MOGE_API int moge_combine(const moge_config *cfg, const void *y_perm, const float *topk_w,
                 const int32_t *perm_dst, const void *y_shared, const void *residual, void *y,
                 void *stream);

/* Whole layer: route, permute, one grouped-FFN launch covering both
 * projections of routed AND shared experts, combine. bf16: up to 8192 routed
 * rows (T*K) the FFN launch also does the permute and runs one CTA per SM;
 * larger batches run it on CTA pairs (2-SM tcgen05 MMA, 256 weight rows per
 * item). Both give results within the same tolerance of the oracle.
 *   y[t] = residual[t] (if not NULL) + MoGE(x)[t];  y may alias residual, not x.
 * s_* may be NULL when S == 0; logit_bias may be NULL. The routing of the
 * call stays readable in the workspace (moge_workspace_routing). */
MOGE_API int moge_layer_forward(const moge_config *cfg, const void *x, const void *w_router,
                       const float *logit_bias, const void *w_gate, const void *w_up,
                       const void *w_down, const void *s_gate, const void *s_up,
                       const void *s_down, const void *residual, void *y, void *workspace,
                       void *stream);

/* moge_layer_forward with x and y in HOST memory (pinned for full speed):
 * copies x in, runs the layer, copies y out, all on `stream`, and returns after
 * synchronising the stream. Weights and workspace stay device pointers. */
MOGE_API int moge_layer_forward_host(const moge_config *cfg, const void *x_host, const void *w_router,
                            const float *logit_bias, const void *w_gate, const void *w_up,
                            const void *w_down, const void *s_gate, const void *s_up,
                            const void *s_down, void *y_host, void *x_dev, void *y_dev,
                            void *workspace, void *stream);

/* A run of independent batches through the layer from and to host memory,
 * with the copies overlapped with the compute: batch i's input x_host + i*T*d
 * is copied in while batch i-1 is computed and batch i-2's output copied out
 * (a host-to-device and a device-to-host stream of the library's own, per
 * device, ordered by events; the layer runs on `stream`). x_host, y_host:
 * [n_batches][T][d] in cfg->dtype, page-locked for the copies to overlap;
 * x_dev2, y_dev2: caller-owned device buffers of 2*T*d elements (two per
 * direction). Returns after every output has arrived in y_host. Same weights,
 * workspace and rules as moge_layer_forward (no residual). The copy streams
 * are shared by the calls on one device: do not run two such calls on one
 * device at the same time (from two host threads). */
MOGE_API int moge_layer_forward_host_stream(const moge_config *cfg, int64_t n_batches,
                                            const void *x_host, const void *w_router,
                                            const float *logit_bias, const void *w_gate,
                                            const void *w_up, const void *w_down,
                                            const void *s_gate, const void *s_up,
                                            const void *s_down, void *y_host, void *x_dev2,
                                            void *y_dev2, void *workspace, void *stream);

/* Device pointers, inside `workspace`, of the routing written by the last
 * moge_layer_forward on it: topk_idx [T][K], topk_w [T][K], counts [N],
 * offsets [N+1] (any out pointer may be NULL). Host-only arithmetic. */
MOGE_API int moge_workspace_routing(const moge_config *cfg, void *workspace, int32_t **topk_idx,
                           float **topk_w, int32_t **counts, int32_t **offsets);

/* RMSNorm with unit gain, per row of x [T][d] (dtype): u = x / sqrt(mean(x^2) + eps),
 * fp32 arithmetic (pre-norm of a stack of MoGE blocks; RMSNorm is named in
 * section 2 of the article above, its form here is a stated choice). */
MOGE_API int moge_rmsnorm(const moge_config *cfg, const void *x, float eps, void *u, void *stream);

/* moge_route without a workspace, for callers that may not allocate device
 * memory on their calling path (a plugin inside a runtime whose device memory
 * is all pre-reserved by its own pool; a latency-bound serving loop where
 * cudaMalloc/cudaFree would synchronise the device). The pages describe no
 * such call; it exists for this library's users only.
 * Same arguments and results as moge_route, minus `workspace`: the routing
 * scratch (per-tile histograms, row bases, ranks) lives in a fixed 1 MiB array
 * inside the library's device image, held by every GPU that loads the library
 * until the process exits. Limit: 2*round256(ceil(T/16)*N*4) +
 * round256(T*K*4) <= 1048576 bytes (e.g. T <= 16384 at N = 64, K = 8);
 * larger batches return MOGE_ERR_UNSUPPORTED with a message. Allocates
 * nothing. The first call on a device (with that device current) looks up the
 * array's device address, and again the first call after the device's context
 * changed (a cudaDeviceReset); make those calls before any stream capture.
 * All calls on a device share the array: calls that overlap on the GPU race,
 * so order them on one stream. Nothing in the array needs clearing between
 * calls (each call writes every scratch word it reads). */
MOGE_API int moge_route_noalloc(const moge_config *cfg, const void *x, const void *w_router,
                                const float *logit_bias, int32_t *topk_idx, float *topk_w,
                                int32_t *counts, int32_t *offsets, int32_t *perm_src,
                                int32_t *perm_dst, void *stream);

/* Stage timing (measurement aid): while enabled, every moge_layer_forward
 * records CUDA events around its five launches -- router, scan, permute,
 * grouped FFN (both projections), combine -- and the library adds up their
 * durations. moge_stage_timing(1) resets the totals and starts, (0) stops.
 * moge_stage_times waits for the recorded events and returns the totals in
 * milliseconds per stage (ms_total[5]) and the number of timed calls. For one
 * host thread and one device; not for use during CUDA stream capture. */
MOGE_API int moge_stage_timing(int enable);
MOGE_API int moge_stage_times(double *ms_total, int64_t *calls);

/* Failure-path check (test aid; the pages have no counterpart). Launches one
 * small kernel whose two bounded device waits can never be satisfied -- an
 * mbarrier phase that no thread completes and a completion counter that
 * nothing increments, the same wait helpers the layer's pipelines use -- so
 * both give up after limit_us microseconds (1 .. 2,000,000), record the
 * timeout bit in the device error word and return. out: caller-owned device
 * int32[3]; afterwards out[0] = 1 (mbarrier wait gave up), out[1] = 1
 * (counter wait gave up), out[2] = 0. The next moge_check_device_errors then
 * returns MOGE_ERR_TIMEOUT (and clears the word); the context stays usable.
 * No fault, trap or hang is involved. */
MOGE_API int moge_selftest_waits(int64_t limit_us, int32_t *out, void *stream);

/* ---------------------------------------------------------------- 8-bit expert weights
 * The pages report 8-bit weight quantisation of the model (hwcomputing.csdn.net
 * news piece, deployment section) and an expert-aware quantisation method
 * (techwalker.com article, section 3) without a number format. This library
 * reads it as weights-only FP8: OCP E4M3 codes with one fp32 scale per weight
 * row (output channel); activations, h and y stay bf16. Calibration (the
 * pages' smoothing and routing-alignment steps) is not part of it.
 *
 * Quantise rows of a bf16 matrix w [rows][cols] (device):
 *   scale[r] = amax_r / 448 (fp32 division; 1 for an all-zero row)
 *   q[r][c]  = E4M3 of fp32(w[r][c] / scale[r]), round to nearest even,
 *              saturating at +-448
 * q [rows][cols] bytes, scale [rows] fp32, both caller-owned device memory.
 * cols % 8 == 0; w 16-byte and q 8-byte aligned. Asynchronous on `stream`.
 * Expert tensors [E][R][C] are quantised as E*R rows. */
MOGE_API int moge_quantize_fp8_rows(const void *w, int64_t rows, int64_t cols, void *q,
                                    float *scale, void *stream);

/* One side's (routed or shared) expert weights in FP8: codes in the layouts of
 * the bf16 weights (gate, up [E][I][d]; down [E][d][I], one byte each) and
 * their row scales (gate_scale, up_scale [E][I]; down_scale [E][d]). The
 * dequantised weight is decode(code) * scale of its row. */
typedef struct {
    const void *gate, *up, *down;
    const float *gate_scale, *up_scale, *down_scale;
} moge_fp8_experts;

/* moge_layer_forward with FP8 expert weights (routed and shared; the router
 * stays bf16). cfg->dtype must be MOGE_BF16; d % 16 == 0 and I % 16 == 0
 * (16-byte rows of codes). `shared` may be NULL when S == 0. Same workspace,
 * routing, residual and aliasing rules as moge_layer_forward. The FFN streams
 * the codes (half the bf16 bytes), widens them exactly to bf16 in shared
 * memory and applies the row scales to the fp32 accumulators. */
MOGE_API int moge_layer_forward_fp8(const moge_config *cfg, const void *x, const void *w_router,
                                    const float *logit_bias, const moge_fp8_experts *routed,
                                    const moge_fp8_experts *shared, const void *residual, void *y,
                                    void *workspace, void *stream);

/* W8A8: 8-bit weights and 8-bit activations. The same deployment section
 * reports a W8A8 configuration (weights and activations in 8 bits), again
 * without a format. This library's reading: the weights as above; the input
 * of every expert matrix product quantised per token with the weight rule --
 * a token's bf16 row of x (for the gate and up products) and its row of h,
 * taken in fp32 (for the down product), each get scale = amax / 448 (fp32
 * division; 1 for an all-zero row) and codes E4M3(fp32(v / scale)). Both
 * operands of every expert GEMM are then E4M3 codes, multiplied by the tensor
 * cores' 8-bit MMA with fp32 accumulation; the fp32 result times the weight
 * row's scale times the token's scale is the product. The router stays bf16,
 * y is bf16.
 *
 * moge_w8a8_workspace_size: bytes of the workspace moge_layer_forward_w8a8
 * needs (larger than moge_workspace_size: it also holds the token codes, h in
 * fp32 and the activation scales); 0 for an invalid config.
 *
 * moge_layer_forward_w8a8: the layer with W8A8 experts (routed and shared).
 * cfg->dtype must be MOGE_BF16; d % 16 == 0 and I % 16 == 0. `shared` may be
 * NULL when S == 0. x, y, residual, routing and aliasing rules as
 * moge_layer_forward_fp8; `workspace` (device, caller-owned, 256-byte
 * aligned) of moge_w8a8_workspace_size bytes. Asynchronous on `stream`. */
MOGE_API size_t moge_w8a8_workspace_size(const moge_config *cfg);
MOGE_API int moge_layer_forward_w8a8(const moge_config *cfg, const void *x, const void *w_router,
                                     const float *logit_bias, const moge_fp8_experts *routed,
                                     const moge_fp8_experts *shared, const void *residual,
                                     void *y, void *workspace, void *stream);


/* ---------------------------------------------------------------- training
 * Backward pass of the layer (the pages' models are trained, and they name a
 * batch-level auxiliary balance loss: reportify.cn concept page "Mixture of
 * grouped experts", bullet "technical innovation details" -- strength alpha,
 * f_i = share of the batch's tokens routed to expert i; no formula is printed,
 * this library reads it as L_aux = alpha * sum_i f_i * P_i with P_i the batch
 * mean of the softmax score p[t][i]; f_i is a count and carries no gradient).
 * The routing (picks) is held at its forward value, as in every top-K router.
 *
 * Only cfg->dtype == MOGE_BF16, with I % 64 == 0, N % 8 == 0, M * Kp <= 32.
 *
 * moge_train_workspace_size: bytes of the training workspace (the forward
 * workspace plus the saved pre-activations and the backward's scratch), 0 for
 * an unsupported config. */
MOGE_API size_t moge_train_workspace_size(const moge_config *cfg);

/* moge_layer_forward (no residual) that also keeps, in `workspace`, what the
 * backward pass reads: the routing, the permuted rows, h, the expert outputs
 * and the up-projection's pre-activations g and u. Same arguments and rules
 * as moge_layer_forward; `workspace` is a training workspace and must be
 * passed unchanged to the moge_layer_backward call that follows. */
MOGE_API int moge_layer_forward_train(const moge_config *cfg, const void *x, const void *w_router,
                                      const float *logit_bias, const void *w_gate,
                                      const void *w_up, const void *w_down, const void *s_gate,
                                      const void *s_up, const void *s_down, void *y,
                                      void *workspace, void *stream);

/* Gradients of  sum_t dy[t] . y[t] + L_aux  with respect to the layer's input
 * and weights, for the forward of the preceding moge_layer_forward_train call
 * (same cfg, x, weights, logit_bias and workspace; x and the weights must be
 * unchanged). dy [T][d] bf16 (device). Outputs (caller-owned device memory,
 * bf16, 16-byte aligned, overwritten, layouts of their forward tensors):
 * dx [T][d]; dw_router [N][d]; dw_gate, dw_up [N][I][d]; dw_down [N][d][I];
 * ds_gate, ds_up [S][I][d]; ds_down [S][d][I] (NULL when S == 0). An expert no
 * token chose gets a zero gradient. aux: device float (nullable) receiving
 * L_aux. logit_bias gets no gradient (it is an input, not a weight).
 * The workspace's saved tensors are consumed (overwritten) by the call.
 * Computation: the expert GEMMs (dh with the SwiGLU backward fused in its
 * epilogue, dx, dW_down, dW_gate / dW_up over each expert's rows) and the
 * router's (logits recomputed, dW_router, the router's share of dx) run on the
 * tensor cores with fp32 accumulation; the softmax backward, the combine's
 * backward (dy_perm = w * dy, dw = dy . expert output) and the un-permute are
 * bandwidth-bound kernels. Asynchronous on `stream`. */
MOGE_API int moge_layer_backward(const moge_config *cfg, float alpha, const void *x,
                                 const void *w_router, const float *logit_bias,
                                 const void *w_gate, const void *w_up, const void *w_down,
                                 const void *s_gate, const void *s_up, const void *s_down,
                                 const void *dy, void *dx, void *dw_router, void *dw_gate,
                                 void *dw_up, void *dw_down, void *ds_gate, void *ds_up,
                                 void *ds_down, float *aux, void *workspace, void *stream);


/* ---------------------------------------------------------- expert parallelism
 * The pages place one expert group per device (techwalker.com article,
 * section 1: experts reorganised by device so that every device carries the
 * same load; sections 2 and 5: AllGather / ReduceScatter around the grouped
 * matmuls, shared experts split by tensor parallelism). Rank r of `world`
 * ranks (world divides M and I) holds the routed experts of groups
 * [r M/world, (r+1) M/world) -- experts [r N/world, (r+1) N/world), the
 * layouts of the full tensors restricted to those experts -- and rows
 * [r I/world, (r+1) I/world) of every shared expert's W_gate and W_up with
 * the matching columns of its W_down (s_gate, s_up [S][I/world][d], s_down
 * [S][d][I/world], contiguous). A layer step on `world` ranks, each with its
 * own T/world tokens:
 *   1. all-gather x into x_all [T][d]               (collective, caller's)
 *   2. moge_layer_forward_ep_local -> y_part [T][d] fp32: this rank's routed
 *      experts on the picks that fall in its groups (weighted by the global
 *      softmax scores, routing replicated on every rank) plus its slice of
 *      every shared expert
 *   3. reduce-scatter (sum) of y_part into this rank's [T/world][d] rows
 *                                                  (collective, caller's)
 *   4. moge_ep_finish: y = that sum (+ residual) in the layer dtype.
 * The sum over ranks of y_part is the layer's output for all T tokens.
 * cfg describes the whole layer: T = all ranks' tokens, N, M, I of the full
 * model. The Python binding's moge_layer_forward_ep runs the four steps with
 * torch.distributed (NCCL).
 *
 * moge_ep_workspace_size(cfg, world): bytes of the workspace of step 2
 * (0: unsupported). */
MOGE_API size_t moge_ep_workspace_size(const moge_config *cfg, int world);

/* Step 2 (see above). x_all [T][d] in cfg->dtype; w_gate, w_up
 * [N/world][I][d], w_down [N/world][d][I]: this rank's routed experts; s_*:
 * its shared-expert slices (NULL when S == 0); y_part [T][d] fp32 (device,
 * 16-byte aligned, overwritten). Asynchronous on `stream`. */
MOGE_API int moge_layer_forward_ep_local(const moge_config *cfg, int rank, int world,
                                         const void *x_all, const void *w_router,
                                         const float *logit_bias, const void *w_gate,
                                         const void *w_up, const void *w_down,
                                         const void *s_gate, const void *s_up,
                                         const void *s_down, float *y_part, void *workspace,
                                         void *stream);

/* Step 4: y[t] = y_sum[t] (+ residual[t]) for `rows` rows of cfg->d, y and
 * residual in cfg->dtype, y_sum fp32. */
MOGE_API int moge_ep_finish(const moge_config *cfg, int64_t rows, const float *y_sum,
                            const void *residual, void *y, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOGE_H */
