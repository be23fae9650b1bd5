// Backward pass of the MoGE layer: the bandwidth-bound steps around its
// grouped GEMMs (gemm_bwd.cu). The routing is held at its forward value.
//   combine backward   dy_perm[r] = w[t][k] dy[t] (bf16),  dw[t][k] = dy[t] . y_perm[r]
//   router backward    p = softmax(l[t]) (recomputed logits), dp = dw at the picks
//                      + alpha f_e / T (batch balance loss), dl = p (dp - p . dp)
//   balance loss       L_aux = alpha sum_e f_e P_e, P_e the batch mean of p (two
//                      fixed-order reduction steps)
//   un-permute         dx[t] = sum_k dx_perm[perm_dst[t][k]] + sum_s dx_perm[T K + s T + t]
//                              + dx_r[t]   (fp32 sums in that order, bf16 out)
#include "common.cuh"
#include "moge_internal.h"

namespace moge {

constexpr int kBwdThreads = 128;
constexpr int kMaxK = 32;
constexpr int kRouterBwdWarps = 8;
constexpr int kRouterBwdPerWarp = 8;  // tokens per warp, one after another
constexpr int kRouterBwdTokens = kRouterBwdWarps * kRouterBwdPerWarp;  // tokens per CTA

__device__ __forceinline__ void unpack8(const uint4 u, float (&f)[8]) {
    f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
    f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

// One CTA per token.
__global__ void __launch_bounds__(kBwdThreads) combine_bwd_kernel(
    moge_config c, const uint4 *__restrict__ dy, const uint4 *__restrict__ y_perm,
    const float *__restrict__ topk_w, const int32_t *__restrict__ perm_dst, uint4 *dy_perm,
    float *dw) {
    __shared__ float red[kBwdThreads / 32][kMaxK];
    grid_dependency_wait();
    const int t = blockIdx.x;
    const int K = c.M * c.Kp;
    const int nvec = c.d / 8;
    float acc[kMaxK];
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) acc[k] = 0.0f;
    for (int v = threadIdx.x; v < nvec; v += kBwdThreads) {
        float g[8];
        unpack8(dy[(size_t)t * nvec + v], g);
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
            if (k >= K) break;
            const size_t r = (size_t)perm_dst[(size_t)t * K + k];
            const float w = topk_w[(size_t)t * K + k];
            float y[8];
            unpack8(y_perm[r * nvec + v], y);
            float s = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) s += g[i] * y[i];
            acc[k] += s;
            uint4 o;
            o.x = pack_bf16x2(w * g[0], w * g[1]);
            o.y = pack_bf16x2(w * g[2], w * g[3]);
            o.z = pack_bf16x2(w * g[4], w * g[5]);
            o.w = pack_bf16x2(w * g[6], w * g[7]);
            dy_perm[r * nvec + v] = o;
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
        if (k >= K) break;
        float s = acc[k];
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) red[warp][k] = s;
    }
    __syncthreads();
    if (threadIdx.x < K) {
        float s = 0.0f;
        for (int w = 0; w < kBwdThreads / 32; ++w) s += red[w][threadIdx.x];
        dw[(size_t)t * K + threadIdx.x] = s;
    }
}

// One warp per token (each warp takes kRouterBwdPerWarp tokens in turn), lane
// l holding experts l, l + 32, ...; also each CTA's sums of p over its tokens
// (part[blockIdx.x][e], fixed order) for the balance loss.
__global__ void __launch_bounds__(32 * kRouterBwdWarps) router_bwd_kernel(
    moge_config c, float alpha, const float *__restrict__ logits, int ksplit,
    const int32_t *__restrict__ topk_idx, const float *__restrict__ dw,
    const int32_t *__restrict__ counts, uint16_t *dl, float *part) {
    __shared__ float psum[kRouterBwdWarps][kMaxExperts];
    const size_t part_stride = (size_t)c.T * c.N;  // the logit GEMM's K parts
    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = c.N, K = c.M * c.Kp;
    const int per = (N + 31) / 32;
    constexpr int kPer = kMaxExperts / 32;
    const float inv_t = 1.0f / (float)c.T;
    float acc[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) acc[j] = 0.0f;
    for (int r = 0; r < kRouterBwdPerWarp; ++r) {
        const int t = blockIdx.x * kRouterBwdTokens + r * kRouterBwdWarps + warp;
        if (t >= c.T) break;
        float pr[kPer], dp[kPer];
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = lane + 32 * j;
            float l = -INFINITY;
            if (j < per && e < N) {
                l = logits[(size_t)t * N + e];
                for (int k = 1; k < ksplit; ++k) l += logits[k * part_stride + (size_t)t * N + e];
            }
            pr[j] = l;
            mx = fmaxf(mx, pr[j]);
        }
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float z = 0.0f;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            pr[j] = (j < per && lane + 32 * j < N) ? expf(pr[j] - mx) : 0.0f;
            z += pr[j];
        }
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = lane + 32 * j;
            pr[j] /= z;
            acc[j] += pr[j];
            dp[j] = (j < per && e < N) ? alpha * ((float)counts[e] * inv_t) * inv_t : 0.0f;
        }
        for (int k = 0; k < K; ++k) {
            const int e = topk_idx[(size_t)t * K + k];
            const float g = dw[(size_t)t * K + k];
#pragma unroll
            for (int j = 0; j < kPer; ++j)
                if (e == lane + 32 * j) dp[j] += g;
        }
        float pdp = 0.0f;
#pragma unroll
        for (int j = 0; j < kPer; ++j) pdp += pr[j] * dp[j];
        for (int o = 16; o > 0; o >>= 1) pdp += __shfl_xor_sync(0xffffffffu, pdp, o);
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = lane + 32 * j;
            if (j < per && e < N) dl[(size_t)t * N + e] = to_bf16_bits(pr[j] * (dp[j] - pdp));
        }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j)
        if (lane + 32 * j < N) psum[warp][lane + 32 * j] = acc[j];
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        float sum = 0.0f;
        for (int w = 0; w < kRouterBwdWarps; ++w) sum += psum[w][e];
        part[(size_t)blockIdx.x * N + e] = sum;
    }
}

// L_aux = alpha sum_e f_e P_e, summed in a fixed order (one CTA).
__global__ void __launch_bounds__(256) aux_loss_kernel(moge_config c, float alpha,
                                                       const float *__restrict__ part, int nparts,
                                                       const int32_t *__restrict__ counts,
                                                       float *aux) {
    __shared__ float red[256];
    grid_dependency_wait();
    float s = 0.0f;
    for (int e = threadIdx.x; e < c.N; e += blockDim.x) {
        float P = 0.0f;
        for (int b = 0; b < nparts; ++b) P += part[(size_t)b * c.N + e];
        s += ((float)counts[e] / (float)c.T) * (P / (float)c.T);
    }
    red[threadIdx.x] = s;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *aux = alpha * red[0];
}

// One CTA per token.
__global__ void __launch_bounds__(kBwdThreads) unpermute_bwd_kernel(
    moge_config c, const uint4 *__restrict__ dx_perm, const int32_t *__restrict__ perm_dst,
    const float4 *__restrict__ dx_r, uint4 *dx) {
    grid_dependency_wait();
    const int t = blockIdx.x;
    const int K = c.M * c.Kp;
    const int nvec = c.d / 8;
    const size_t rrows = (size_t)c.T * K;
    for (int v = threadIdx.x; v < nvec; v += kBwdThreads) {
        float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float f[8];
        for (int k = 0; k < K; ++k) {
            unpack8(dx_perm[(size_t)perm_dst[(size_t)t * K + k] * nvec + v], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) s[i] += f[i];
        }
        for (int b = 0; b < c.S; ++b) {
            unpack8(dx_perm[(rrows + (size_t)b * c.T + t) * nvec + v], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) s[i] += f[i];
        }
        const float4 a = dx_r[((size_t)t * nvec + v) * 2], b = dx_r[((size_t)t * nvec + v) * 2 + 1];
        s[0] += a.x; s[1] += a.y; s[2] += a.z; s[3] += a.w;
        s[4] += b.x; s[5] += b.y; s[6] += b.z; s[7] += b.w;
        uint4 o;
        o.x = pack_bf16x2(s[0], s[1]);
        o.y = pack_bf16x2(s[2], s[3]);
        o.z = pack_bf16x2(s[4], s[5]);
        o.w = pack_bf16x2(s[6], s[7]);
        dx[(size_t)t * nvec + v] = o;
    }
}

cudaError_t launch_combine_bwd(const moge_config &c, const void *dy, const void *y_perm,
                               const float *topk_w, const int32_t *perm_dst, void *dy_perm,
                               float *dw, cudaStream_t st) {
    return launch_pdl(combine_bwd_kernel, dim3(c.T), dim3(kBwdThreads), 0, st, c, (const uint4 *)dy,
                      (const uint4 *)y_perm, topk_w, perm_dst, (uint4 *)dy_perm, dw);
}

int router_bwd_parts(const moge_config &c) { return (c.T + kRouterBwdTokens - 1) / kRouterBwdTokens; }

cudaError_t launch_router_bwd(const moge_config &c, float alpha, const float *logits, int ksplit,
                              const int32_t *topk_idx, const float *dw, const int32_t *counts,
                              void *dl, float *part, float *aux, cudaStream_t st) {
    const int parts = router_bwd_parts(c);
    cudaError_t e = launch_pdl(router_bwd_kernel, dim3(parts), dim3(32 * kRouterBwdWarps), 0, st, c,
                               alpha, logits, ksplit, topk_idx, dw, counts, (uint16_t *)dl, part);
    if (e != cudaSuccess || !aux) return e;
    return launch_pdl(aux_loss_kernel, dim3(1), dim3(256), 0, st, c, alpha, (const float *)part,
                      parts, counts, aux);
}

cudaError_t launch_unpermute_bwd(const moge_config &c, const void *dx_perm, const int32_t *perm_dst,
                                 const float *dx_r, void *dx, cudaStream_t st) {
    return launch_pdl(unpermute_bwd_kernel, dim3(c.T), dim3(kBwdThreads), 0, st, c,
                      (const uint4 *)dx_perm, perm_dst, (const float4 *)dx_r, (uint4 *)dx);
}

}  // namespace moge
