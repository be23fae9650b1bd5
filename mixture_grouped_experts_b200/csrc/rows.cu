// Row-wise kernels of the MoGE layer: the expert-major permutation of the
// token rows (scatter form fused with the index finalisation, and the plain
// gather form), the score-weighted combine with the shared experts and an
// optional residual, and RMSNorm. All move rows as 16-byte vectors; these are
// HBM-bound copies, so they use plain coalesced vector loads/stores and a
// grid of one CTA per row.
//
// Combine weights are the picked experts' global softmax scores ("Huawei
// releases Pangu Pro MoE", techwalker.com, section 1); shared experts are
// always on with weight 1 (same page, section 2).
#include <cuda_fp8.h>

#include "common.cuh"
#include "moge_internal.h"

namespace moge {

constexpr int kRowThreads = 128;
// The layer's scatter spreads one token's row over several CTAs of
// kVecThreads threads, one 8-element vector (16 bytes in bf16) per thread.
constexpr int kVecThreads = 256;

__host__ __device__ __forceinline__ int vec_elems(int dtype) { return dtype == MOGE_F32 ? 4 : 8; }

// CTA (t, part): computes the token's K destination rows, copies its part of
// x[t] (one vector per thread) into each of them; part 0 also writes the
// permutation indices.
__global__ void __launch_bounds__(kVecThreads) scatter_rows_kernel(
    moge_config c, const uint4 *__restrict__ x, const int32_t *__restrict__ topk_idx,
    const int32_t *__restrict__ rank, const int32_t *__restrict__ base,
    const int32_t *__restrict__ offsets, int32_t *perm_src, int32_t *perm_dst, uint4 *x_perm) {
    __shared__ int dst_s[kMaxExperts];
    grid_dependency_wait();
    const int t = blockIdx.x;
    const int K = c.M * c.Kp;
    const int nvec = c.d / vec_elems(c.dtype);
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const size_t i = (size_t)t * K + k;
        const int e = topk_idx[i];
        int row = -1;
        if (e >= 0 && e < c.N) {
            row = offsets[e] + base[(size_t)(t / kRouterTile) * c.N + e] + rank[i];
            if (blockIdx.y == 0) {
                perm_dst[i] = row;
                perm_src[row] = t;
            }
        } else if (blockIdx.y == 0) {
            raise_error(ERRBIT_INVARIANT);
        }
        dst_s[k] = row;
    }
    __syncthreads();
    const int v = blockIdx.y * kVecThreads + threadIdx.x;
    if (v < nvec) {
        const uint4 val = x[(size_t)t * nvec + v];
        for (int k = 0; k < K; ++k) {
            const int row = dst_s[k];
            if (row >= 0) x_perm[(size_t)row * nvec + v] = val;
        }
    }
}

cudaError_t launch_scatter_rows(const moge_config &c, const void *x, const int32_t *topk_idx,
                                const int32_t *rank, const int32_t *base, const int32_t *offsets,
                                int32_t *perm_src, int32_t *perm_dst, void *x_perm,
                                cudaStream_t st) {
    const int nvec = c.d / vec_elems(c.dtype);
    return launch_pdl(scatter_rows_kernel, dim3(c.T, (nvec + kVecThreads - 1) / kVecThreads),
                      dim3(kVecThreads), 0, st, c, (const uint4 *)x, topk_idx, rank, base, offsets,
                      perm_src, perm_dst, (uint4 *)x_perm);
}

// W8A8 activations: one CTA per token t. The row's amax (exact in fp32),
// scale = amax / 448 (IEEE fp32 division; 1 for an all-zero row), each code =
// E4M3 (round to nearest even, saturating) of fp32(x / scale) -- the rule of
// the weight quantiser -- written to x8[t] and to the token's K routed rows of
// x8p, the scale beside each; the permutation indices as the scatter above;
// the amax words of the token's h rows (routed and shared) zeroed for the
// grouped FFN that follows.
__global__ void __launch_bounds__(kVecThreads) quantize_scatter_kernel(
    moge_config c, const uint4 *__restrict__ x, const int32_t *__restrict__ topk_idx,
    const int32_t *__restrict__ rank, const int32_t *__restrict__ base,
    const int32_t *__restrict__ offsets, int32_t *perm_src, int32_t *perm_dst, uint2 *x8,
    float *sx, uint2 *x8p, float *sxp, uint32_t *hmax) {
    __shared__ int dst_s[kMaxExperts];
    __shared__ float red[kVecThreads / 32];
    grid_dependency_wait();
    const int t = blockIdx.x;
    const int K = c.M * c.Kp;
    const int nvec = c.d / 8;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const size_t i = (size_t)t * K + k;
        const int e = topk_idx[i];
        int row = -1;
        if (e >= 0 && e < c.N) {
            row = offsets[e] + base[(size_t)(t / kRouterTile) * c.N + e] + rank[i];
            perm_dst[i] = row;
            perm_src[row] = t;
            hmax[row] = 0u;
        } else {
            raise_error(ERRBIT_INVARIANT);
        }
        dst_s[k] = row;
    }
    for (int s = threadIdx.x; s < c.S; s += blockDim.x)
        hmax[(size_t)c.T * K + (size_t)s * c.T + t] = 0u;
    const uint4 *xr = x + (size_t)t * nvec;
    float amax = 0.0f;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        const uint4 u = xr[v];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();  // also publishes dst_s
    amax = red[0];
    for (int w = 1; w < kVecThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (threadIdx.x == 0) sx[t] = sc;
    for (int k = threadIdx.x; k < K; k += blockDim.x)
        if (dst_s[k] >= 0) sxp[dst_s[k]] = sc;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        const uint4 u = xr[v];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t out[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t b0 =
                __nv_cvt_float_to_fp8(__fdiv_rn(bf16_lo(w[j]), sc), __NV_SATFINITE, __NV_E4M3);
            const uint32_t b1 =
                __nv_cvt_float_to_fp8(__fdiv_rn(bf16_hi(w[j]), sc), __NV_SATFINITE, __NV_E4M3);
            out[j >> 1] |= (b0 | (b1 << 8)) << (16 * (j & 1));
        }
        const uint2 q = make_uint2(out[0], out[1]);
        x8[(size_t)t * nvec + v] = q;
        for (int k = 0; k < K; ++k) {
            const int row = dst_s[k];
            if (row >= 0) x8p[(size_t)row * nvec + v] = q;
        }
    }
}

cudaError_t launch_quantize_scatter(const moge_config &c, const void *x, const int32_t *topk_idx,
                                    const int32_t *rank, const int32_t *base,
                                    const int32_t *offsets, int32_t *perm_src, int32_t *perm_dst,
                                    void *x8, float *sx, void *x8p, float *sxp, uint32_t *hmax,
                                    cudaStream_t st) {
    if (c.T <= 0) return cudaSuccess;
    return launch_pdl(quantize_scatter_kernel, dim3(c.T), dim3(kVecThreads), 0, st, c,
                      (const uint4 *)x, topk_idx, rank, base, offsets, perm_src, perm_dst,
                      (uint2 *)x8, sx, (uint2 *)x8p, sxp, hmax);
}

// x_perm[r] = x[perm_src[r]], one CTA per destination row
__global__ void __launch_bounds__(kRowThreads) gather_rows_kernel(
    moge_config c, const uint4 *__restrict__ x, const int32_t *__restrict__ perm_src,
    uint4 *x_perm) {
    grid_dependency_wait();
    const int r = blockIdx.x;
    const int nvec = c.d / vec_elems(c.dtype);
    const int t = perm_src[r];
    if (t < 0 || t >= c.T) {
        if (threadIdx.x == 0) raise_error(ERRBIT_INVARIANT);
        return;
    }
    const uint4 *src = x + (size_t)t * nvec;
    uint4 *dst = x_perm + (size_t)r * nvec;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) dst[v] = src[v];
}

cudaError_t launch_gather_rows(const moge_config &c, const void *x, const int32_t *perm_src,
                               void *x_perm, cudaStream_t st) {
    const int rows = c.T * c.M * c.Kp;
    return launch_pdl(gather_rows_kernel, dim3(rows), dim3(kRowThreads), 0, st, c, (const uint4 *)x,
                      perm_src, (uint4 *)x_perm);
}

// ---------------------------------------------------------------------------
// y[t] = residual[t] + sum_k w[t][k] * y_perm[perm_dst[t][k]] + sum_b shared_b[t]
// fp32 sums, k ascending, then the shared blocks in order, then the residual.
template <int DT>
__device__ __forceinline__ void load_vec(const void *p, size_t v, float (&f)[8]) {
    if (DT == MOGE_BF16) {
        const uint4 u = reinterpret_cast<const uint4 *>(p)[v];
        f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
        f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
    } else {
        const float4 a = reinterpret_cast<const float4 *>(p)[2 * v];
        const float4 b = reinterpret_cast<const float4 *>(p)[2 * v + 1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
}
template <int DT>
__device__ __forceinline__ void store_vec(void *p, size_t v, const float (&f)[8]) {
    if (DT == MOGE_BF16) {
        uint4 u;
        u.x = pack_bf16x2(f[0], f[1]); u.y = pack_bf16x2(f[2], f[3]);
        u.z = pack_bf16x2(f[4], f[5]); u.w = pack_bf16x2(f[6], f[7]);
        reinterpret_cast<uint4 *>(p)[v] = u;
    } else {
        reinterpret_cast<float4 *>(p)[2 * v] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4 *>(p)[2 * v + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
}

// Vectors here are 8 elements (16 B in bf16, 32 B in fp32); d % 8 == 0.
// The row loads of one vector are issued in batches of 8 before any of them
// is used, so that the kernel waits for memory once per batch, not per row.
struct Raw8 {
    uint4 a, b;  // bf16: a only; fp32: a and b
};
template <int DT>
__device__ __forceinline__ Raw8 load_raw(const void *row, int v) {
    Raw8 r;
    if (DT == MOGE_BF16) {
        r.a = reinterpret_cast<const uint4 *>(row)[v];
        r.b = make_uint4(0, 0, 0, 0);
    } else {
        r.a = reinterpret_cast<const uint4 *>(row)[2 * v];
        r.b = reinterpret_cast<const uint4 *>(row)[2 * v + 1];
    }
    return r;
}
template <int DT>
__device__ __forceinline__ void unpack8(const Raw8 &r, float (&f)[8]) {
    if (DT == MOGE_BF16) {
        f[0] = bf16_lo(r.a.x); f[1] = bf16_hi(r.a.x); f[2] = bf16_lo(r.a.y); f[3] = bf16_hi(r.a.y);
        f[4] = bf16_lo(r.a.z); f[5] = bf16_hi(r.a.z); f[6] = bf16_lo(r.a.w); f[7] = bf16_hi(r.a.w);
    } else {
        f[0] = __uint_as_float(r.a.x); f[1] = __uint_as_float(r.a.y);
        f[2] = __uint_as_float(r.a.z); f[3] = __uint_as_float(r.a.w);
        f[4] = __uint_as_float(r.b.x); f[5] = __uint_as_float(r.b.y);
        f[6] = __uint_as_float(r.b.z); f[7] = __uint_as_float(r.b.w);
    }
}

template <int DT>
__global__ void __launch_bounds__(kRowThreads) combine_kernel(
    int T, int d, int N, const void *__restrict__ y_perm, const float *__restrict__ topk_w,
    const int32_t *__restrict__ perm_dst, int K, const void *__restrict__ shared_rows,
    int n_shared, const void *residual, void *y, int out_f32) {
    __shared__ const char *src_s[2 * kMaxExperts + 1];
    __shared__ float w_s[kMaxExperts];
    grid_dependency_wait();
    const int t = blockIdx.x;
    const int nvec = d / 8;
    const size_t row_bytes = (size_t)d * (DT == MOGE_BF16 ? 2 : 4);
    (void)N;
    // source rows in summation order: K routed rows, then the shared blocks
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        int row = perm_dst[(size_t)t * K + k];
        if (row < 0 || row >= T * K) {
            raise_error(ERRBIT_INVARIANT);
            row = 0;
        }
        src_s[k] = static_cast<const char *>(y_perm) + (size_t)row * row_bytes;
        w_s[k] = topk_w[(size_t)t * K + k];
    }
    for (int b = threadIdx.x; b < n_shared; b += blockDim.x)
        src_s[K + b] = static_cast<const char *>(shared_rows) + ((size_t)b * T + t) * row_bytes;
    __syncthreads();
    const int nsrc = K + n_shared;
    // CTA (t, part): vectors part*blockDim.x .. of the row (one per thread)
    for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < nvec; v += gridDim.y * blockDim.x) {
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int k0 = 0; k0 < nsrc; k0 += 8) {
            Raw8 raw[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (k0 + j < nsrc) raw[j] = load_raw<DT>(src_s[k0 + j], v);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int k = k0 + j;
                if (k < nsrc) {
                    float f[8];
                    unpack8<DT>(raw[j], f);
                    if (k < K) {
                        const float w = w_s[k];
#pragma unroll
                        for (int q = 0; q < 8; ++q) acc[q] = fmaf(w, f[q], acc[q]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q) acc[q] += f[q];
                    }
                }
            }
        }
        if (residual) {
            float f[8];
            load_vec<DT>((const char *)residual + (size_t)t * row_bytes, v, f);
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = f[q] + acc[q];
        }
        if (out_f32)
            store_vec<MOGE_F32>((char *)y + (size_t)t * d * 4, v, acc);
        else
            store_vec<DT>((char *)y + (size_t)t * row_bytes, v, acc);
    }
}

cudaError_t launch_combine(const moge_config &c, const void *y_perm, const float *topk_w,
                           const int32_t *perm_dst, int K, const void *shared_rows,
                           int n_shared_blocks, const void *residual, void *y, cudaStream_t st,
                           bool out_f32) {
    auto kern = c.dtype == MOGE_BF16 ? combine_kernel<MOGE_BF16> : combine_kernel<MOGE_F32>;
    // few tokens (decode): a token's row spread over several CTAs, down to one
    // 8-element vector per thread, for about 2048 CTAs; many tokens: one CTA each
    const int nvec = c.d / 8;
    const int max_parts = (nvec + kRowThreads - 1) / kRowThreads;
    const int want = (2048 + c.T - 1) / (c.T > 0 ? c.T : 1);
    const int parts = want < max_parts ? (want > 1 ? want : 1) : max_parts;
    return launch_pdl(kern, dim3(c.T, parts), dim3(kRowThreads), 0, st, c.T, c.d, c.N, y_perm, topk_w,
                      perm_dst, K, shared_rows, n_shared_blocks, residual, y, out_f32 ? 1 : 0);
}

// ---------------------------------------------------------------------------
// u = x / sqrt(mean(x^2) + eps), unit gain; fp32 sum in a fixed tree order.
template <int DT>
__global__ void __launch_bounds__(kRowThreads) rmsnorm_kernel(int d, const void *__restrict__ x,
                                                              float eps, void *u) {
    __shared__ float red[kRowThreads / 32];
    grid_dependency_wait();
    const int t = blockIdx.x;
    const int nvec = d / 8;
    const size_t esz = DT == MOGE_BF16 ? 2 : 4;
    const char *xr = (const char *)x + (size_t)t * d * esz;
    float ss = 0.0f;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        float f[8];
        load_vec<DT>(xr, v, f);
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = fmaf(f[j], f[j], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < kRowThreads / 32; ++w) tot += red[w];
    const float r = rsqrtf(tot / (float)d + eps);
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        float f[8];
        load_vec<DT>(xr, v, f);
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] *= r;
        store_vec<DT>((char *)u + (size_t)t * d * esz, v, f);
    }
}

cudaError_t launch_rmsnorm(const moge_config &c, const void *x, float eps, void *u,
                           cudaStream_t st) {
    auto kern = c.dtype == MOGE_BF16 ? rmsnorm_kernel<MOGE_BF16> : rmsnorm_kernel<MOGE_F32>;
    return launch_pdl(kern, dim3(c.T), dim3(kRowThreads), 0, st, c.d, x, eps, u);
}

}  // namespace moge
