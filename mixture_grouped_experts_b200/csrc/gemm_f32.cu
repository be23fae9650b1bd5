// fp32 grouped SwiGLU FFN on CUDA cores (no TF32: its 10-bit mantissa cannot
// hold a 1e-4 relative tolerance). Used for fp32 layers, which are small; the
// bf16 layers run on the tcgen05 kernel in gemm_tc.cu.
//
// Same work plan as the tensor-core path: entry ex of the plan is one expert
// with `rows` token rows; one CTA computes a 64 x 64 output tile of it.
#include "common.cuh"
#include "moge_internal.h"

namespace moge {

constexpr int kF32Tile = 64;
constexpr int kF32K = 16;

// up: h[dst + r][i] = silu(sum_k x[r][k] Wg[i][k]) * sum_k x[r][k] Wu[i][k]
__global__ void __launch_bounds__(256) ffn_up_f32_kernel(moge_config c, const ExpertWork *work,
                                                         FfnOperands op) {
    __shared__ float xs[kF32K][kF32Tile + 1];
    __shared__ float gs[kF32K][kF32Tile + 1];
    __shared__ float us[kF32K][kF32Tile + 1];
    grid_dependency_wait();
    const ExpertWork w = work[blockIdx.z];
    const int r0 = blockIdx.y * kF32Tile, i0 = blockIdx.x * kF32Tile;
    if (r0 >= w.rows) return;
    const int d = c.d, I = c.I;
    const float *X = (const float *)(w.b_sel ? op.b1 : op.b0) + (size_t)w.src_row0 * d;
    const size_t wo = (size_t)w.a_idx * I * d;
    const float *Wg = (const float *)(w.a_sel ? op.sg : op.wg) + wo;
    const float *Wu = (const float *)(w.a_sel ? op.su : op.wu) + wo;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float ag[4][4] = {}, au[4][4] = {};
    for (int k0 = 0; k0 < d; k0 += kF32K) {
        for (int l = threadIdx.x; l < kF32K * kF32Tile; l += 256) {
            const int rr = l / kF32K, kk = l % kF32K;
            const int k = k0 + kk;
            xs[kk][rr] = (r0 + rr < w.rows && k < d) ? X[(size_t)(r0 + rr) * d + k] : 0.0f;
            gs[kk][rr] = (i0 + rr < I && k < d) ? Wg[(size_t)(i0 + rr) * d + k] : 0.0f;
            us[kk][rr] = (i0 + rr < I && k < d) ? Wu[(size_t)(i0 + rr) * d + k] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kF32K; ++kk) {
            float a[4], g[4], u[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                a[j] = xs[kk][ty * 4 + j];
                g[j] = gs[kk][tx * 4 + j];
                u[j] = us[kk][tx * 4 + j];
            }
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    ag[p][q] = fmaf(a[p], g[q], ag[p][q]);
                    au[p][q] = fmaf(a[p], u[q], au[p][q]);
                }
        }
        __syncthreads();
    }
    float *H = (float *)op.h + (size_t)w.dst_row0 * I;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int r = r0 + ty * 4 + p;
        if (r >= w.rows) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = i0 + tx * 4 + q;
            if (i >= I) continue;
            const float g = ag[p][q];
            H[(size_t)r * I + i] = g / (1.0f + expf(-g)) * au[p][q];
        }
    }
}

// down: y[dst + r][o] = sum_i h[src + r][i] Wd[o][i]
__global__ void __launch_bounds__(256) ffn_down_f32_kernel(moge_config c, const ExpertWork *work,
                                                           FfnOperands op) {
    __shared__ float hs[kF32K][kF32Tile + 1];
    __shared__ float ws[kF32K][kF32Tile + 1];
    grid_dependency_wait();
    const ExpertWork w = work[blockIdx.z];
    const int r0 = blockIdx.y * kF32Tile, o0 = blockIdx.x * kF32Tile;
    if (r0 >= w.rows) return;
    const int d = c.d, I = c.I;
    const float *Hm = (const float *)op.h + (size_t)w.src_row0 * I;
    const float *Wd = (const float *)(w.a_sel ? op.sd : op.wd) + (size_t)w.a_idx * d * I;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < I; k0 += kF32K) {
        for (int l = threadIdx.x; l < kF32K * kF32Tile; l += 256) {
            const int rr = l / kF32K, kk = l % kF32K;
            const int k = k0 + kk;
            hs[kk][rr] = (r0 + rr < w.rows && k < I) ? Hm[(size_t)(r0 + rr) * I + k] : 0.0f;
            ws[kk][rr] = (o0 + rr < d && k < I) ? Wd[(size_t)(o0 + rr) * I + k] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kF32K; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                a[j] = hs[kk][ty * 4 + j];
                b[j] = ws[kk][tx * 4 + j];
            }
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
        }
        __syncthreads();
    }
    float *Y = (float *)op.y + (size_t)w.dst_row0 * d;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int r = r0 + ty * 4 + p;
        if (r >= w.rows) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int o = o0 + tx * 4 + q;
            if (o < d) Y[(size_t)r * d + o] = acc[p][q];
        }
    }
}

cudaError_t launch_ffn_f32(const moge_config &c, const Plan &plan, int n_entries,
                           const FfnOperands &op, cudaStream_t st, cudaEvent_t mid) {
    if (n_entries <= 0 || c.T <= 0) return cudaSuccess;
    const int rt = (c.T + kF32Tile - 1) / kF32Tile;
    dim3 gu((c.I + kF32Tile - 1) / kF32Tile, rt, n_entries);
    cudaError_t e = launch_pdl(ffn_up_f32_kernel, gu, dim3(256), 0, st, c, plan.up, op);
    if (e != cudaSuccess) return e;
    if (mid && (e = cudaEventRecord(mid, st)) != cudaSuccess) return e;
    dim3 gd((c.d + kF32Tile - 1) / kF32Tile, rt, n_entries);
    return launch_pdl(ffn_down_f32_kernel, gd, dim3(256), 0, st, c, plan.down, op);
}

}  // namespace moge
