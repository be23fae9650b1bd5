// Expert parallelism: the pages place one expert group per device ("experts
// reorganised by device", techwalker.com article, section 1; the decode
// deployment pairs it with AllGather / ReduceScatter communication, sections 2
// and 5). Rank r of R holds groups [r M/R, (r+1) M/R) -- experts
// [r N/R, (r+1) N/R) -- and an I/R slice of every shared expert. A layer on R
// ranks: all-gather x; every rank routes all T tokens (the router is
// replicated) and runs its own experts on the picks that fall in its groups
// plus its shared-expert slice, summing into an fp32 partial y; a
// reduce-scatter of the partials leaves each rank its tokens' y. The
// collectives are NCCL's (torch.distributed); these kernels are the local
// steps around them.
#include "common.cuh"
#include "moge_internal.h"

namespace moge {

// This rank's share of the global routing: picks of its groups (expert ids
// made local), their weights and in-tile ranks, and its experts' per-tile
// histogram columns.
__global__ void localize_kernel(int T, int N, int K, int k0, int K_loc, int e0, int N_loc,
                                int tiles, const int32_t *__restrict__ topk_idx,
                                const float *__restrict__ topk_w, const int32_t *__restrict__ rank,
                                const int32_t *__restrict__ hist, int32_t *idx_loc, float *w_loc,
                                int32_t *rank_loc, int32_t *hist_loc) {
    grid_dependency_wait();
    const long long n_pick = (long long)T * K_loc, n_hist = (long long)tiles * N_loc;
    const long long n = n_pick > n_hist ? n_pick : n_hist;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        if (i < n_pick) {
            const long long t = i / K_loc, j = i % K_loc;
            const size_t src = (size_t)t * K + k0 + j;
            const int e = topk_idx[src] - e0;
            if (e < 0 || e >= N_loc) raise_error(ERRBIT_INVARIANT);
            idx_loc[i] = e;
            w_loc[i] = topk_w[src];
            rank_loc[i] = rank[src];
        }
        if (i < n_hist) {
            const long long tile = i / N_loc, e = i % N_loc;
            hist_loc[i] = hist[(size_t)tile * N + e0 + e];
        }
    }
}

cudaError_t launch_localize(int T, int N, int K, int k0, int K_loc, int e0, int N_loc, int tiles,
                            const int32_t *topk_idx, const float *topk_w, const int32_t *rank,
                            const int32_t *hist, int32_t *idx_loc, float *w_loc, int32_t *rank_loc,
                            int32_t *hist_loc, cudaStream_t st) {
    const long long n = std::max((long long)T * K_loc, (long long)tiles * N_loc);
    const int blocks = (int)std::min<long long>((n + 255) / 256, 4096);
    return launch_pdl(localize_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st, T, N, K, k0,
                      K_loc, e0, N_loc, tiles, topk_idx, topk_w, rank, hist, idx_loc, w_loc,
                      rank_loc, hist_loc);
}

// y[t] = y_sum[t] (+ residual[t]) in the layer's dtype; 8 elements per thread.
template <int DT>
__global__ void ep_finish_kernel(long long rows, int d, const float4 *__restrict__ y_sum,
                                 const void *residual, void *y) {
    grid_dependency_wait();
    const long long nvec = (long long)rows * (d / 8);
    for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < nvec;
         v += (long long)gridDim.x * blockDim.x) {
        const float4 a = y_sum[2 * v], b = y_sum[2 * v + 1];
        float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        if (DT == MOGE_BF16) {
            if (residual) {
                const uint4 r = static_cast<const uint4 *>(residual)[v];
                f[0] += bf16_lo(r.x); f[1] += bf16_hi(r.x); f[2] += bf16_lo(r.y); f[3] += bf16_hi(r.y);
                f[4] += bf16_lo(r.z); f[5] += bf16_hi(r.z); f[6] += bf16_lo(r.w); f[7] += bf16_hi(r.w);
            }
            static_cast<uint4 *>(y)[v] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                    pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
        } else {
            if (residual) {
                const float4 r0 = static_cast<const float4 *>(residual)[2 * v];
                const float4 r1 = static_cast<const float4 *>(residual)[2 * v + 1];
                f[0] += r0.x; f[1] += r0.y; f[2] += r0.z; f[3] += r0.w;
                f[4] += r1.x; f[5] += r1.y; f[6] += r1.z; f[7] += r1.w;
            }
            static_cast<float4 *>(y)[2 * v] = make_float4(f[0], f[1], f[2], f[3]);
            static_cast<float4 *>(y)[2 * v + 1] = make_float4(f[4], f[5], f[6], f[7]);
        }
    }
}

cudaError_t launch_ep_finish(int dtype, long long rows, int d, const float *y_sum,
                             const void *residual, void *y, cudaStream_t st) {
    const long long nvec = rows * (d / 8);
    const int blocks = (int)std::min<long long>((nvec + 255) / 256, 8192);
    auto kern = dtype == MOGE_BF16 ? ep_finish_kernel<MOGE_BF16> : ep_finish_kernel<MOGE_F32>;
    return launch_pdl(kern, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st, rows, d,
                      (const float4 *)y_sum, residual, y);
}

}  // namespace moge
