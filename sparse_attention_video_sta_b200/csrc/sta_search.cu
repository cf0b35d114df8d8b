// sta_search.cu -- per-head statistics for choosing STA windows.
//
// The pages choose a window per head by profiling ("Fast Video Generation
// with Sliding Tile Attention": podcast transcript at hotaipapers.com, segment
// on head specialisation; dianyo.github.io ICML-2025 post, STA section,
// "Observation & Proposed Method"): the attention recall of a window (the
// share of full-attention softmax mass it keeps) and a mask-search loss
// averaged over inputs.  Given the forward's outputs for a candidate window
// (o_w, lse_w) and for the full window (o_full, lse_full), row i's recall is
// exp(lse_w[i] - lse_full[i]) (both LSEs are logs of sums of the same
// exponentials, over the window's keys and over all keys); the loss is the
// mean squared difference of the outputs.  This kernel reduces both per
// (b, h) slice.
//
// One thread-block cluster of 8 CTAs per slice, 1024 threads each: every CTA
// reduces one contiguous eighth of the slice (16-byte loads of the two
// outputs, fp32 partial sums per thread widened to fp64, a fixed-order tree in
// shared memory), then CTA 0 of the cluster adds the eight partials, read
// from the other CTAs' shared memory in rank order.  The result is
// deterministic and needs no scratch memory; with 8 CTAs per slice the grid
// covers every SM at the workloads' 24+ slices.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sta_internal.h"

namespace sta {
namespace {

constexpr int kStatThreads = 1024;
constexpr int kStatCluster = 8;

// [lo, hi) share of `n` items for part `r` of `parts`.
__device__ __forceinline__ void split_range(int64_t n, int r, int parts, int64_t& lo, int64_t& hi) {
    lo = n * r / parts;
    hi = n * (r + 1) / parts;
}

__global__ void __cluster_dims__(kStatCluster, 1, 1) __launch_bounds__(kStatThreads)
window_stats_kernel(const float* __restrict__ lse_w, const float* __restrict__ lse_full,
                    const uint4* __restrict__ o_w, const uint4* __restrict__ o_full, int64_t tokens,
                    int64_t vecs_per_slice, double* __restrict__ recall, double* __restrict__ mse) {
    namespace cg = cooperative_groups;
    __shared__ double red[2][kStatThreads];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = int(cluster.block_rank());
    const int64_t s = blockIdx.x / kStatCluster;
    int64_t lo, hi;
    split_range(tokens, rank, kStatCluster, lo, hi);
    const float* lw = lse_w + s * tokens;
    const float* lf = lse_full + s * tokens;
    double r_acc = 0.0;
    for (int64_t i = lo + threadIdx.x; i < hi; i += kStatThreads) r_acc += double(expf(lw[i] - lf[i]));
    split_range(vecs_per_slice, rank, kStatCluster, lo, hi);
    const uint4* a = o_w + s * vecs_per_slice;
    const uint4* b = o_full + s * vecs_per_slice;
    double m_acc = 0.0;
    for (int64_t i = lo + threadIdx.x; i < hi; i += kStatThreads) {
        const uint4 x = __ldg(a + i), y = __ldg(b + i);
        const uint32_t xw[4] = {x.x, x.y, x.z, x.w}, yw[4] = {y.x, y.y, y.z, y.w};
        float part = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float d0 = __uint_as_float(xw[j] << 16) - __uint_as_float(yw[j] << 16);
            const float d1 = __uint_as_float(xw[j] & 0xffff0000u) - __uint_as_float(yw[j] & 0xffff0000u);
            part = fmaf(d0, d0, part);
            part = fmaf(d1, d1, part);
        }
        m_acc += double(part);
    }
    red[0][threadIdx.x] = r_acc;
    red[1][threadIdx.x] = m_acc;
    __syncthreads();
    for (int w = kStatThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w) {
            red[0][threadIdx.x] += red[0][threadIdx.x + w];
            red[1][threadIdx.x] += red[1][threadIdx.x + w];
        }
        __syncthreads();
    }
    cluster.sync();  // every CTA's partial is in its red[*][0]
    if (rank == 0 && threadIdx.x == 0) {
        double rs = 0.0, ms = 0.0;
        for (int r = 0; r < kStatCluster; ++r) {
            const double* peer = cluster.map_shared_rank(&red[0][0], r);
            rs += peer[0];
            ms += peer[kStatThreads];
        }
        recall[s] = rs / double(tokens);
        mse[s] = ms / double(vecs_per_slice * 8);
    }
    cluster.sync();  // keep the partials alive until CTA 0 has read them
}

}  // namespace

cudaError_t launch_window_stats(const float* lse_w, const float* lse_full, const void* o_w, const void* o_full,
                                int64_t slices, int64_t tokens, int head_dim, double* recall, double* mse,
                                cudaStream_t stream) {
    const int64_t vecs = tokens * head_dim / 8;
    window_stats_kernel<<<dim3(uint32_t(slices * kStatCluster)), kStatThreads, 0, stream>>>(
        lse_w, lse_full, static_cast<const uint4*>(o_w), static_cast<const uint4*>(o_full), tokens, vecs, recall,
        mse);
    return cudaGetLastError();
}

}  // namespace sta
