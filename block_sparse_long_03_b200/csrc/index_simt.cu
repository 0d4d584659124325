// index_simt.cu -- index branch on CUDA cores (fp32 workloads).
//
// Block scores ("MiniMax Sparse Attention", Summary, second paragraph:
// max-pooled token-level index dot products):
//   bs[b, t, g, n] = max_{j in block n, j <= p(t)} q_idx[b, t, g, :] . k_idx[b, j, :]
//   bs[b, t, g, n] = -inf when block n starts after p(t).
//
// One CTA per (KV block n, tile of tq query tokens, batch entry), tq * G <= 256
// rows (tq = 16 while G <= 16).  The CTA
// stages the tile's index queries (tq * G rows) and the block's index keys
// in shared memory as fp32; each (token, group) row is owned by `tpr`
// adjacent threads that split the block's keys and combine their maxima
// with shuffles.  Only the block score leaves the CTA.
#include <math.h>

#include <algorithm>

#include "msa_internal.cuh"

namespace msa {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxTQ = 16;

template <typename T>
__global__ void __launch_bounds__(kThreads)
index_scores_simt_kernel(const T *__restrict__ q_idx, const T *__restrict__ k_idx,
                         float *__restrict__ bs, int T_, int S, int G, int d_idx, int block,
                         int NB, int tpr, int tq) {
    extern __shared__ float smem[];
    const int n = blockIdx.x;
    const int t0 = blockIdx.y * tq;
    const int b = blockIdx.z;
    const int ld = d_idx + 1;                 // padded row stride (bank spread)
    float *qs = smem;                         // [tq * G][ld]
    float *ks = smem + tq * G * ld;           // [block][ld]
    const int rows = tq * G;
    const int tq_end = min(tq, T_ - t0);
    const int64_t p_last = (int64_t)S - T_ + t0 + tq_end - 1;

    // rows of this tile: r = tq * G + g
    const int row = threadIdx.x / tpr;
    const int sub = threadIdx.x % tpr;
    const bool active = row < rows && (row / G) < tq_end;
    const int64_t p = (int64_t)S - T_ + t0 + row / G;
    float *out = bs + (((int64_t)b * T_ + t0 + row / G) * G + (row % G)) * NB + n;

    if ((int64_t)n * block > p_last) {        // no causal token for any row
        if (active && sub == 0) *out = -INFINITY;
        return;
    }
    for (int i = threadIdx.x; i < tq_end * G * d_idx; i += kThreads) {
        const int r = i / d_idx, c = i % d_idx;
        qs[r * ld + c] = to_f32(q_idx[((int64_t)b * T_ + t0) * G * d_idx + i]);
    }
    for (int i = threadIdx.x; i < block * d_idx; i += kThreads) {
        const int jj = i / d_idx, c = i % d_idx;
        ks[jj * ld + c] = to_f32(k_idx[((int64_t)b * S + (int64_t)n * block) * d_idx + i]);
    }
    __syncthreads();

    float best = -INFINITY;
    if (active) {
        const float *q = qs + row * ld;
        for (int jj = sub; jj < block; jj += tpr) {
            if ((int64_t)n * block + jj > p) break;
            const float *k = ks + jj * ld;
            float dot = 0.f;
            for (int c = 0; c < d_idx; ++c) dot = fmaf(q[c], k[c], dot);
            best = fmaxf(best, dot);
        }
    }
    for (int off = tpr / 2; off > 0; off /= 2)
        best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
    if (active && sub == 0) *out = canon_zero(best);
}

}  // namespace

cudaError_t launch_index_scores_simt(const Shape &s, const void *q_idx, const void *k_idx,
                                     float *bs, cudaStream_t st) {
    if (s.G > kThreads) return cudaErrorInvalidConfiguration;
    const int tq = std::min(kMaxTQ, kThreads / s.G);
    const int rows = tq * s.G;
    int tpr = 1;
    while (tpr * 2 * rows <= kThreads && tpr < 32) tpr *= 2;
    const size_t smem = sizeof(float) * (size_t)(rows + s.block) * (s.d_idx + 1);
    dim3 grid(s.NB, (s.T + tq - 1) / tq, s.B);
    if (s.dtype == MSA_F32) {
        auto k = index_scores_simt_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, kThreads, smem, st>>>((const float *)q_idx, (const float *)k_idx, bs, s.T, s.S,
                                         s.G, s.d_idx, s.block, s.NB, tpr, tq);
    } else {
        auto k = index_scores_simt_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, kThreads, smem, st>>>((const __nv_bfloat16 *)q_idx,
                                         (const __nv_bfloat16 *)k_idx, bs, s.T, s.S, s.G,
                                         s.d_idx, s.block, s.NB, tpr, tq);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
