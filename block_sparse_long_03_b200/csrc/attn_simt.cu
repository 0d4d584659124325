// attn_simt.cu -- sparse attention over the kept blocks on CUDA cores.
//
// Main branch ("MiniMax Sparse Attention", Summary, second paragraph: exact
// softmax attention restricted to the kept blocks; Key points, kernel
// design: the LSE is produced by the forward pass).  For query (b, t), head
// h in group g, over the causal tokens j <= p(t) of the kept blocks:
//   O = sum_j softmax(scale * Q.K_j) V_j,   lse = log sum_j exp(scale * Q.K_j).
//
// This is the fp32 path (and the reference shape of the computation for
// every dtype): one CTA per (b, t, g) serves the group's R query heads,
// which share the kept set.  Each kept block is staged in shared memory
// (fp32), thread j scores key j against all R heads, a warp per head
// updates that head's running max / normaliser (online softmax), and
// thread c accumulates output channel c for all R heads.  On request it also
// writes each kept slot's head-averaged share of the softmax (the indexer's
// KL target), from per-block sums kept with the maxima they were taken at.
#include <math.h>

#include "msa_internal.cuh"

namespace msa {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxR = 16;
constexpr int kMaxTopk = 256;

template <typename T, bool kMass>
__global__ void __launch_bounds__(kThreads)
attn_simt_kernel(const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
                 const int32_t *__restrict__ ids, T *__restrict__ O, float *__restrict__ lse,
                 float *__restrict__ mass, uint32_t *err, int T_, int S, int Hq, int Hkv, int d,
                 int block, int topk, int NB, float scale) {
    extern __shared__ float sm[];
    const int g = blockIdx.x % Hkv;
    const int64_t bt = blockIdx.x / Hkv;          // b * T + t
    const int b = (int)(bt / T_), t = (int)(bt % T_);
    const int R = Hq / Hkv;
    const int64_t p = (int64_t)S - T_ + t;
    const int ld = d + 1;
    float *ks = sm;                                // [block][ld]
    float *vs = ks + block * ld;                   // [block][d]
    float *qs = vs + block * d;                    // [R][d]
    float *ss = qs + R * d;                        // [R][block] scores, then weights
    float *m_s = ss + R * block;                   // [R] running max
    float *l_s = m_s + kMaxR;                      // [R] running normaliser
    float *a_s = l_s + kMaxR;                      // [R] rescale factor of this block
    float *bsum = a_s + kMaxR;                     // [topk][R] block sums (for mass)
    float *bmax = bsum + topk * R;                 // [topk][R] the maxima they are taken at
    __shared__ int kept[kMaxTopk];
    __shared__ int kslot[kMaxTopk];                // slot of each kept block
    __shared__ int nkept;

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int32_t *row_ids = ids + bt * Hkv * topk + (int64_t)g * topk;
    if (tid == 0) {   // validate the caller's ids: in range, causal, no repeats
        int n_ok = 0;
        for (int i = 0; i < topk; ++i) {
            const int n = row_ids[i];
            if (n < 0) continue;
            bool bad = n >= NB || (int64_t)n * block > p;
            for (int k = 0; k < n_ok && !bad; ++k) bad = kept[k] == n;
            if (bad) { record_error(err, MSA_ERR_BAD_BLOCK_IDS, 1); continue; }
            kslot[n_ok] = i;
            kept[n_ok++] = n;
        }
        nkept = n_ok;
    }
    for (int i = tid; i < R * d; i += kThreads)
        qs[i] = to_f32(Q[(bt * Hq + (int64_t)g * R) * d + i]) * scale;
    if (tid < R) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }
    if (kMass)
        for (int i = tid; i < topk; i += kThreads) mass[(bt * Hkv + g) * topk + i] = 0.f;
    __syncthreads();

    float acc[kMaxR];
#pragma unroll
    for (int h = 0; h < kMaxR; ++h) acc[h] = 0.f;

    for (int kb = 0; kb < nkept; ++kb) {
        const int64_t j0 = (int64_t)kept[kb] * block;
        if (j0 > p) continue;                      // no causal token (uniform branch)
        const int nk = (p - j0 + 1 < block) ? (int)(p - j0 + 1) : block;
        for (int i = tid; i < nk * d; i += kThreads) {
            const int jj = i / d, c = i % d;
            const int64_t src = (((int64_t)b * S + j0 + jj) * Hkv + g) * d + c;
            ks[jj * ld + c] = to_f32(K[src]);
            vs[jj * d + c] = to_f32(V[src]);
        }
        __syncthreads();
        // scores: thread jj owns key jj for every head of the group
        for (int jj = tid; jj < nk; jj += kThreads) {
            float s[kMaxR];
#pragma unroll
            for (int h = 0; h < kMaxR; ++h) s[h] = 0.f;
            for (int c = 0; c < d; ++c) {
                const float kv = ks[jj * ld + c];
#pragma unroll
                for (int h = 0; h < kMaxR; ++h)
                    if (h < R) s[h] = fmaf(qs[h * d + c], kv, s[h]);
            }
#pragma unroll
            for (int h = 0; h < kMaxR; ++h)
                if (h < R) ss[h * block + jj] = s[h];
        }
        __syncthreads();
        // online softmax state: one warp per head
        for (int h = warp; h < R; h += kThreads / 32) {
            float mb = -INFINITY;
            for (int jj = lane; jj < nk; jj += 32) mb = fmaxf(mb, ss[h * block + jj]);
            for (int off = 16; off > 0; off /= 2) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
            const float m_old = m_s[h];
            const float m_new = fmaxf(m_old, mb);
            float sum = 0.f;
            for (int jj = lane; jj < nk; jj += 32) {
                const float w = expf(ss[h * block + jj] - m_new);
                ss[h * block + jj] = w;
                sum += w;
            }
            for (int off = 16; off > 0; off /= 2) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            if (lane == 0) {
                const float alpha = (m_old == -INFINITY) ? 0.f : expf(m_old - m_new);
                a_s[h] = alpha;
                l_s[h] = l_s[h] * alpha + sum;
                m_s[h] = m_new;
                if (kMass) {
                    bsum[kb * R + h] = sum;
                    bmax[kb * R + h] = m_new;
                }
            }
        }
        __syncthreads();
        // values: thread c owns channel c for every head
        for (int c = tid; c < d; c += kThreads) {
#pragma unroll
            for (int h = 0; h < kMaxR; ++h) {
                if (h >= R) break;
                float a = acc[h] * a_s[h];
                for (int jj = 0; jj < nk; ++jj) a = fmaf(ss[h * block + jj], vs[jj * d + c], a);
                acc[h] = a;
            }
        }
        __syncthreads();
    }
    for (int c = tid; c < d; c += kThreads) {
#pragma unroll
        for (int h = 0; h < kMaxR; ++h) {
            if (h >= R) break;
            const float l = l_s[h];
            const float o = (l > 0.f) ? acc[h] / l : 0.f;
            O[(bt * Hq + (int64_t)g * R + h) * d + c] = from_f32<T>(o);
        }
    }
    if (tid < R) {
        const float l = l_s[tid];
        lse[bt * Hq + (int64_t)g * R + tid] = (l > 0.f) ? m_s[tid] + logf(l) : -INFINITY;
    }
    if (kMass) {
        // the indexer's KL target: each kept block's share of the softmax,
        // averaged over the group's heads (blocks past p(t) keep 0)
        for (int kb = tid; kb < nkept; kb += kThreads) {
            if ((int64_t)kept[kb] * block > p) continue;
            float share = 0.f;
            for (int h = 0; h < R; ++h)
                if (l_s[h] > 0.f) share += bsum[kb * R + h] * expf(bmax[kb * R + h] - m_s[h]) / l_s[h];
            mass[(bt * Hkv + g) * topk + kslot[kb]] = share / (float)R;
        }
    }
}

}  // namespace

cudaError_t launch_attn_simt(const Shape &s, const void *Q, const void *K, const void *V,
                             const int32_t *ids, void *O, float *lse, uint32_t *err,
                             cudaStream_t st, float *mass) {
    if (s.R > kMaxR || s.topk > kMaxTopk || s.d > kThreads) return cudaErrorInvalidConfiguration;
    const size_t smem = sizeof(float) * ((size_t)s.block * (s.d + 1) + (size_t)s.block * s.d +
                                         (size_t)s.R * s.d + (size_t)s.R * s.block + 3 * kMaxR +
                                         2 * (size_t)s.topk * s.R);
    const dim3 grid((unsigned)(s.rows() * s.Hkv));
    if (s.dtype == MSA_F32) {
        auto k = mass ? attn_simt_kernel<float, true> : attn_simt_kernel<float, false>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, kThreads, smem, st>>>((const float *)Q, (const float *)K, (const float *)V, ids,
                                        (float *)O, lse, mass, err, s.T, s.S, s.Hq, s.Hkv, s.d,
                                        s.block, s.topk, s.NB, s.scale);
    } else {
        auto k = mass ? attn_simt_kernel<__nv_bfloat16, true>
                      : attn_simt_kernel<__nv_bfloat16, false>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, kThreads, smem, st>>>((const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                                        (const __nv_bfloat16 *)V, ids, (__nv_bfloat16 *)O, lse,
                                        mass, err, s.T, s.S, s.Hq, s.Hkv, s.d, s.block, s.topk,
                                        s.NB, s.scale);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
