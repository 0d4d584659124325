// hier.cu -- coarse-to-fine block selection (an index-cost reducer).
//
// "LongCat Sparse Attention" (Abstract, item (3), hierarchical indexing)
// narrows each query's candidate set with a coarse-to-fine scoring scheme;
// here it is applied to MSA's max-pooled block scores ("MiniMax Sparse
// Attention", Summary, second paragraph).  Per (query, group):
//   coarse   c[n] = q_idx . kmean[n], kmean[n] the mean index key of block n,
//            for the blocks n < cb(t): d_idx multiply-adds per block instead
//            of block * d_idx;
//   select   the kc - 1 best blocks by c (the Top-k kernel with k = kc);
//   fine     the exact max-pooled block score of each candidate;
//   keep     cb(t) and the topk - 1 best candidates by fine score.
// On index inputs on the 1/4 grid every value here is exact in fp32 (block
// means are multiples of 1/1024, their dot products multiples of 1/4096
// below 2^24 units), so the selection is the fp64 definition's to the bit.
//
// The fine scores need the keys of each candidate block for the queries
// that chose it; as in the attention, the candidates are listed per
// (batch, group, block) on the device (a CSR of 128-row tiles), so a block's
// keys are staged once per tile of queries.
#include <math.h>

#include "msa_internal.cuh"

namespace msa {
namespace {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(p)));
}
// D = A (16x16, row) * B (16x8, col) + C, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Byte offset of 16-byte chunk c of row r, chunk index XOR-ed with r % 8.
__device__ __forceinline__ int swz(int r, int c, int row_bytes) {
    return r * row_bytes + ((c ^ (r & 7)) << 4);
}

// ---------------------------------------------------------------- coarse keys

// kmean[b, n, :] = the mean of block n's index keys (fp32).  One CTA per
// (batch, block), one thread per channel (coalesced rows of k_idx).
template <typename T>
__global__ void coarse_keys_kernel(const T *__restrict__ k_idx, float *__restrict__ kmean,
                                   int S, int NB, int block, int d_idx) {
    const int64_t bn = blockIdx.x;
    const int b = (int)(bn / NB), n = (int)(bn % NB);
    const float inv = 1.f / (float)block;          // block is a power of two: exact
    for (int i = threadIdx.x; i < d_idx; i += blockDim.x) {
        const T *src = k_idx + ((int64_t)b * S + (int64_t)n * block) * d_idx + i;
        float sum = 0.f;
        for (int j = 0; j < block; ++j) sum += to_f32(src[(int64_t)j * d_idx]);
        kmean[bn * d_idx + i] = sum * inv;
    }
}

// ---------------------------------------------------------------- coarse scores

// cs[r, n] = q_idx[r, :] . kmean[b, n, :] for the index rows r = (t, g) of one
// sequence and the blocks n < cb(t) (other entries are not written: the
// Top-k reads only n < cb).  CTA tile: 64 rows x 64 blocks, each of the 256
// threads 4 x 4 outputs, fp32 FMA on CUDA cores.
constexpr int kCT = 64;

template <typename T>
__global__ void __launch_bounds__(256)
coarse_scores_kernel(const T *__restrict__ q_idx, const float *__restrict__ kmean,
                     float *__restrict__ cs, int T_, int S, int G, int NB, int block, int d_idx) {
    extern __shared__ float sm[];
    const int ld = d_idx + 1;
    float *qs = sm;                                // [kCT][ld]
    float *ks = sm + kCT * ld;                     // [kCT][ld]
    const int rows = T_ * G;
    const int r0 = blockIdx.x * kCT, n0 = blockIdx.y * kCT;
    const int r_last = min(rows, r0 + kCT) - 1;
    const int cb_max = (int)(((int64_t)S - T_ + r_last / G) / block);
    if (n0 >= cb_max) return;                      // no block of this tile is a candidate
    const int tid = threadIdx.x;
    for (int i = tid; i < kCT * d_idx; i += 256) {
        const int rr = i / d_idx, c = i % d_idx;
        qs[rr * ld + c] = r0 + rr < rows ? to_f32(q_idx[(int64_t)(r0 + rr) * d_idx + c]) : 0.f;
        ks[rr * ld + c] = n0 + rr < NB ? kmean[(int64_t)(n0 + rr) * d_idx + c] : 0.f;
    }
    __syncthreads();
    const int tx = tid % 16, ty = tid / 16;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int c = 0; c < d_idx; ++c) {
        float qv[4], kv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qv[i] = qs[(ty * 4 + i) * ld + c];
#pragma unroll
        for (int j = 0; j < 4; ++j) kv[j] = ks[(tx * 4 + j) * ld + c];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + ty * 4 + i;
        if (r >= rows) break;
        const int cb = (int)(((int64_t)S - T_ + r / G) / block);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < cb) cs[(int64_t)r * NB + n] = canon_zero(acc[i][j]);
        }
    }
}

// ---------------------------------------------------------------- fine scores

// Exact block scores of the candidates, tile by tile of the candidate CSR:
// a tile is up to 128 index rows that kept candidate block n of group g.
// The CTA stages block n's index keys (cp.async, swizzled) and each warp
// computes S^T = K Q^T for 32 of the rows with mma.sync (16 keys x 8 rows x
// 16 channels per instruction; exact on grid inputs), takes the causal
// maximum over the block's keys and writes it to the row's candidate slot.
// Persistent CTAs walk the tiles.
constexpr int kFineThreads = 128;

template <int DIDX, int BLOCK>
__global__ void __launch_bounds__(kFineThreads)
fine_scores_kernel(const __nv_bfloat16 *__restrict__ q_idx, const __nv_bfloat16 *__restrict__ k_idx,
                   const int *__restrict__ recs, const int *__restrict__ n_tiles,
                   float *__restrict__ fine, int T_, int S, int G, int NB, int kc, int rec_ints) {
    constexpr int kRowBytes = DIDX * 2;
    constexpr int kChunks = DIDX / 8;
    __shared__ __align__(128) uint8_t sK[BLOCK * kRowBytes];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g4 = lane / 4, t4 = lane % 4;
    const int total = *n_tiles;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const int *rec = recs + (int64_t)tile * rec_ints;
        const int list = __ldg(rec), count = __ldg(rec + 1);
        const int n = list % NB, g = (list / NB) % G, b = list / (NB * G);
        __syncthreads();                            // the previous tile's reads of sK are done
        const __nv_bfloat16 *src = k_idx + ((int64_t)b * S + (int64_t)n * BLOCK) * DIDX;
        for (int c = threadIdx.x; c < BLOCK * kChunks; c += kFineThreads) {
            const int r = c / kChunks, ch = c % kChunks;
            cp_async16(sK + swz(r, ch, kRowBytes), src + (int64_t)r * DIDX + ch * 8);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        // B fragments (Q^T): column g4 of row group cg is the tile's row
        // 32 * warp + 8 * cg + g4
        uint32_t bq[4][DIDX / 16][2];
        int qrow[4];
        bool live[4];
#pragma unroll
        for (int cg = 0; cg < 4; ++cg) {
            const int k = 32 * warp + 8 * cg + g4;
            live[cg] = k < count;
            const int ent = live[cg] ? __ldg(rec + 4 + k) : 0;
            live[cg] = live[cg] && MSA_IN_BOUNDS(ent >> 8, T_);
            qrow[cg] = ent;
#pragma unroll
            for (int ks = 0; ks < DIDX / 16; ++ks) {
                if (live[cg]) {
                    const __nv_bfloat16 *q =
                        q_idx + ((int64_t)(ent >> 8) * G + g) * DIDX + ks * 16 + 2 * t4;
                    bq[cg][ks][0] = __ldg((const uint32_t *)q);
                    bq[cg][ks][1] = __ldg((const uint32_t *)(q + 8));
                } else {
                    bq[cg][ks][0] = bq[cg][ks][1] = 0u;
                }
            }
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        if (32 * warp >= count) continue;           // no row of this warp (after the barrier)
        // the causal position of the two rows each lane holds per row group
        int64_t pcol[4][2];
#pragma unroll
        for (int cg = 0; cg < 4; ++cg)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                // lanes 4 (2 t4 + e) .. + 3 hold the entry of this lane's column 2 t4 + e
                const int ent = __shfl_sync(0xffffffffu, qrow[cg], (2 * t4 + e) * 4);
                const int t = (ent >> 8) % T_;
                pcol[cg][e] = (int64_t)S - T_ + t;
            }
        float best[4][2];
#pragma unroll
        for (int cg = 0; cg < 4; ++cg) best[cg][0] = best[cg][1] = -INFINITY;
        const int64_t j_base = (int64_t)n * BLOCK;
#pragma unroll
        for (int mt = 0; mt < BLOCK / 16; ++mt) {
            float acc[4][4];
#pragma unroll
            for (int cg = 0; cg < 4; ++cg) acc[cg][0] = acc[cg][1] = acc[cg][2] = acc[cg][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < DIDX / 16; ++ks) {
                uint32_t a[4];
                const int r = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                ldmatrix_x4(a, sK + swz(r, 2 * ks + (lane >> 4), kRowBytes));
#pragma unroll
                for (int cg = 0; cg < 4; ++cg) mma_16816(acc[cg], a, bq[cg][ks][0], bq[cg][ks][1]);
            }
            const int64_t j0 = j_base + mt * 16 + g4;     // key of acc[.][0..1]; +8 for [2..3]
#pragma unroll
            for (int cg = 0; cg < 4; ++cg)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    if (j0 <= pcol[cg][e]) best[cg][e] = fmaxf(best[cg][e], acc[cg][e]);
                    if (j0 + 8 <= pcol[cg][e]) best[cg][e] = fmaxf(best[cg][e], acc[cg][2 + e]);
                }
        }
#pragma unroll
        for (int cg = 0; cg < 4; ++cg)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float v = best[cg][e];
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                const int k = 32 * warp + 8 * cg + 2 * t4 + e;    // the tile row of this column
                const int ent = __shfl_sync(0xffffffffu, qrow[cg], (2 * t4 + e) * 4);
                const int64_t at = ((int64_t)(ent >> 8) * G + g) * kc + (ent & 255);
                if (g4 == 0 && k < count && MSA_IN_BOUNDS(at, (int64_t)T_ * G * kc))
                    fine[at] = canon_zero(v);
            }
    }
}

}  // namespace

cudaError_t launch_coarse_keys(const Shape &s, const void *k_idx, float *kmean, cudaStream_t st) {
    const unsigned grid = (unsigned)((int64_t)s.B * s.NB);
    const int threads = s.d_idx < 128 ? s.d_idx : 128;
    if (s.dtype == MSA_F32)
        coarse_keys_kernel<float><<<grid, threads, 0, st>>>((const float *)k_idx, kmean, s.S,
                                                            s.NB, s.block, s.d_idx);
    else
        coarse_keys_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
            (const __nv_bfloat16 *)k_idx, kmean, s.S, s.NB, s.block, s.d_idx);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_coarse_scores(const Shape &s, const void *q_idx, const float *kmean,
                                 float *cs, cudaStream_t st) {
    if (s.B != 1) return cudaErrorInvalidValue;     // one sequence per call
    const size_t smem = sizeof(float) * 2 * kCT * (size_t)(s.d_idx + 1);
    const dim3 grid((unsigned)((s.T * s.G + kCT - 1) / kCT), (unsigned)((s.NB + kCT - 1) / kCT));
    if (s.dtype == MSA_F32) {
        auto k = coarse_scores_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, 256, smem, st>>>((const float *)q_idx, kmean, cs, s.T, s.S, s.G, s.NB, s.block,
                                   s.d_idx);
    } else {
        auto k = coarse_scores_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, 256, smem, st>>>((const __nv_bfloat16 *)q_idx, kmean, cs, s.T, s.S, s.G, s.NB,
                                   s.block, s.d_idx);
    }
    count_launches(1);
    return cudaGetLastError();
}

bool fine_scores_supported(const Shape &s) {
    return s.dtype == MSA_BF16 && (s.d_idx == 64 || s.d_idx == 128) &&
           (s.block == 64 || s.block == 128);
}

cudaError_t launch_fine_scores(const Shape &s, const void *q_idx, const void *k_idx,
                               const int *recs, const int *n_tiles, float *fine, int kc,
                               cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = (unsigned)(sms * 8);
    const int ri = slot_csr_record_ints(128);
    const __nv_bfloat16 *q = (const __nv_bfloat16 *)q_idx, *k = (const __nv_bfloat16 *)k_idx;
#define MSA_FINE(DI, BL)                                                                        \
    fine_scores_kernel<DI, BL><<<grid, kFineThreads, 0, st>>>(q, k, recs, n_tiles, fine, s.T,  \
                                                             s.S, s.G, s.NB, kc, ri)
    if (s.d_idx == 64 && s.block == 128) MSA_FINE(64, 128);
    else if (s.d_idx == 64) MSA_FINE(64, 64);
    else if (s.block == 128) MSA_FINE(128, 128);
    else MSA_FINE(128, 64);
#undef MSA_FINE
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
