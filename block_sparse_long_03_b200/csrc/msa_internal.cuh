// msa_internal.cuh -- declarations shared by the library's translation units.
// Not part of the public interface (that is include/msa.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/msa.h"

namespace msa {

// Shapes after host-side validation, with derived sizes.
struct Shape {
    int B, T, S, Hq, Hkv, G, R, d, d_idx, block, topk, NB;
    int dtype;          // MSA_F32 or MSA_BF16
    float scale;        // resolved softmax scale
    int64_t rows() const { return (int64_t)B * T; }          // query tokens
    int64_t index_rows() const { return rows() * G; }        // (token, group) rows
};

// Device error word: the first 256 bytes of every workspace.
//   word[0]: first recorded msa_status_t (0 = none)
//   word[1]: number of caller block ids skipped as invalid
//   word[2]: number of bounded device waits that gave up
constexpr size_t kErrorBytes = 256;

__device__ __forceinline__ void record_error(uint32_t *err, uint32_t code, int counter) {
    if (err == nullptr) return;
    atomicCAS(err, 0u, code);
    atomicAdd(err + counter, 1u);
}

// A block score of -0.0 (every product of a zero dot product negative zero)
// is stored as +0.0: scores compare as numbers, and the stored bits then
// match a sum that starts from +0.0.
__device__ __forceinline__ float canon_zero(float x) {
    return __float_as_uint(x) == 0x80000000u ? 0.f : x;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Every kernel launch of the library is counted (msa_kernel_launches).
void count_launches(int n);

// Launchers (each returns a cudaError_t from the launch).
cudaError_t launch_index_scores_simt(const Shape &s, const void *q_idx, const void *k_idx,
                                     float *bs, cudaStream_t st);
// Tensor-core index scoring (bf16, d_idx in {64, 128}, at least 128 index rows).
bool index_tc_supported(const Shape &s);
cudaError_t launch_index_scores_tc(const Shape &s, const void *q_idx, const void *k_idx,
                                   float *bs, bool fill_noncausal, uint32_t *err,
                                   cudaStream_t st);
// Tensor-core KV-block-outer sparse attention (bf16, d = 128) and its workspace.
bool attn_tc_supported(const Shape &s);
size_t attn_tc_workspace(const Shape &s);
// Query tokens one pass of the tensor-core attention covers (its partials fit
// a fixed budget); larger calls run several passes.
int64_t attn_tc_rows_per_pass(const Shape &s);
// mass (optional, [rows, G, topk] fp32): each kept slot's share of the row's
// softmax averaged over the group's heads (0 for slots that attend nothing).
cudaError_t launch_attn_tc(const Shape &s, const void *Q, const void *K, const void *V,
                           const int32_t *ids, void *O, float *lse, uint32_t *err, void *ws,
                           cudaStream_t st, float *mass = nullptr);
// Partial outputs (bf16, one row of d channels per (query row, head, kept
// slot)) are stored in 16-byte chunks, blocked by 32 rows: the chunk c of row
// prow is uint4 number partial_chunk(prow, c).  Consecutive rows of one chunk
// are adjacent (coalesced stores), and all chunks of 32 rows share one
// contiguous d/8 * 512-byte span (page-local reads).
__host__ __device__ __forceinline__ int64_t partial_chunk(int64_t prow, int c, int d) {
    return (prow >> 5) * (int64_t)(d / 8) * 32 + (int64_t)c * 32 + (prow & 31);
}

// Shapes the combine kernel handles: R divides 32, topk <= 64, topk * R <= 512.
bool combine_supported(const Shape &s);
// LSE-weighted combine of per-(row, head, kept slot) partials into O and lse
// for query rows [r0, r0 + rc) (d = 128).
cudaError_t launch_combine(const Shape &s, const int32_t *ids, const __nv_bfloat16 *part_o,
                           const float *part_lse, void *O, float *lse, int64_t r0, int64_t rc,
                           cudaStream_t st, float *mass = nullptr);
// Decode path (few query tokens per sequence): HBM-streaming index scoring and
// one-CTA-per-kept-block attention feeding the same combine.
bool decode_index_supported(const Shape &s);
cudaError_t launch_decode_index(const Shape &s, const void *q_idx, const void *k_idx, float *bs,
                                cudaStream_t st);
bool decode_attn_supported(const Shape &s);
size_t decode_attn_workspace(const Shape &s);
cudaError_t launch_decode_attn(const Shape &s, const void *Q, const void *K, const void *V,
                               const int32_t *ids, void *O, float *lse, uint32_t *err, void *ws,
                               cudaStream_t st, float *mass = nullptr);
cudaError_t launch_topk(const Shape &s, const float *bs, int32_t *ids, cudaStream_t st);
cudaError_t launch_attn_simt(const Shape &s, const void *Q, const void *K, const void *V,
                             const int32_t *ids, void *O, float *lse, uint32_t *err,
                             cudaStream_t st, float *mass = nullptr);

}  // namespace msa
