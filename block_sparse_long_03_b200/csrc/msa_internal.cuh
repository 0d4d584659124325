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
//   word[3]: number of sequences a paged call skipped (bad length or page id)
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

// Where key row j (0 <= j < its sequence's length) of sequence b lives in
// the index-key, K and V arrays: sequences of S rows one after another
// (table == nullptr), or pages of page_size rows found through a block
// table [B, max_pages] of page ids (the paged KV cache of msa_decode_paged).
struct KeyRows {
    const int32_t *table;
    int64_t S;
    int max_pages, page_size, num_pages;
    // the row index, or -1 when the page id is out of range (never loaded)
    __device__ __forceinline__ int64_t row(int b, int64_t j) const {
        if (table == nullptr) return (int64_t)b * S + j;
        const int pg = __ldg(table + (int64_t)b * max_pages + j / page_size);
        if (pg < 0 || pg >= num_pages) return -1;
        return (int64_t)pg * page_size + j % page_size;
    }
};
inline KeyRows dense_rows(int64_t S) { return KeyRows{nullptr, S, 0, 1, 0}; }

// Keys of sequence b: lens[b] when per-sequence lengths are given (a length
// of 0 marks a sequence that does no work), S otherwise.
__device__ __forceinline__ int64_t seq_len(const int32_t *lens, int b, int64_t S) {
    return lens == nullptr ? S : (int64_t)__ldg(lens + b);
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
// lens (optional, [B]): per-sequence key counts (query t of sequence b then
// sits at lens[b] - T + t; a length of 0 leaves the sequence's ids at -1).
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
                           cudaStream_t st, float *mass = nullptr,
                           const int32_t *lens = nullptr);
// Decode path (few query tokens per sequence): HBM-streaming index scoring and
// one-CTA-per-kept-block attention feeding the same combine.
bool decode_index_supported(const Shape &s);
cudaError_t launch_decode_index(const Shape &s, const void *q_idx, const void *k_idx, float *bs,
                                cudaStream_t st, const KeyRows *rows = nullptr,
                                const int32_t *lens = nullptr);
bool decode_attn_supported(const Shape &s);
size_t decode_attn_workspace(const Shape &s);
cudaError_t launch_decode_attn(const Shape &s, const void *Q, const void *K, const void *V,
                               const int32_t *ids, void *O, float *lse, uint32_t *err, void *ws,
                               cudaStream_t st, float *mass = nullptr,
                               const KeyRows *rows = nullptr, const int32_t *lens = nullptr);
cudaError_t launch_topk(const Shape &s, const float *bs, int32_t *ids, cudaStream_t st,
                        const int32_t *lens = nullptr);
// Page-table check of a paged call: lens_ok[b] = lens[b] when s.T <= lens[b]
// <= s.S and every page id the sequence uses lies in [0, rows.num_pages),
// otherwise 0 (the sequence does no work) with MSA_ERR_BAD_PAGE_TABLE recorded.
cudaError_t launch_paged_check(const Shape &s, const int32_t *lens, const KeyRows &rows,
                               int32_t *lens_ok, uint32_t *err, cudaStream_t st);
cudaError_t launch_attn_simt(const Shape &s, const void *Q, const void *K, const void *V,
                             const int32_t *ids, void *O, float *lse, uint32_t *err,
                             cudaStream_t st, float *mass = nullptr);

}  // namespace msa
