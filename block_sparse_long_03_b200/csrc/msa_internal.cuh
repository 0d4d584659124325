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

// Checked build (compiled with -DMSA_CHECKED=1 into libmsa_checked.so): every
// global-memory index that comes from data -- block ids, CSR tile records,
// page tables, per-sequence lengths -- is tested against the extent of its
// buffer before the access; a failed test skips the access and counts in a
// device counter (msa_bounds_failures), and nothing traps.  The normal build
// compiles the tests away.
#ifndef MSA_CHECKED
#define MSA_CHECKED 0
#endif
#if MSA_CHECKED
extern __device__ unsigned int g_msa_bounds_failures;
__device__ __forceinline__ bool in_bounds_checked(int64_t i, int64_t n) {
    if (i >= 0 && i < n) return true;
    atomicAdd(&g_msa_bounds_failures, 1u);
    return false;
}
#define MSA_IN_BOUNDS(i, n) ::msa::in_bounds_checked((int64_t)(i), (int64_t)(n))
#else
#define MSA_IN_BOUNDS(i, n) true
#endif

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

// Per-launch timing of the prefill attention (msa_profile_begin/end): an
// event on `st` before (end = false) or after (end = true) a launch of kind
// kProfAttn or kProfMerge; nothing while profiling is off.
constexpr int kProfAttn = 0, kProfMerge = 1;
cudaError_t prof_mark(cudaStream_t st, int kind, bool end);

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

// Slot lists per (batch, group, block) -- a CSR built on the device -- for
// query rows [r0, r0 + rc) of ids [B*T, G, s.topk] (s.topk <= 256): counts
// and cursor [L = B*G*NB] (zeroed here), tile_offs [L + 1] (tile_offs[L] =
// the number of tiles), and tile records of slot_csr_record_ints(tpt) ints:
// {list, entries in the tile, 0, 0, entry[0 .. tpt)} with entry =
// (row - r0) << 8 | slot.  Slots with bad or non-causal ids are skipped and
// counted in the error word.  slot_csr_records bounds the records needed.
cudaError_t launch_slot_csr(const Shape &s, const int32_t *ids, int tpt, int64_t r0, int64_t rc,
                            int *counts, int *cursor, int *toffs, int *recs, uint32_t *err,
                            cudaStream_t st);
size_t slot_csr_records(const Shape &s, int64_t rc, int tpt);
int slot_csr_record_ints(int tpt);

// The indexer's KL target of query rows [r0, r0 + rc) from their partial
// LSEs and merged lse (run after their merge).
cudaError_t launch_block_mass(const Shape &s, const int32_t *ids, const float *part_lse,
                              const float *lse, float *mass, int64_t r0, int64_t rc,
                              cudaStream_t st, const int32_t *lens = nullptr);
// Shapes the combine kernel handles: R divides 32, topk <= 256.
bool combine_supported(const Shape &s);
// LSE-weighted combine of per-(row, head, kept slot) partials into O and lse
// for query rows [r0, r0 + rc) (d = 128).
cudaError_t launch_combine(const Shape &s, const int32_t *ids, const __nv_bfloat16 *part_o,
                           float *part_lse, void *O, float *lse, int64_t r0, int64_t rc,
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
// Coarse-to-fine selection, last step: from candidates cand [rows, kc]
// (ascending ids from launch_topk with topk = kc) and their exact block
// scores fine [rows, kc], ids [rows, s.topk]: the current block and the
// s.topk - 1 best candidates below it.  kc <= 64.
cudaError_t launch_select_among(const Shape &s, const int32_t *cand, const float *fine, int kc,
                                int32_t *ids, cudaStream_t st);
// Coarse-to-fine selection (hier.cu): block-mean index keys kmean
// [B, NB, d_idx] fp32; coarse scores cs [T*G, NB] of ONE sequence (B = 1;
// only n < cb(t) written); exact scores of the candidates listed by a slot
// CSR (tpt = 128) into fine [T*G, kc].
cudaError_t launch_coarse_keys(const Shape &s, const void *k_idx, float *kmean, cudaStream_t st);
cudaError_t launch_coarse_scores(const Shape &s, const void *q_idx, const float *kmean,
                                 float *cs, cudaStream_t st);
bool fine_scores_supported(const Shape &s);
cudaError_t launch_fine_scores(const Shape &s, const void *q_idx, const void *k_idx,
                               const int *recs, const int *n_tiles, float *fine, int kc,
                               cudaStream_t st);
// Page-table check of a paged call: lens_ok[b] = lens[b] when s.T <= lens[b]
// <= s.S and every page id the sequence uses lies in [0, rows.num_pages),
// otherwise 0 (the sequence does no work) with MSA_ERR_BAD_PAGE_TABLE recorded.
cudaError_t launch_paged_check(const Shape &s, const int32_t *lens, const KeyRows &rows,
                               int32_t *lens_ok, uint32_t *err, cudaStream_t st);
cudaError_t launch_attn_simt(const Shape &s, const void *Q, const void *K, const void *V,
                             const int32_t *ids, void *O, float *lse, uint32_t *err,
                             cudaStream_t st, float *mass = nullptr);

}  // namespace msa
