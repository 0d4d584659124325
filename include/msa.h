/*
 * msa.h -- C ABI of the B200 (sm_100a) library for the forward pass of
 * MiniMax-Sparse-Attention-style block-sparse grouped-query attention.
 *
 * The method ("MiniMax Sparse Attention -- paper by Lai et al. (2026)",
 * section "Summary", second paragraph; section "Key points"): a light index
 * branch scores every KV block for each query by max-pooling token-level dot
 * products of an index query with index keys; each GQA group keeps its own
 * Top-k blocks, the block holding the query's own position always among
 * them; exact softmax attention then runs over the kept blocks only, and the
 * log-sum-exp of that softmax is a forward output.
 *
 * Notation used below:
 *   G = Hkv            one index head per GQA group; KV head g is group g
 *   R = Hq / Hkv       query heads per group; head h is in group h / R
 *   NB = S / block     KV blocks (S must be a multiple of block)
 *   p(t) = S - T + t   absolute position of query t (bottom-right causal
 *                      alignment; prefill with T == S gives p(t) = t)
 *   cb(t) = p(t) / block   the query's own ("current") block
 *
 * Conventions shared by every call:
 *   - Every tensor pointer is DEVICE memory (msa_forward_host alone takes
 *     page-locked host buffers), dense and row-major in the layout stated at
 *     the call, 16-byte aligned.  The caller allocates and owns all of it,
 *     workspace included; the library allocates no memory and keeps no state
 *     between calls other than per-device launch settings and the copy
 *     streams and events of msa_forward_host.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  A returned MSA_OK means the work was
 *     enqueued; device-side problems are recorded in the workspace's error
 *     word and read back with msa_get_device_error.
 *   - Invalid arguments are rejected on the host, before anything is
 *     enqueued.  No C++ exception crosses this interface.
 *   - Floating-point element type: MSA_BF16 (bf16 storage, fp32
 *     accumulation) or MSA_F32 (fp32 throughout).  The index tensors, Q, K,
 *     V and O all use params->dtype; block scores and LSE are always fp32;
 *     block ids are int32.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_EXPORT __attribute__((visibility("default")))
#else
#define MSA_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1,     /* null pointer, bad shape, misalignment     */
    MSA_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. d=96)     */
    MSA_ERR_CUDA = 3,            /* a CUDA runtime call failed                */
    MSA_ERR_DEVICE_TIMEOUT = 4,  /* a bounded device wait gave up             */
    MSA_ERR_WORKSPACE = 5,       /* workspace missing or too small            */
    MSA_ERR_BAD_BLOCK_IDS = 6,   /* caller ids out of range / not causal      */
    MSA_ERR_BAD_PAGE_TABLE = 7   /* paged call: a length or page id invalid   */
} msa_status_t;

typedef enum { MSA_F32 = 0, MSA_BF16 = 1 } msa_dtype_t;

/* Shapes of one call.  All fields are required. */
typedef struct {
    int32_t B;       /* batch (independent sequences)                       */
    int32_t T;       /* query tokens per sequence, 1 <= T <= S              */
    int32_t S;       /* keys per sequence, a multiple of block              */
    int32_t Hq;      /* query heads                                         */
    int32_t Hkv;     /* KV heads = GQA groups = index heads; Hq % Hkv == 0, */
                     /* Hq / Hkv <= 16, Hkv <= 256                          */
    int32_t d;       /* head dimension: 64 or 128                           */
    int32_t d_idx;   /* index head dimension: a multiple of 16, <= 128      */
    int32_t block;   /* KV block size B_k: 64 or 128                        */
    int32_t topk;    /* blocks kept per (query, group), current one included; */
                     /* <= 256                                              */
    int32_t dtype;   /* msa_dtype_t                                         */
    float scale;     /* softmax scale; <= 0 selects 1/sqrt(d)               */
} msa_params_t;

/* Human-readable name of a status code (static storage). */
MSA_EXPORT const char *msa_status_string(msa_status_t status);

/*
 * Index branch: block scores ("Summary", second paragraph: blocks are
 * scored by max-pooling token-level dot products).
 *
 *   block_scores[b, t, g, n] = max over j in block n with j <= p(t) of
 *                              sum_i q_idx[b, t, g, i] * k_idx[b, j, i]
 *   and -infinity when block n starts after p(t).
 *
 * q_idx        [B, T, G, d_idx]  dtype      (read)
 * k_idx        [B, S, d_idx]     dtype      (read)
 * block_scores [B, T, G, NB]     float32    (written)
 * The token-level scores are never written to memory.
 */
MSA_EXPORT msa_status_t msa_index_block_scores(const msa_params_t *params, const void *q_idx,
                                    const void *k_idx, float *block_scores, void *stream);

/*
 * Per-group Top-k over blocks with the current block forced ("Summary",
 * second paragraph: each GQA group picks its own Top-k blocks and the block
 * containing the current position is always kept; "Key points", benchmark
 * configuration: the current block is one of the k).
 *
 * For each (b, t, g): kept = {cb(t)} united with the topk - 1 best blocks
 * n < cb(t), best meaning the larger block score and, on equal scores, the
 * lower block id.  min(topk, cb(t) + 1) ids are written in ascending order
 * and the remaining slots are set to -1.  Scores are compared as fp32 and
 * never exponentiated.
 *
 * block_scores [B, T, G, NB]    float32  (read; only n < cb(t) is read)
 * block_ids    [B, T, G, topk]  int32    (written)
 */
MSA_EXPORT msa_status_t msa_topk_blocks(const msa_params_t *params, const float *block_scores,
                             int32_t *block_ids, void *stream);

/* Workspace needs, in bytes, of msa_sparse_attn_fwd (which = 0) and
 * msa_forward (which = 1) for these shapes, the device buffer of
 * msa_forward_host (which = 2, MSA_WS_FORWARD_HOST, defined with that call)
 * the workspace of msa_decode_paged (which = 3, MSA_WS_DECODE_PAGED) or of
 * msa_index_hierarchical (which = 4, MSA_WS_INDEX_HIER); 0 for invalid
 * shapes or shapes the call does not support. */
#define MSA_WS_SPARSE_ATTN 0
#define MSA_WS_FORWARD 1
MSA_EXPORT size_t msa_workspace_size(const msa_params_t *params, int which);

/*
 * Main branch: exact softmax attention over the kept blocks ("Summary",
 * second paragraph) with the log-sum-exp as a second output ("Key points",
 * kernel design: LSE is fused into the forward pass).
 *
 * For each (b, t, h) with g = h / R and J = the tokens j <= p(t) of the
 * blocks listed in block_ids[b, t, g, :] (entries < 0 are empty slots):
 *   s_j = scale * sum_c Q[b, t, h, c] * K[b, j, g, c]
 *   O[b, t, h, :] = sum_j softmax(s)_j V[b, j, g, :]
 *   lse[b, t, h]  = log(sum_j exp(s_j))      (natural log)
 * The order of the ids in a row does not matter.  Caller ids are not
 * trusted: an id >= NB, an id above cb(t) (a block with no causal token), or
 * an id repeated within a row is skipped (a repeat counts once) and the
 * device error word records MSA_ERR_BAD_BLOCK_IDS; the other ids of the row
 * are attended as usual.  A row with no attended key gets O = 0 and
 * lse = -infinity.
 *
 * Q [B, T, Hq, d], K and V [B, S, Hkv, d] (dtype, read);
 * block_ids [B, T, G, topk] int32 (read); O [B, T, Hq, d] (dtype, written);
 * lse [B, T, Hq] float32 (written).
 * workspace: device memory of at least msa_workspace_size(params, 0) bytes,
 * 256-byte aligned; its first 256 bytes hold the device error word.
 */
MSA_EXPORT msa_status_t msa_sparse_attn_fwd(const msa_params_t *params, const void *Q, const void *K,
                                 const void *V, const int32_t *block_ids, void *O, float *lse,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * The whole forward pass: index scores, Top-k and sparse attention, fused
 * where that pays.  Same meaning and layouts as the three calls above.
 * block_ids may be NULL (the ids then live in the workspace only); when not
 * NULL it receives the kept ids [B, T, G, topk].  workspace must hold
 * msa_workspace_size(params, 1) bytes.  The block scores never leave the
 * workspace; when all of them would take more than 4 GiB (long prefill),
 * the call scores and selects in pieces of consecutive queries of at most
 * 1 GiB of scores each, with the same result, so the workspace stays
 * bounded.
 */
MSA_EXPORT msa_status_t msa_forward(const msa_params_t *params, const void *q_idx, const void *k_idx,
                         const void *Q, const void *K, const void *V, int32_t *block_ids,
                         void *O, float *lse, void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * The same two calls with a third output: the target of the indexer's KL
 * objective ("Summary", second paragraph: the indexer learns to match the
 * Main Branch distribution averaged over a GQA group's heads; "Key points",
 * kernel design: the LSE that loss needs comes out of the forward pass).
 *
 *   block_mass[b, t, g, i] = (1 / R) * sum over heads h of group g of
 *       sum over the tokens j <= p(t) of block block_ids[b, t, g, i] of
 *       exp(s_j - lse[b, t, h])
 *
 * i.e. each kept slot's share of the row's softmax, averaged over the
 * group's heads, with s_j and lse as in msa_sparse_attn_fwd.  Empty slots
 * (-1), skipped caller ids (out of range, repeated) and blocks with no
 * causal token get 0; over a row's slots the masses sum to 1 (up to fp32
 * rounding) whenever the row attends to any key.  Cost: on the tensor-core
 * and decode paths one more kernel per row chunk, after the merge, reads the
 * chunk's per-(row, head, slot) partial LSEs (4 bytes each: about 1.1 GB at
 * T = 131072, Hq = 64, topk = 32) and writes block_mass; the CUDA-core path
 * keeps per-block sums in the attention kernel itself.
 *
 * block_mass [B, T, G, topk] float32 (written; 16-byte aligned).  Every other
 * argument, layout and error is that of msa_sparse_attn_fwd / msa_forward
 * (msa_forward_mass's block_ids may be NULL), with the same workspace sizes.
 */
MSA_EXPORT msa_status_t msa_sparse_attn_fwd_mass(const msa_params_t *params, const void *Q,
                                                 const void *K, const void *V,
                                                 const int32_t *block_ids, void *O, float *lse,
                                                 float *block_mass, void *workspace,
                                                 size_t workspace_bytes, void *stream);
MSA_EXPORT msa_status_t msa_forward_mass(const msa_params_t *params, const void *q_idx,
                                         const void *k_idx, const void *Q, const void *K,
                                         const void *V, int32_t *block_ids, void *O, float *lse,
                                         float *block_mass, void *workspace,
                                         size_t workspace_bytes, void *stream);

/*
 * Read the device error word of a workspace (synchronises `stream`) and
 * clear it.  Returns MSA_OK when no kernel recorded a problem, otherwise
 * the recorded status (MSA_ERR_BAD_BLOCK_IDS, MSA_ERR_DEVICE_TIMEOUT).
 */
MSA_EXPORT msa_status_t msa_get_device_error(void *workspace, void *stream);

/*
 * msa_forward for callers that cannot allocate device memory: a custom
 * allocator's own hooks (which must not re-enter the allocator they
 * implement), an embedding runtime that owns every device allocation of the
 * process, or code that must not add allocations to a tightly budgeted
 * process.  The call must still be made from an ordinary host thread: CUDA
 * forbids CUDA API calls inside a host function enqueued on a stream
 * (cudaLaunchHostFunc or a stream callback), and this call makes several
 * (device query, symbol lookup, memset, kernel launches).  The paper has no
 * counterpart of this call.
 *
 * Same meaning and layouts as msa_forward, but no workspace is passed: the
 * block scores, ids and error word live in a fixed scratch array of
 * MSA_NOALLOC_SCRATCH_BYTES that the library defines as a device global.
 * Every GPU that loads the library holds that array until the process
 * exits.  The call itself allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library routine).  It always runs the CUDA-core kernels (the
 * ones msa_forward uses for fp32): its block ids are bitwise those of
 * msa_forward, and for bf16 its O and lse agree with msa_forward's within
 * the bf16 tolerance (max-abs 2e-2 on O, 2e-3 on lse) rather than bitwise;
 * it is much slower than msa_forward on the tensor-core shapes.
 *   - Shapes whose scratch (msa_workspace_size(params, MSA_WS_FORWARD))
 *     exceeds MSA_NOALLOC_SCRATCH_BYTES are rejected with MSA_ERR_WORKSPACE
 *     before anything is enqueued.
 *   - The first call on each device looks up the array's device address
 *     (once per device, with that device current); make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array, and it keeps the last
 *     call's contents.  Calls that may overlap on the GPU (different
 *     streams, or host threads racing on the same device) race on it:
 *     serialise them.
 *   - The call clears the array's error word before its kernels run.  No
 *     call reads that word back (msa_get_device_error takes a caller
 *     workspace), so device-side errors of this call cannot be observed;
 *     the ids come from the call's own Top-k, so none are expected.
 */
#define MSA_NOALLOC_SCRATCH_BYTES (32u << 20)
MSA_EXPORT msa_status_t msa_forward_noalloc(const msa_params_t *params, const void *q_idx,
                                            const void *k_idx, const void *Q, const void *K,
                                            const void *V, int32_t *block_ids, void *O,
                                            float *lse, void *stream);

/*
 * msa_forward for inputs and outputs in page-locked HOST memory.  The call
 * copies the inputs to the device, runs the forward pass and copies O, lse
 * (and the kept ids) back, with the copies in both directions overlapped
 * with the kernels.  The paper has no counterpart of this call; the
 * arithmetic is msa_forward's, and the outputs are bitwise those of
 * msa_forward on the same inputs.
 *
 * Host buffers (same layouts and dtypes as msa_forward): q_idx, k_idx, Q, K,
 * V are read, O and lse written, block_ids written when not NULL.  Each one
 * must be page-locked over its whole extent (cudaHostAlloc, or a range
 * registered with cudaHostRegister); otherwise MSA_ERR_INVALID_ARG.
 *
 * device_buffer: device memory of at least
 * msa_workspace_size(params, MSA_WS_FORWARD_HOST) bytes, 256-byte aligned.
 * It holds the device copies of every tensor and the forward scratch; its
 * first 256 bytes are the device error word (msa_get_device_error).
 *
 * Schedule.  When a sequence is longer than one query chunk C (a multiple
 * of block chosen from the shapes: about T/16, at least 4096 tokens, and no
 * more than one pass of the tensor-core attention), each sequence is split
 * into pieces of consecutive queries: a short first piece (about C/8),
 * pieces of C, and a short last piece (about C/4), each ending where
 * T - end is a multiple of block.  For each piece the call copies its index
 * queries and the index keys it newly needs, then its Q rows and the K/V
 * rows it newly needs; the piece's index scores and Top-k run once its index
 * rows are resident, its attention once its Q, K and V rows are, and its O,
 * lse (and ids) are copied back while the next piece computes.  Shorter
 * sequences run as one piece (copy in, compute, copy out).
 *
 * Streams.  The call is ordered on `stream` like every other call: its work
 * starts after what was enqueued on `stream` before it, and work enqueued
 * on `stream` after it starts once its last copy to the host has ended.
 * The copies run on two non-blocking streams that the library creates once
 * per device, with events from a per-device pool; those streams and events
 * live until the process exits.  Calls on one device are serialised by a
 * lock while they enqueue.  The host buffers must stay valid, and O, lse and
 * block_ids unread, until `stream` has passed the call (e.g. after
 * cudaStreamSynchronize(stream)).
 */
#define MSA_WS_FORWARD_HOST 2
MSA_EXPORT msa_status_t msa_forward_host(const msa_params_t *params, const void *q_idx,
                                         const void *k_idx, const void *Q, const void *K,
                                         const void *V, int32_t *block_ids, void *O, float *lse,
                                         void *device_buffer, size_t device_buffer_bytes,
                                         void *stream);

/*
 * Coarse-to-fine block selection: an index-cost reducer that replaces
 * msa_index_block_scores + msa_topk_blocks ("LongCat Sparse Attention",
 * Abstract, item (3): hierarchical indexing narrows each query's candidate
 * set by coarse-to-fine scoring; applied here to the max-pooled block scores
 * of "MiniMax Sparse Attention", Summary, second paragraph).  The page gives
 * no formula; this call computes, per (b, t, g):
 *   1. coarse score of each block n < cb(t): q_idx[b, t, g, :] . kmean[n],
 *      kmean[n] the mean of block n's index keys (d_idx multiply-adds per
 *      block instead of block * d_idx);
 *   2. candidates: the kc - 1 best blocks n < cb(t) by coarse score (larger
 *      first, lower id on ties);
 *   3. the exact block score (as msa_index_block_scores) of each candidate;
 *      kept = {cb(t)} plus the topk - 1 best candidates by that score, same
 *      order; min(topk, cb(t) + 1) ids ascending, -1 padded.
 * With kc - 1 >= cb(t) every earlier block is a candidate and the row's ids
 * equal msa_topk_blocks' on msa_index_block_scores' scores.  The result is
 * an approximation of that selection otherwise; its recall depends on how
 * well block means rank blocks.  Feed the ids to msa_sparse_attn_fwd (for
 * this layer, or for following layers that reuse them).
 *
 * kc: candidates per (query, group), current block included: topk <= kc
 *     <= 64 (otherwise MSA_ERR_INVALID_ARG / MSA_ERR_UNSUPPORTED).
 * bf16 only, d_idx in {64, 128} (otherwise MSA_ERR_UNSUPPORTED).
 * q_idx [B, T, G, d_idx], k_idx [B, S, d_idx] (read); block_ids
 * [B, T, G, topk] int32 (written).  workspace: at least
 * msa_workspace_size(params, MSA_WS_INDEX_HIER) bytes (enough for any kc),
 * 256-byte aligned; its first 256 bytes are the device error word.  Long
 * prefills are processed in the query pieces msa_forward scores in.
 */
#define MSA_WS_INDEX_HIER 4
MSA_EXPORT msa_status_t msa_index_hierarchical(const msa_params_t *params, int32_t kc,
                                               const void *q_idx, const void *k_idx,
                                               int32_t *block_ids, void *workspace,
                                               size_t workspace_bytes, void *stream);

/*
 * Decode steps over a PAGED KV cache with per-sequence lengths: the forward
 * pass of msa_forward (index scores, per-group Top-k with the current block
 * kept, sparse attention with LSE) for a batch of sequences of different
 * lengths whose index keys, K and V live in fixed-size pages.  The method is
 * that of "MiniMax Sparse Attention" (Summary, second paragraph; Key points,
 * "Efficiency at 1M context": decoding); the paged layout and the variable
 * lengths have no counterpart in the paper and follow common serving
 * practice.
 *
 * Sequence b holds L_b = seq_lens[b] keys; its key j (0 <= j < L_b) is row
 * j % page_size of page block_table[b, j / page_size] in each cache.  Its T
 * query tokens sit at positions L_b - T + t (the last T positions), so
 * cb(t) = (L_b - T + t) / block and every definition above applies with S
 * replaced by L_b.  L_b need not be a multiple of block: the last block of
 * a sequence may be partial (its missing keys do not exist, and no query
 * sits past them).  Outputs are those of msa_forward on each sequence's
 * keys laid out densely.
 *
 * params: B sequences, T query tokens each (T * Hkv <= 32), S the capacity:
 *   a multiple of block with T <= L_b <= S; bf16, d = 128, d_idx in {64, 128}
 *   (otherwise MSA_ERR_UNSUPPORTED).
 * seq_lens     [B]                               int32 (device, read)
 * block_table  [B, max_pages]                    int32 (device, read); only
 *              the first ceil(L_b / page_size) entries of row b are read
 * page_size, max_pages, num_pages: max_pages * page_size >= S; page ids
 *              must lie in [0, num_pages)
 * q_idx        [B, T, G, d_idx]                  dtype (read)
 * k_idx_cache  [num_pages, page_size, d_idx]     dtype (read)
 * Q            [B, T, Hq, d]                     dtype (read)
 * K_cache, V_cache [num_pages, page_size, Hkv, d] dtype (read)
 * block_ids    [B, T, G, topk] int32 (written; may be NULL)
 * O            [B, T, Hq, d] (written), lse [B, T, Hq] float32 (written)
 * workspace    msa_workspace_size(params, MSA_WS_DECODE_PAGED) bytes,
 *              256-byte aligned; first 256 bytes: the device error word.
 *
 * The lengths and page ids are checked on the device before any key is
 * read: a sequence whose length is outside [T, S] or which uses a page id
 * outside [0, num_pages) is skipped (its ids -1, O = 0, lse = -infinity)
 * and the error word records MSA_ERR_BAD_PAGE_TABLE; the other sequences
 * are computed as usual.
 */
#define MSA_WS_DECODE_PAGED 3
MSA_EXPORT msa_status_t msa_decode_paged(const msa_params_t *params, const int32_t *seq_lens,
                                         const int32_t *block_table, int32_t page_size,
                                         int32_t max_pages, int32_t num_pages, const void *q_idx,
                                         const void *k_idx_cache, const void *Q,
                                         const void *K_cache, const void *V_cache,
                                         int32_t *block_ids, void *O, float *lse,
                                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * Diagnostics: the query pieces a call splits its work into, computed on the
 * host (no GPU is touched).  which = MSA_WS_FORWARD: the pieces msa_forward
 * scores and selects in (one piece when the block scores fit its budget);
 * which = MSA_WS_FORWARD_HOST: the copy/compute pieces of msa_forward_host.
 * Writes min(count, cap) pieces into `pieces` as int32 triples
 * (sequence, first query, end query), pieces of one sequence in order; a
 * piece that covers every sequence whole is reported as (-1, 0, T).
 * Returns the number of pieces, 0 for invalid shapes or `which`, and -1
 * when `pieces` is NULL with cap > 0.
 */
MSA_EXPORT int64_t msa_query_pieces(const msa_params_t *params, int which, int32_t *pieces,
                                    int64_t cap);

/*
 * Diagnostics: a check of the device failure path.  Launches one CTA that
 * takes the library's bounded mbarrier wait on a barrier nothing completes,
 * with a limit of limit_us microseconds (1 .. 1,000,000).  When the wait
 * gives up the kernel records MSA_ERR_DEVICE_TIMEOUT in the error word of
 * `workspace` (at least 256 bytes, 256-byte aligned), releases its tensor
 * memory and returns; read the status with msa_get_device_error.  Every wait
 * of the library's kernels ends this way (limit 2 s) instead of hanging.
 */
MSA_EXPORT msa_status_t msa_selftest_wait_timeout(void *workspace, size_t workspace_bytes,
                                                  uint32_t limit_us, void *stream);

/*
 * Diagnostics: the number of CUDA kernels this library has launched in this
 * process since it was loaded (all devices, all calls).  Lets a caller count
 * the kernels a region of work issued.
 */
MSA_EXPORT uint64_t msa_kernel_launches(void);

/*
 * Diagnostics: the number of device bounds checks that failed since the
 * library was loaded, in the checked build (libmsa_checked.so, compiled with
 * MSA_CHECKED=1: every global-memory index derived from data -- block ids,
 * the attention's tile records, page tables, sequence lengths -- is tested
 * against its buffer's extent; a failed test skips the access and counts
 * here, nothing traps).  Always 0 in the normal build, which has no checks.
 * Synchronises the device; 0xffffffff if the counter cannot be read.
 */
MSA_EXPORT uint32_t msa_bounds_failures(void);

/*
 * Measurement: per-kernel device time of the prefill attention.  Between
 * msa_profile_begin and msa_profile_end, every launch of the tensor-core
 * attention kernel (the KV-block-outer tiles) and of the merge kernel that
 * follows it is bracketed by two CUDA events recorded on the call's own
 * stream; msa_profile_end waits for those events, returns the summed elapsed
 * times (milliseconds) and launch counts, and releases the events.  Outputs
 * are unchanged; the event records add no kernel.  This is the one piece of
 * library state a caller switches (process-wide, guarded by a lock); calls
 * on several threads while it is on all add to the same totals.  Any output
 * pointer may be NULL.  Returns MSA_ERR_CUDA if an event call fails (the
 * totals then cover the launches before the failure).
 */
MSA_EXPORT msa_status_t msa_profile_begin(void);
MSA_EXPORT msa_status_t msa_profile_end(double *attn_ms, int64_t *attn_launches,
                                        double *merge_ms, int64_t *merge_launches);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
