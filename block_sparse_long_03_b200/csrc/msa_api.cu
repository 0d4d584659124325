// msa_api.cu -- the C ABI (include/msa.h): host-side validation, workspace
// layout and kernel dispatch.  Nothing here allocates device memory.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "msa_internal.cuh"

namespace msa {

#if MSA_CHECKED
__device__ unsigned int g_msa_bounds_failures = 0;
#endif

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// Per-launch timing (msa_profile_begin/end): event pairs per kind, recorded
// on the launching stream, summed and released at the end.
struct ProfState {
    std::mutex mu;
    std::atomic<bool> on{false};
    cudaEvent_t open[2] = {nullptr, nullptr};
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> done[2];
};
static ProfState g_prof;

static void prof_release_locked() {
    for (int k = 0; k < 2; ++k) {
        for (auto &pr : g_prof.done[k]) {
            cudaEventDestroy(pr.first);
            cudaEventDestroy(pr.second);
        }
        g_prof.done[k].clear();
        if (g_prof.open[k]) cudaEventDestroy(g_prof.open[k]);
        g_prof.open[k] = nullptr;
    }
}

cudaError_t prof_mark(cudaStream_t st, int kind, bool end) {
    if (!g_prof.on.load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(g_prof.mu);
    if (!g_prof.on.load(std::memory_order_relaxed)) return cudaSuccess;
    cudaEvent_t ev;
    cudaError_t e = cudaEventCreate(&ev);
    if (e != cudaSuccess) return e;
    if ((e = cudaEventRecord(ev, st)) != cudaSuccess) {
        cudaEventDestroy(ev);
        return e;
    }
    if (!end) {
        if (g_prof.open[kind]) cudaEventDestroy(g_prof.open[kind]);
        g_prof.open[kind] = ev;
    } else if (g_prof.open[kind]) {
        g_prof.done[kind].push_back({g_prof.open[kind], ev});
        g_prof.open[kind] = nullptr;
    } else {
        cudaEventDestroy(ev);
    }
    return cudaSuccess;
}

cudaError_t prof_begin() {
    std::lock_guard<std::mutex> lock(g_prof.mu);
    prof_release_locked();
    g_prof.on.store(true, std::memory_order_release);
    return cudaSuccess;
}

cudaError_t prof_end(double ms[2], int64_t n[2]) {
    std::lock_guard<std::mutex> lock(g_prof.mu);
    g_prof.on.store(false, std::memory_order_release);
    cudaError_t first = cudaSuccess;
    for (int k = 0; k < 2; ++k) {
        ms[k] = 0.0;
        n[k] = 0;
        for (auto &pr : g_prof.done[k]) {
            float t = 0.f;
            cudaError_t e = cudaEventSynchronize(pr.second);
            if (e == cudaSuccess) e = cudaEventElapsedTime(&t, pr.first, pr.second);
            if (e != cudaSuccess) {
                if (first == cudaSuccess) first = e;
                continue;
            }
            ms[k] += t;
            ++n[k];
        }
    }
    prof_release_locked();
    return first;
}

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Validate a parameter block; on success fill `s`.
msa_status_t make_shape(const msa_params_t *p, Shape *s) {
    if (p == nullptr) return MSA_ERR_INVALID_ARG;
    if (p->B <= 0 || p->T <= 0 || p->S <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->d <= 0 ||
        p->d_idx <= 0 || p->block <= 0 || p->topk <= 0)
        return MSA_ERR_INVALID_ARG;
    if (p->T > p->S || p->Hq % p->Hkv != 0) return MSA_ERR_INVALID_ARG;
    if (p->dtype != MSA_F32 && p->dtype != MSA_BF16) return MSA_ERR_INVALID_ARG;
    if (!(p->scale == p->scale) || isinf(p->scale)) return MSA_ERR_INVALID_ARG;
    if (p->S % p->block != 0) return MSA_ERR_UNSUPPORTED;
    if (p->d != 64 && p->d != 128) return MSA_ERR_UNSUPPORTED;
    if (p->block != 64 && p->block != 128) return MSA_ERR_UNSUPPORTED;
    if (p->d_idx % 16 != 0 || p->d_idx > 128) return MSA_ERR_UNSUPPORTED;
    if (p->Hq / p->Hkv > 16 || p->topk > 256 || p->Hkv > 256) return MSA_ERR_UNSUPPORTED;
    // every flat index must fit comfortably in int64 and the grids in 2^31
    const double q_elems = (double)p->B * p->T * p->Hq * p->d;
    const double kv_elems = (double)p->B * p->S * p->Hkv * p->d;
    const double bs_elems = (double)p->B * p->T * p->Hkv * (p->S / p->block);
    if (q_elems > 4e18 || kv_elems > 4e18 || bs_elems > 4e18) return MSA_ERR_INVALID_ARG;
    if ((double)p->B * p->T * p->Hkv > 2.0e9) return MSA_ERR_UNSUPPORTED;
    s->B = p->B; s->T = p->T; s->S = p->S; s->Hq = p->Hq; s->Hkv = p->Hkv; s->G = p->Hkv;
    s->R = p->Hq / p->Hkv; s->d = p->d; s->d_idx = p->d_idx; s->block = p->block;
    s->topk = p->topk; s->NB = p->S / p->block; s->dtype = p->dtype;
    s->scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
    return MSA_OK;
}

size_t block_score_bytes(const Shape &s) { return sizeof(float) * (size_t)s.index_rows() * s.NB; }
size_t block_id_bytes(const Shape &s) { return sizeof(int32_t) * (size_t)s.index_rows() * s.topk; }

// Prefill shapes go to the tensor-core KV-block-outer kernel; decode-like
// shapes (few query tokens per sequence) to the query-outer kernel, or to the
// tensor-core kernel where the decode kernel lacks the shape (d = 64).  fp32
// runs on CUDA cores; a bf16 shape with neither tensor-core path (a group
// size R outside {1, 2, 4, 8, 16}) is not supported rather than run there.
bool use_attn_tc(const Shape &s) {
    return attn_tc_supported(s) && (s.T >= 64 || !decode_attn_supported(s));
}
bool use_attn_decode(const Shape &s) { return !use_attn_tc(s) && decode_attn_supported(s); }
bool attn_supported(const Shape &s) {
    return s.dtype == MSA_F32 || use_attn_tc(s) || use_attn_decode(s);
}
size_t attn_scratch(const Shape &s) {
    if (use_attn_tc(s)) return align_up(attn_tc_workspace(s));
    if (use_attn_decode(s)) return align_up(decode_attn_workspace(s));
    return 0;
}

cudaError_t launch_index(const Shape &s, const void *q_idx, const void *k_idx, float *bs,
                         bool fill_noncausal, uint32_t *err, cudaStream_t st) {
    if (index_tc_supported(s))
        return launch_index_scores_tc(s, q_idx, k_idx, bs, fill_noncausal, err, st);
    if (decode_index_supported(s)) return launch_decode_index(s, q_idx, k_idx, bs, st);
    return launch_index_scores_simt(s, q_idx, k_idx, bs, st);
}

// Sequences [b0, b0 + nb), query tokens [t0, t1) of each: the whole call
// (nb = B, t0 = 0, t1 = T) or a piece of one sequence (nb = 1).
struct Piece {
    int b0, nb, t0, t1;
};

// The shape a piece's calls see: its queries are the last t1 - t0 of the
// first S - T + t1 keys, so p(t) is unchanged (t1 = T, or T - t1 a multiple
// of block, keeps S' a multiple of block).
Shape piece_shape(const Shape &s, const Piece &p) {
    Shape q = s;
    q.B = p.nb;
    q.T = p.t1 - p.t0;
    q.S = s.S - s.T + p.t1;
    q.NB = q.S / s.block;
    return q;
}

size_t elem_bytes(const Shape &s) { return s.dtype == MSA_BF16 ? 2 : 4; }

// msa_forward keeps the whole block-score array [B, T, G, NB] while it fits
// kScoreBudget; beyond that (long prefill: 128 GiB at T = S = 2^20 with four
// groups) it scores and selects in pieces of queries whose scores take at
// most kScorePiece, ending at T, T - C, T - 2C, ... of every sequence (a first
// piece under 128 queries joins the next, so every piece runs the same
// index kernel as the whole call would).  Every row's scores and ids are the
// same either way.
constexpr size_t kScoreBudget = (size_t)4 << 30;
constexpr size_t kScorePiece = (size_t)1 << 30;

int64_t score_piece_rows(const Shape &s) {
    if (block_score_bytes(s) <= kScoreBudget) return 0;
    const int64_t per_row = (int64_t)s.G * s.NB * (int64_t)sizeof(float);
    const int64_t c = std::max<int64_t>(kScorePiece / per_row / s.block * s.block, 2 * s.block);
    return c >= s.T ? 0 : c;
}

std::vector<Piece> score_pieces(const Shape &s) {
    std::vector<Piece> v;
    const int64_t c = score_piece_rows(s);
    if (c == 0) {
        v.push_back({0, s.B, 0, s.T});
        return v;
    }
    for (int b = 0; b < s.B; ++b) {
        int64_t lo = 0;
        for (int64_t k = (s.T + c - 1) / c - 1; k >= 0; --k) {
            const int64_t hi = s.T - k * c;
            if (k > 0 && hi - lo < 128) continue;
            v.push_back({b, 1, (int)lo, (int)hi});
            lo = hi;
        }
    }
    return v;
}

size_t score_bytes(const Shape &s) {
    const int64_t c = score_piece_rows(s);
    return c == 0 ? block_score_bytes(s) : (size_t)(c + 128) * s.G * s.NB * sizeof(float);
}

// Workspace layout: [error word 256 B][attention scratch]
size_t attn_ws(const Shape &s) { return kErrorBytes + attn_scratch(s); }
// msa_forward: [error word][attention scratch][block scores (or one piece's)][block ids]
size_t forward_ws(const Shape &s) {
    return kErrorBytes + attn_scratch(s) + align_up(score_bytes(s)) +
           align_up(block_id_bytes(s));
}

cudaError_t launch_attention(const Shape &s, const void *Q, const void *K, const void *V,
                             const int32_t *ids, void *O, float *lse, uint32_t *err,
                             char *scratch, cudaStream_t st, float *mass = nullptr) {
    if (use_attn_tc(s)) return launch_attn_tc(s, Q, K, V, ids, O, lse, err, scratch, st, mass);
    if (use_attn_decode(s))
        return launch_decode_attn(s, Q, K, V, ids, O, lse, err, scratch, st, mass);
    return launch_attn_simt(s, Q, K, V, ids, O, lse, err, st, mass);
}

msa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

// Device buffer bytes of msa_forward_host (defined with that call below).
size_t host_ws_size(const Shape &s);
// Workspace bytes of msa_decode_paged (defined with that call below); 0 when
// the shapes have no paged path.
size_t paged_ws_size(const Shape &s);
// Workspace bytes of msa_index_hierarchical (defined with that call below).
size_t hier_ws_size(const Shape &s);

}  // namespace
}  // namespace msa

using namespace msa;

extern "C" {

const char *msa_status_string(msa_status_t status) {
    switch (status) {
        case MSA_OK: return "MSA_OK";
        case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG: null pointer, bad shape or misaligned buffer";
        case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED: valid shape that this library does not implement";
        case MSA_ERR_CUDA: return "MSA_ERR_CUDA: a CUDA runtime call failed";
        case MSA_ERR_DEVICE_TIMEOUT: return "MSA_ERR_DEVICE_TIMEOUT: a bounded device wait gave up";
        case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case MSA_ERR_BAD_BLOCK_IDS: return "MSA_ERR_BAD_BLOCK_IDS: caller block ids out of range, not causal or repeated";
        case MSA_ERR_BAD_PAGE_TABLE: return "MSA_ERR_BAD_PAGE_TABLE: a sequence length or page id of a paged call is out of range";
    }
    return "unknown msa_status_t";
}

size_t msa_workspace_size(const msa_params_t *params, int which) {
    Shape s;
    if (make_shape(params, &s) != MSA_OK) return 0;
    if ((which == MSA_WS_SPARSE_ATTN || which == MSA_WS_FORWARD || which == MSA_WS_FORWARD_HOST) &&
        !attn_supported(s))
        return 0;
    if (which == MSA_WS_SPARSE_ATTN) return attn_ws(s);
    if (which == MSA_WS_FORWARD) return forward_ws(s);
    if (which == MSA_WS_FORWARD_HOST) return host_ws_size(s);
    if (which == MSA_WS_DECODE_PAGED) return paged_ws_size(s);
    if (which == MSA_WS_INDEX_HIER) return hier_ws_size(s);
    return 0;
}

msa_status_t msa_index_block_scores(const msa_params_t *params, const void *q_idx,
                                    const void *k_idx, float *block_scores, void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (!q_idx || !k_idx || !block_scores) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(block_scores)) return MSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    return cuda_status(launch_index(s, q_idx, k_idx, block_scores, true, nullptr, st));
}

msa_status_t msa_topk_blocks(const msa_params_t *params, const float *block_scores,
                             int32_t *block_ids, void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (!block_scores || !block_ids) return MSA_ERR_INVALID_ARG;
    if (!aligned16(block_scores) || !aligned16(block_ids)) return MSA_ERR_INVALID_ARG;
    return cuda_status(launch_topk(s, block_scores, block_ids, (cudaStream_t)stream));
}

msa_status_t msa_sparse_attn_fwd(const msa_params_t *params, const void *Q, const void *K,
                                 const void *V, const int32_t *block_ids, void *O, float *lse,
                                 void *workspace, size_t workspace_bytes, void *stream) {
    return msa_sparse_attn_fwd_mass(params, Q, K, V, block_ids, O, lse, nullptr, workspace,
                                    workspace_bytes, stream);
}

msa_status_t msa_sparse_attn_fwd_mass(const msa_params_t *params, const void *Q, const void *K,
                                      const void *V, const int32_t *block_ids, void *O,
                                      float *lse, float *block_mass, void *workspace,
                                      size_t workspace_bytes, void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (!Q || !K || !V || !block_ids || !O || !lse) return MSA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(block_ids) ||
        !aligned16(O) || !aligned16(lse) || (block_mass && !aligned16(block_mass)))
        return MSA_ERR_INVALID_ARG;
    if (!attn_supported(s)) return MSA_ERR_UNSUPPORTED;
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < attn_ws(s))
        return MSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t *err = (uint32_t *)workspace;
    cudaError_t e = cudaMemsetAsync(err, 0, kErrorBytes, st);
    if (e == cudaSuccess)
        e = launch_attention(s, Q, K, V, block_ids, O, lse, err, (char *)workspace + kErrorBytes,
                             st, block_mass);
    return cuda_status(e);
}

msa_status_t msa_forward(const msa_params_t *params, const void *q_idx, const void *k_idx,
                         const void *Q, const void *K, const void *V, int32_t *block_ids,
                         void *O, float *lse, void *workspace, size_t workspace_bytes,
                         void *stream) {
    return msa_forward_mass(params, q_idx, k_idx, Q, K, V, block_ids, O, lse, nullptr, workspace,
                            workspace_bytes, stream);
}

msa_status_t msa_forward_mass(const msa_params_t *params, const void *q_idx, const void *k_idx,
                              const void *Q, const void *K, const void *V, int32_t *block_ids,
                              void *O, float *lse, float *block_mass, void *workspace,
                              size_t workspace_bytes, void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (!q_idx || !k_idx || !Q || !K || !V || !O || !lse) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(Q) || !aligned16(K) ||
        !aligned16(V) || !aligned16(O) || !aligned16(lse) ||
        (block_ids && !aligned16(block_ids)) || (block_mass && !aligned16(block_mass)))
        return MSA_ERR_INVALID_ARG;
    if (!attn_supported(s)) return MSA_ERR_UNSUPPORTED;
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < forward_ws(s))
        return MSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    uint32_t *err = (uint32_t *)ws;
    char *scratch = ws + kErrorBytes;
    float *bs = (float *)(scratch + attn_scratch(s));
    int32_t *ids = block_ids ? block_ids : (int32_t *)((char *)bs + align_up(score_bytes(s)));
    cudaError_t e = cudaMemsetAsync(err, 0, kErrorBytes, st);
    const size_t e_sz = elem_bytes(s);
    for (const Piece &p : score_pieces(s)) {
        if (e != cudaSuccess) break;
        const Shape ps = piece_shape(s, p);
        const int64_t row0 = (int64_t)p.b0 * s.T + p.t0;
        e = launch_index(ps, (const char *)q_idx + row0 * s.G * s.d_idx * e_sz,
                         (const char *)k_idx + (int64_t)p.b0 * s.S * s.d_idx * e_sz, bs, false,
                         err, st);
        if (e == cudaSuccess) e = launch_topk(ps, bs, ids + row0 * s.G * s.topk, st);
    }
    if (e == cudaSuccess)
        e = launch_attention(s, Q, K, V, ids, O, lse, err, scratch, st, block_mass);
    return cuda_status(e);
}

uint64_t msa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

msa_status_t msa_profile_begin(void) { return msa::prof_begin() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

msa_status_t msa_profile_end(double *attn_ms, int64_t *attn_launches, double *merge_ms,
                             int64_t *merge_launches) {
    double ms[2] = {0.0, 0.0};
    int64_t n[2] = {0, 0};
    const cudaError_t e = msa::prof_end(ms, n);
    if (attn_ms) *attn_ms = ms[msa::kProfAttn];
    if (attn_launches) *attn_launches = n[msa::kProfAttn];
    if (merge_ms) *merge_ms = ms[msa::kProfMerge];
    if (merge_launches) *merge_launches = n[msa::kProfMerge];
    return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

uint32_t msa_bounds_failures(void) {
#if MSA_CHECKED
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, msa::g_msa_bounds_failures, sizeof v) != cudaSuccess)
        return 0xffffffffu;
    return v;
#else
    return 0;
#endif
}

msa_status_t msa_get_device_error(void *workspace, void *stream) {
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0) return MSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t host[4] = {0, 0, 0, 0};
    cudaError_t e = cudaMemcpyAsync(host, workspace, sizeof host, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, kErrorBytes, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    return (msa_status_t)host[0];
}

}  // extern "C"

// ---------------------------------------------------------------------------
// msa_forward_noalloc: msa_forward for callers that cannot allocate device
// memory (see include/msa.h).  Its scratch is a fixed file-scope device
// array, so every GPU that loads this library holds kNoAllocScratchBytes for
// the life of the process.
// ---------------------------------------------------------------------------
#include <mutex>

namespace msa {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)MSA_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mu;
void *g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
cudaError_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_forward_noalloc(const msa_params_t *params, const void *q_idx,
                                            const void *k_idx, const void *Q, const void *K,
                                            const void *V, int32_t *block_ids, void *O,
                                            float *lse, void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (!q_idx || !k_idx || !Q || !K || !V || !O || !lse) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(Q) || !aligned16(K) ||
        !aligned16(V) || !aligned16(O) || !aligned16(lse) ||
        (block_ids && !aligned16(block_ids)))
        return MSA_ERR_INVALID_ARG;
    if (forward_ws(s) > kNoAllocScratchBytes) return MSA_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return MSA_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    char *ws = (char *)scratch;
    uint32_t *err = (uint32_t *)ws;
    float *bs = (float *)(ws + kErrorBytes);
    int32_t *ids = block_ids ? block_ids
                             : (int32_t *)(ws + kErrorBytes + align_up(block_score_bytes(s)));
    cudaError_t e = cudaMemsetAsync(err, 0, kErrorBytes, st);   // error word starts at zero
    if (e == cudaSuccess) e = launch_index_scores_simt(s, q_idx, k_idx, bs, st);
    if (e == cudaSuccess) e = launch_topk(s, bs, ids, st);
    if (e == cudaSuccess) e = launch_attn_simt(s, Q, K, V, ids, O, lse, err, st);
    return cuda_status(e);
}

// ---------------------------------------------------------------------------
// msa_forward_host: the forward pass from page-locked host buffers, with the
// copies in both directions overlapped with the kernels (see include/msa.h).
// The caller's stream carries the kernels; two library-owned streams per
// device carry the host-to-device and device-to-host copies, joined to it by
// events.
// ---------------------------------------------------------------------------
#include <algorithm>
#include <vector>

namespace msa {
namespace {


// Query tokens per chunk, or 0 when sequences run whole.  Chunks are a
// multiple of block, about T / 16 and at least 4096 tokens, and at most one
// pass of the tensor-core attention so that no chunk is split again inside
// the call.
int64_t host_chunk(const Shape &s) {
    if (!use_attn_tc(s)) return 0;
    const int64_t blk = s.block;
    int64_t c = ((int64_t)s.T / 16 + blk - 1) / blk * blk;
    c = std::max<int64_t>(c, (4096 + blk - 1) / blk * blk);
    Shape one = s;                                  // the partial budget's rows, not capped by T
    one.B = 1;
    one.T = 1 << 30;
    c = std::min<int64_t>(c, attn_tc_rows_per_pass(one) / blk * blk);
    if (c < 4096 || c >= s.T) return 0;             // short sequences run whole
    return c;
}

// Pieces of each sequence.  Every piece but the last ends on a key-block
// boundary of p(t) (its end e has (T - e) % block == 0), so each piece's call
// of shape (T' = e - t0, S' = S - T + e) has S' a multiple of block.  The
// first piece is short (about c / 8) so the first attention starts soon after
// the copies begin, the last is short (about c / 4) so little is left to copy
// back after the last kernel, and the pieces between hold c queries.  A piece
// shorter than 128 queries is merged into the next one, so every piece runs
// the same index and attention kernels as the whole call would (the tensor-
// core kernels need 128 index rows and 64 queries) and gives the same bits.
std::vector<Piece> host_pieces(const Shape &s, int64_t c, int n_seq) {
    std::vector<Piece> v;
    if (c == 0) {
        v.push_back({0, s.B, 0, s.T});
        return v;
    }
    const int64_t blk = s.block, T = s.T;
    const int64_t phase = T % blk;                        // valid ends: phase + m * blk, and T
    auto end_at_or_after = [&](int64_t x) {               // smallest valid end >= x
        const int64_t m = x <= phase ? 0 : (x - phase + blk - 1) / blk;
        return std::min<int64_t>(T, phase + m * blk);
    };
    const int64_t first = std::max<int64_t>(blk, c / 8 / blk * blk);
    const int64_t last = std::max<int64_t>(blk, c / 4 / blk * blk);
    std::vector<int64_t> ends;
    int64_t e = end_at_or_after(std::max<int64_t>(64, first));
    while (e < T) {
        ends.push_back(e);
        e = end_at_or_after(e < T - last ? std::min<int64_t>(e + c, T - last) : T);
    }
    ends.push_back(T);
    for (int b = 0; b < n_seq; ++b) {
        int64_t lo = 0;
        for (size_t k = 0; k < ends.size(); ++k) {
            const int64_t hi = ends[k];
            if (hi - lo < 128 && k + 1 < ends.size()) continue;  // merge into the next piece
            v.push_back({b, 1, (int)lo, (int)hi});
            lo = hi;
        }
    }
    return v;
}


// Device buffer: [error word][attention scratch][block scores][block ids]
// [q_idx][k_idx][Q][K][V][O][lse], each region 256-byte aligned.
struct HostLayout {
    size_t scratch, bs, ids, q_idx, k_idx, Q, K, V, O, lse, total;
    size_t q_idx_bytes, k_idx_bytes, Q_bytes, KV_bytes, lse_bytes, ids_bytes;
};

HostLayout host_layout(const Shape &s) {
    HostLayout L;
    const size_t e = elem_bytes(s);
    L.q_idx_bytes = (size_t)s.index_rows() * s.d_idx * e;
    L.k_idx_bytes = (size_t)s.B * s.S * s.d_idx * e;
    L.Q_bytes = (size_t)s.rows() * s.Hq * s.d * e;
    L.KV_bytes = (size_t)s.B * s.S * s.Hkv * s.d * e;
    L.lse_bytes = (size_t)s.rows() * s.Hq * sizeof(float);
    L.ids_bytes = block_id_bytes(s);
    size_t scratch = 0, bs = 0;                 // the largest piece's needs
    for (const Piece &p : host_pieces(s, host_chunk(s), 1)) {
        scratch = std::max(scratch, attn_scratch(piece_shape(s, p)));
        bs = std::max(bs, block_score_bytes(piece_shape(s, p)));
    }
    size_t o = kErrorBytes;
    L.scratch = o; o += align_up(scratch);
    L.bs = o;      o += align_up(bs);
    L.ids = o;     o += align_up(L.ids_bytes);
    L.q_idx = o;   o += align_up(L.q_idx_bytes);
    L.k_idx = o;   o += align_up(L.k_idx_bytes);
    L.Q = o;       o += align_up(L.Q_bytes);
    L.K = o;       o += align_up(L.KV_bytes);
    L.V = o;       o += align_up(L.KV_bytes);
    L.O = o;       o += align_up(L.Q_bytes);
    L.lse = o;     o += align_up(L.lse_bytes);
    L.total = o;
    return L;
}

size_t host_ws_size(const Shape &s) { return host_layout(s).total; }

// True when [p, p + bytes) starts and ends in page-locked host memory.
bool page_locked(const void *p, size_t bytes) {
    if (p == nullptr || bytes == 0) return false;
    const char *ends[2] = {(const char *)p, (const char *)p + bytes - 1};
    for (const char *q : ends) {
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, q) != cudaSuccess) {
            cudaGetLastError();   // clear the sticky-free error of the query
            return false;
        }
        if (a.type != cudaMemoryTypeHost) return false;
    }
    return true;
}

struct CopyStreams {
    cudaStream_t up = nullptr, down = nullptr;   // host-to-device, device-to-host
    std::vector<cudaEvent_t> ev;
};
std::mutex g_host_mu;
CopyStreams g_copy[kMaxDevices];

// Streams of the current device and at least n events (caller holds the lock).
cudaError_t copy_streams(int dev, size_t n, CopyStreams **out) {
    CopyStreams &c = g_copy[dev];
    cudaError_t e = cudaSuccess;
    if (c.up == nullptr) e = cudaStreamCreateWithFlags(&c.up, cudaStreamNonBlocking);
    if (e == cudaSuccess && c.down == nullptr)
        e = cudaStreamCreateWithFlags(&c.down, cudaStreamNonBlocking);
    while (e == cudaSuccess && c.ev.size() < n) {
        cudaEvent_t ev;
        e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
        if (e == cudaSuccess) c.ev.push_back(ev);
    }
    *out = &c;
    return e;
}

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_forward_host(const msa_params_t *params, const void *q_idx,
                                         const void *k_idx, const void *Q, const void *K,
                                         const void *V, int32_t *block_ids, void *O, float *lse,
                                         void *device_buffer, size_t device_buffer_bytes,
                                         void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (!attn_supported(s)) return MSA_ERR_UNSUPPORTED;
    const HostLayout L = host_layout(s);
    if (!device_buffer || ((uintptr_t)device_buffer % kAlign) != 0 ||
        device_buffer_bytes < L.total)
        return MSA_ERR_WORKSPACE;
    if (!page_locked(q_idx, L.q_idx_bytes) || !page_locked(k_idx, L.k_idx_bytes) ||
        !page_locked(Q, L.Q_bytes) || !page_locked(K, L.KV_bytes) ||
        !page_locked(V, L.KV_bytes) || !page_locked(O, L.Q_bytes) ||
        !page_locked(lse, L.lse_bytes) || (block_ids && !page_locked(block_ids, L.ids_bytes)))
        return MSA_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_CUDA;

    const std::vector<Piece> pieces = host_pieces(s, host_chunk(s), s.B);
    std::lock_guard<std::mutex> lock(g_host_mu);
    CopyStreams *cs = nullptr;
    // events: start, the two joins, and three per piece
    if (copy_streams(dev, 3 + 3 * pieces.size(), &cs) != cudaSuccess) return MSA_ERR_CUDA;
    cudaEvent_t *ev = cs->ev.data();
    cudaEvent_t ev_start = ev[0], ev_up = ev[1], ev_down = ev[2];
    cudaEvent_t *ev_idx = ev + 3, *ev_in = ev_idx + pieces.size(), *ev_out = ev_in + pieces.size();
    cudaStream_t st = (cudaStream_t)stream, up = cs->up, down = cs->down;

    char *db = (char *)device_buffer;
    uint32_t *err = (uint32_t *)db;
    char *scratch = db + L.scratch;
    float *bs = (float *)(db + L.bs);
    int32_t *ids = (int32_t *)(db + L.ids);
    char *dq_idx = db + L.q_idx, *dk_idx = db + L.k_idx, *dQ = db + L.Q, *dK = db + L.K;
    char *dV = db + L.V, *dO = db + L.O;
    float *dlse = (float *)(db + L.lse);
    const char *hq_idx = (const char *)q_idx, *hk_idx = (const char *)k_idx;
    const char *hQ = (const char *)Q, *hK = (const char *)K, *hV = (const char *)V;
    char *hO = (char *)O;
    const size_t e = elem_bytes(s);
    const size_t q_row = (size_t)s.Hq * s.d * e, kv_row = (size_t)s.Hkv * s.d * e;
    const size_t qi_row = (size_t)s.G * s.d_idx * e, ki_row = (size_t)s.d_idx * e;
    const size_t id_row = (size_t)s.G * s.topk * sizeof(int32_t);

    cudaError_t ce = cudaEventRecord(ev_start, st);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(up, ev_start, 0);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(down, ev_start, 0);
    if (ce == cudaSuccess) ce = cudaMemsetAsync(err, 0, kErrorBytes, st);
    // Piece by piece: the index rows go first, so the piece's scores and
    // Top-k run while its Q and K/V rows are still being copied.
    std::vector<int64_t> keys_done((size_t)s.B, 0);   // key rows already on the device
    std::vector<int64_t> kv_done((size_t)s.B, 0);
    for (size_t i = 0; i < pieces.size() && ce == cudaSuccess; ++i) {
        const Piece &p = pieces[i];
        const Shape ps = piece_shape(s, p);
        const int64_t row0 = (int64_t)p.b0 * s.T + p.t0;   // first query token
        const size_t nq = (size_t)p.nb * (p.t1 - p.t0);    // query tokens of the piece
        const size_t kv0 = (size_t)p.b0 * s.S;              // first key row of the piece
        // index branch inputs: the piece's index queries and the keys it newly needs
        ce = cudaMemcpyAsync(dq_idx + row0 * qi_row, hq_idx + row0 * qi_row, nq * qi_row,
                             cudaMemcpyHostToDevice, up);
        for (int b = p.b0; b < p.b0 + p.nb && ce == cudaSuccess; ++b) {
            const int64_t lo = keys_done[b], hi = (int64_t)ps.S;
            if (hi <= lo) continue;
            const size_t off = ((size_t)b * s.S + lo) * ki_row;
            ce = cudaMemcpyAsync(dk_idx + off, hk_idx + off, (size_t)(hi - lo) * ki_row,
                                 cudaMemcpyHostToDevice, up);
            keys_done[b] = hi;
        }
        if (ce == cudaSuccess) ce = cudaEventRecord(ev_idx[i], up);
        // main branch inputs
        if (ce == cudaSuccess)
            ce = cudaMemcpyAsync(dQ + row0 * q_row, hQ + row0 * q_row, nq * q_row,
                                 cudaMemcpyHostToDevice, up);
        for (int b = p.b0; b < p.b0 + p.nb && ce == cudaSuccess; ++b) {
            const int64_t lo = kv_done[b], hi = (int64_t)ps.S;
            if (hi <= lo) continue;
            const size_t off = ((size_t)b * s.S + lo) * kv_row, n = (size_t)(hi - lo) * kv_row;
            ce = cudaMemcpyAsync(dK + off, hK + off, n, cudaMemcpyHostToDevice, up);
            if (ce == cudaSuccess)
                ce = cudaMemcpyAsync(dV + off, hV + off, n, cudaMemcpyHostToDevice, up);
            kv_done[b] = hi;
        }
        if (ce == cudaSuccess) ce = cudaEventRecord(ev_in[i], up);
        // kernels of the piece
        if (ce == cudaSuccess) ce = cudaStreamWaitEvent(st, ev_idx[i], 0);
        if (ce == cudaSuccess)
            ce = launch_index(ps, dq_idx + row0 * qi_row, dk_idx + kv0 * ki_row, bs, false, err,
                              st);
        if (ce == cudaSuccess) ce = launch_topk(ps, bs, ids + row0 * s.G * s.topk, st);
        if (ce == cudaSuccess) ce = cudaStreamWaitEvent(st, ev_in[i], 0);
        if (ce == cudaSuccess)
            ce = launch_attention(ps, dQ + row0 * q_row, dK + kv0 * kv_row, dV + kv0 * kv_row,
                                  ids + row0 * s.G * s.topk, dO + row0 * q_row,
                                  dlse + row0 * s.Hq, err, scratch, st);
        if (ce == cudaSuccess) ce = cudaEventRecord(ev_out[i], st);
        // outputs of the piece
        if (ce == cudaSuccess) ce = cudaStreamWaitEvent(down, ev_out[i], 0);
        if (ce == cudaSuccess)
            ce = cudaMemcpyAsync(hO + row0 * q_row, dO + row0 * q_row, nq * q_row,
                                 cudaMemcpyDeviceToHost, down);
        if (ce == cudaSuccess)
            ce = cudaMemcpyAsync(lse + row0 * s.Hq, dlse + row0 * s.Hq,
                                 nq * s.Hq * sizeof(float), cudaMemcpyDeviceToHost, down);
        if (ce == cudaSuccess && block_ids)
            ce = cudaMemcpyAsync((char *)block_ids + row0 * id_row, (char *)ids + row0 * id_row,
                                 nq * id_row, cudaMemcpyDeviceToHost, down);
    }
    // whatever happened above, later work on the caller's stream waits for
    // both copy streams
    cudaError_t je = cudaEventRecord(ev_up, up);
    if (je == cudaSuccess) je = cudaEventRecord(ev_down, down);
    if (je == cudaSuccess) je = cudaStreamWaitEvent(st, ev_up, 0);
    if (je == cudaSuccess) je = cudaStreamWaitEvent(st, ev_down, 0);
    if (ce == cudaSuccess) ce = je;
    return cuda_status(ce);
}

extern "C" int64_t msa_query_pieces(const msa_params_t *params, int which, int32_t *pieces,
                                    int64_t cap) {
    Shape s;
    if (make_shape(params, &s) != MSA_OK) return 0;
    if (cap > 0 && pieces == nullptr) return -1;
    std::vector<Piece> v;
    if (which == MSA_WS_FORWARD)
        v = score_pieces(s);
    else if (which == MSA_WS_FORWARD_HOST)
        v = host_pieces(s, host_chunk(s), s.B);
    else
        return 0;
    for (int64_t i = 0; i < (int64_t)v.size() && i < cap; ++i) {
        const bool whole = v.size() == 1 && v[i].t0 == 0 && v[i].t1 == s.T;
        pieces[3 * i] = (whole || v[i].nb > 1) ? -1 : v[i].b0;
        pieces[3 * i + 1] = v[i].t0;
        pieces[3 * i + 2] = v[i].t1;
    }
    return (int64_t)v.size();
}

// ---------------------------------------------------------------------------
// msa_decode_paged: decode steps over a paged KV cache with per-sequence
// lengths (see include/msa.h).  The decode kernels read every key row
// through the block table; a check kernel first validates the lengths and
// the page ids each sequence uses, so no kernel reads an invalid page.
// ---------------------------------------------------------------------------
namespace msa {
namespace {

bool paged_supported(const Shape &s) {
    return decode_index_supported(s) && decode_attn_supported(s);
}

// Workspace: [error word][checked lengths][decode attention scratch]
// [block scores][block ids]
struct PagedLayout {
    size_t lens, scratch, bs, ids, total;
};

PagedLayout paged_layout(const Shape &s) {
    PagedLayout L;
    size_t o = kErrorBytes;
    L.lens = o;    o += align_up(sizeof(int32_t) * (size_t)s.B);
    L.scratch = o; o += align_up(decode_attn_workspace(s));
    L.bs = o;      o += align_up(block_score_bytes(s));
    L.ids = o;     o += align_up(block_id_bytes(s));
    L.total = o;
    return L;
}

size_t paged_ws_size(const Shape &s) { return paged_supported(s) ? paged_layout(s).total : 0; }

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_decode_paged(const msa_params_t *params, const int32_t *seq_lens,
                                         const int32_t *block_table, int32_t page_size,
                                         int32_t max_pages, int32_t num_pages, const void *q_idx,
                                         const void *k_idx_cache, const void *Q,
                                         const void *K_cache, const void *V_cache,
                                         int32_t *block_ids, void *O, float *lse,
                                         void *workspace, size_t workspace_bytes, void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (page_size <= 0 || max_pages <= 0 || num_pages <= 0 ||
        (int64_t)max_pages * page_size < (int64_t)s.S)
        return MSA_ERR_INVALID_ARG;
    if (!seq_lens || !block_table || !q_idx || !k_idx_cache || !Q || !K_cache || !V_cache || !O ||
        !lse)
        return MSA_ERR_INVALID_ARG;
    if (!aligned16(seq_lens) || !aligned16(block_table) || !aligned16(q_idx) ||
        !aligned16(k_idx_cache) || !aligned16(Q) || !aligned16(K_cache) || !aligned16(V_cache) ||
        !aligned16(O) || !aligned16(lse) || (block_ids && !aligned16(block_ids)))
        return MSA_ERR_INVALID_ARG;
    if (!paged_supported(s)) return MSA_ERR_UNSUPPORTED;
    const PagedLayout L = paged_layout(s);
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < L.total)
        return MSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    uint32_t *err = (uint32_t *)ws;
    int32_t *lens_ok = (int32_t *)(ws + L.lens);
    float *bs = (float *)(ws + L.bs);
    int32_t *ids = block_ids ? block_ids : (int32_t *)(ws + L.ids);
    const KeyRows rows{block_table, (int64_t)s.S, max_pages, page_size, num_pages};
    cudaError_t e = cudaMemsetAsync(err, 0, kErrorBytes, st);
    if (e == cudaSuccess) e = launch_paged_check(s, seq_lens, rows, lens_ok, err, st);
    if (e == cudaSuccess) e = launch_decode_index(s, q_idx, k_idx_cache, bs, st, &rows, lens_ok);
    if (e == cudaSuccess) e = launch_topk(s, bs, ids, st, lens_ok);
    if (e == cudaSuccess)
        e = launch_decode_attn(s, Q, K_cache, V_cache, ids, O, lse, err, ws + L.scratch, st,
                               nullptr, &rows, lens_ok);
    return cuda_status(e);
}

// ---------------------------------------------------------------------------
// msa_index_hierarchical: coarse-to-fine block selection (see include/msa.h
// and hier.cu).  Each sequence is taken in the query pieces msa_forward
// scores in (the coarse scores have the block scores' size); per piece:
// coarse scores, the kc best candidates (Top-k kernel), their slot CSR,
// their exact scores, and the final selection among them.
// ---------------------------------------------------------------------------
namespace msa {
namespace {

constexpr int kHierMaxKc = 64;
constexpr int kHierTpt = 128;

struct HierLayout {
    size_t kmean, cs, cand, fine, counts, cursor, toffs, recs, total;
};

HierLayout hier_layout(const Shape &s) {
    Shape s1 = s;
    s1.B = 1;
    int64_t rows = 0;                              // index rows of the largest piece
    for (const Piece &p : score_pieces(s1))
        rows = std::max<int64_t>(rows, (int64_t)(p.t1 - p.t0) * s.G);
    Shape pk = s1;
    pk.topk = kHierMaxKc;
    const int64_t L = (int64_t)s.G * s.NB;
    HierLayout H;
    size_t o = kErrorBytes;
    H.kmean = o;  o += align_up(sizeof(float) * (size_t)s.B * s.NB * s.d_idx);
    H.cs = o;     o += align_up(score_bytes(s1));
    H.cand = o;   o += align_up(sizeof(int32_t) * (size_t)rows * kHierMaxKc);
    H.fine = o;   o += align_up(sizeof(float) * (size_t)rows * kHierMaxKc);
    H.counts = o; o += align_up(sizeof(int) * (size_t)L);
    H.cursor = o; o += align_up(sizeof(int) * (size_t)L);
    H.toffs = o;  o += align_up(sizeof(int) * (size_t)(L + 1));
    H.recs = o;
    o += align_up(sizeof(int) * (size_t)slot_csr_record_ints(kHierTpt) *
                  slot_csr_records(pk, rows / s.G, kHierTpt));
    H.total = o;
    return H;
}

size_t hier_ws_size(const Shape &s) {
    return fine_scores_supported(s) ? hier_layout(s).total : 0;
}

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_index_hierarchical(const msa_params_t *params, int32_t kc,
                                               const void *q_idx, const void *k_idx,
                                               int32_t *block_ids, void *workspace,
                                               size_t workspace_bytes, void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (kc < s.topk) return MSA_ERR_INVALID_ARG;
    if (kc > kHierMaxKc || !fine_scores_supported(s)) return MSA_ERR_UNSUPPORTED;
    if (!q_idx || !k_idx || !block_ids) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(block_ids))
        return MSA_ERR_INVALID_ARG;
    const HierLayout H = hier_layout(s);
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < H.total)
        return MSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    uint32_t *err = (uint32_t *)ws;
    float *kmean = (float *)(ws + H.kmean), *cs = (float *)(ws + H.cs);
    float *fine = (float *)(ws + H.fine);
    int32_t *cand = (int32_t *)(ws + H.cand);
    int *counts = (int *)(ws + H.counts), *cursor = (int *)(ws + H.cursor);
    int *toffs = (int *)(ws + H.toffs), *recs = (int *)(ws + H.recs);
    const size_t e_sz = elem_bytes(s);
    Shape s1 = s;
    s1.B = 1;
    const std::vector<Piece> pieces = score_pieces(s1);
    cudaError_t e = cudaMemsetAsync(err, 0, kErrorBytes, st);
    if (e == cudaSuccess) e = launch_coarse_keys(s, k_idx, kmean, st);
    for (int b = 0; b < s.B && e == cudaSuccess; ++b) {
        for (const Piece &p : pieces) {
            if (e != cudaSuccess) break;
            const Shape ps = piece_shape(s1, p);      // B = 1, T' = t1 - t0, S' = S - T + t1
            Shape pk = ps;
            pk.topk = kc;
            const int64_t row0 = (int64_t)b * s.T + p.t0;
            const char *q = (const char *)q_idx + row0 * s.G * s.d_idx * e_sz;
            const char *k = (const char *)k_idx + (int64_t)b * s.S * s.d_idx * e_sz;
            e = launch_coarse_scores(ps, q, kmean + (size_t)b * s.NB * s.d_idx, cs, st);
            if (e == cudaSuccess) e = launch_topk(pk, cs, cand, st);
            if (e == cudaSuccess)
                e = launch_slot_csr(pk, cand, kHierTpt, 0, ps.rows(), counts, cursor, toffs,
                                    recs, err, st);
            if (e == cudaSuccess)
                e = launch_fine_scores(ps, q, k, recs, toffs + (int64_t)ps.G * ps.NB, fine, kc,
                                       st);
            if (e == cudaSuccess)
                e = launch_select_among(ps, cand, fine, kc, block_ids + row0 * s.G * s.topk, st);
        }
    }
    return cuda_status(e);
}
