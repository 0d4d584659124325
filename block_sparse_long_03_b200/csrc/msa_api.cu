// msa_api.cu -- the C ABI (include/msa.h): host-side validation, workspace
// layout and kernel dispatch.  Nothing here allocates device memory.
#include <math.h>
#include <string.h>

#include <atomic>

#include "msa_internal.cuh"

namespace msa {

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

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
    if (p->Hq / p->Hkv > 16 || p->topk > 256) return MSA_ERR_UNSUPPORTED;
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
// shapes (few query tokens per sequence) to the query-outer kernel.
bool use_attn_tc(const Shape &s) { return attn_tc_supported(s) && s.T >= 64; }
bool use_attn_decode(const Shape &s) { return !use_attn_tc(s) && decode_attn_supported(s); }
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

// Workspace layout: [error word 256 B][attention scratch]
size_t attn_ws(const Shape &s) { return kErrorBytes + attn_scratch(s); }
// msa_forward: [error word][attention scratch][block scores][block ids]
size_t forward_ws(const Shape &s) {
    return kErrorBytes + attn_scratch(s) + align_up(block_score_bytes(s)) +
           align_up(block_id_bytes(s));
}

cudaError_t launch_attention(const Shape &s, const void *Q, const void *K, const void *V,
                             const int32_t *ids, void *O, float *lse, uint32_t *err,
                             char *scratch, cudaStream_t st) {
    if (use_attn_tc(s)) return launch_attn_tc(s, Q, K, V, ids, O, lse, err, scratch, st);
    if (use_attn_decode(s)) return launch_decode_attn(s, Q, K, V, ids, O, lse, err, scratch, st);
    return launch_attn_simt(s, Q, K, V, ids, O, lse, err, st);
}

msa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

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
        case MSA_ERR_BAD_BLOCK_IDS: return "MSA_ERR_BAD_BLOCK_IDS: caller block ids out of range or repeated";
    }
    return "unknown msa_status_t";
}

size_t msa_workspace_size(const msa_params_t *params, int which) {
    Shape s;
    if (make_shape(params, &s) != MSA_OK) return 0;
    if (which == MSA_WS_SPARSE_ATTN) return attn_ws(s);
    if (which == MSA_WS_FORWARD) return forward_ws(s);
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
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (!Q || !K || !V || !block_ids || !O || !lse) return MSA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(block_ids) ||
        !aligned16(O) || !aligned16(lse))
        return MSA_ERR_INVALID_ARG;
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < attn_ws(s))
        return MSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t *err = (uint32_t *)workspace;
    cudaError_t e = cudaMemsetAsync(err, 0, kErrorBytes, st);
    if (e == cudaSuccess)
        e = launch_attention(s, Q, K, V, block_ids, O, lse, err, (char *)workspace + kErrorBytes, st);
    return cuda_status(e);
}

msa_status_t msa_forward(const msa_params_t *params, const void *q_idx, const void *k_idx,
                         const void *Q, const void *K, const void *V, int32_t *block_ids,
                         void *O, float *lse, void *workspace, size_t workspace_bytes,
                         void *stream) {
    Shape s;
    msa_status_t rc = make_shape(params, &s);
    if (rc != MSA_OK) return rc;
    if (!q_idx || !k_idx || !Q || !K || !V || !O || !lse) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(Q) || !aligned16(K) ||
        !aligned16(V) || !aligned16(O) || !aligned16(lse) ||
        (block_ids && !aligned16(block_ids)))
        return MSA_ERR_INVALID_ARG;
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < forward_ws(s))
        return MSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    uint32_t *err = (uint32_t *)ws;
    char *scratch = ws + kErrorBytes;
    float *bs = (float *)(scratch + attn_scratch(s));
    int32_t *ids = block_ids ? block_ids
                             : (int32_t *)((char *)bs + align_up(block_score_bytes(s)));
    cudaError_t e = cudaMemsetAsync(err, 0, kErrorBytes, st);
    if (e == cudaSuccess) e = launch_index(s, q_idx, k_idx, bs, false, err, st);
    if (e == cudaSuccess) e = launch_topk(s, bs, ids, st);
    if (e == cudaSuccess) e = launch_attention(s, Q, K, V, ids, O, lse, err, scratch, st);
    return cuda_status(e);
}

uint64_t msa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

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
