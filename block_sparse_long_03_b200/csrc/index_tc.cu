// index_tc.cu -- index branch on the tensor cores (bf16 prefill).
//
// Block scores ("MiniMax Sparse Attention", Summary, second paragraph:
// blocks are scored by max-pooling token-level index dot products):
//   bs[b, t, g, n] = max_{j in block n, j <= p(t)} q_idx[b, t, g, :] . k_idx[b, j, :]
//
// The token-level scores form a GEMM: rows are the (token, group) pairs of
// q_idx viewed as a [B*T*G, d_idx] matrix, columns are index keys.  A work
// item is (batch entry, 256-row tile, chunk of key tiles).  Key tiles of 128
// keys stream through a TMA ring in shared memory; each is multiplied with
// the item's two 128-row A tiles (tcgen05.mma M=128, N=128, K=16 steps, bf16
// in, fp32 accumulate), so a key tile is read from L2 once per 256 rows.  The
// two products of a key tile go to one of two TMEM accumulator buffers
// (2 x 128 columns each).  Epilogue warp group g reads the 128 columns of A
// tile g (each thread one row, one TMEM round trip), applies the causal mask
// j <= p(t) and max-pools every block's columns, so only one fp32 per (row,
// block) reaches HBM.  With index inputs on the 1/4 grid every dot product is
// exact in fp32, so the scores equal the fp64 definition.
//
// Warp roles (352 threads): warp 0 TMA producer, warps 1 and 10 MMA issuers
// (even and odd key tiles, each with its own waits, so one issuer's barrier
// round trips overlap the other's tensor-core work; warp 1 owns TMEM), warps
// 2-9 epilogue in two groups of four (warp w reads TMEM lanes 32*(w%4) ..
// +31).
#include <math.h>

#include "tc.cuh"

namespace msa {
namespace {

constexpr int kM = 128;            // rows per A tile (one MMA)
constexpr int kRowsPerItem = 2 * kM;   // two A tiles share every key tile
constexpr int kN = 128;            // keys per key tile
constexpr int kThreads = 352;          // 3 + 8 warps
constexpr int kKtChunk = 64;       // key tiles per work item

struct IndexArgs {
    float *bs;
    uint32_t *err;
    int B, T, S, G, NB, block, d_idx;
    int MT;                        // 256-row tiles per batch entry
    int CPT;                       // chunks per row tile (max over tiles)
    int items;
};

struct Item {
    int b, mt, kt0, kt1, nkt;
    bool valid;
};

__device__ __forceinline__ Item decode_item(const IndexArgs &a, int i) {
    Item it;
    const int c = i % a.CPT;
    const int rest = i / a.CPT;
    it.mt = a.MT - 1 - (rest % a.MT);          // large causal ranges first
    it.b = rest / a.MT;
    const int rows = a.T * a.G;
    const int r_hi = min(rows - 1, it.mt * kRowsPerItem + kRowsPerItem - 1);
    const int64_t p_hi = (int64_t)a.S - a.T + r_hi / a.G;
    it.nkt = (int)(p_hi / kN) + 1;
    it.kt0 = c * kKtChunk;
    it.kt1 = min(it.nkt, it.kt0 + kKtChunk);
    it.valid = it.kt0 < it.nkt;
    return it;
}

// The k-th item of this CTA.  Items come roughly in decreasing size (long
// causal ranges first); alternate rounds run the CTAs in reverse order
// ("snake" order) so every CTA gets a similar share of large and small items.
__device__ __forceinline__ int cta_item(int k) {
    return k * gridDim.x + ((k & 1) ? gridDim.x - 1 - blockIdx.x : blockIdx.x);
}

template <int DIDX, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
index_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                IndexArgs a) {
    static_assert(STAGES % 2 == 0, "each MMA issuer owns the ring stages of its parity");
    constexpr int kAtoms = DIDX / 64;                     // 128-byte swizzle atoms along d_idx
    constexpr uint32_t kABytes = kM * DIDX * 2;
    constexpr uint32_t kBBytes = kN * DIDX * 2;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;                                   // [2 buffers][2 tiles][kAtoms][kM][64]
    uint8_t *sB = smem + 4 * kABytes;                     // [STAGES][kAtoms][kN][64]
    uint64_t *bar = (uint64_t *)(sB + STAGES * kBBytes);
    uint64_t *a_full = bar, *a_empty = bar + 2;
    uint64_t *b_full = bar + 4, *b_empty = bar + 4 + STAGES;
    uint64_t *acc_full = bar + 4 + 2 * STAGES, *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = (uint32_t *)(acc_empty + 2);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&a_full[i], 1);
            tc::mbar_init(&a_empty[i], 2);          // both MMA issuers
            tc::mbar_init(&acc_full[i], 1);
            tc::mbar_init(&acc_empty[i], 8);        // one arrival per epilogue warp
        }
        for (int i = 0; i < STAGES; ++i) {
            tc::mbar_init(&b_full[i], 1);
            tc::mbar_init(&b_empty[i], 1);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0, bphase = 0, abuf = 0, aphase = 0;
            for (int k = 0, i = cta_item(0); i < a.items && !*abort_flag; i = cta_item(++k)) {
                const Item it = decode_item(a, i);
                if (!it.valid) continue;
                if (!tc::mbar_wait(&a_empty[abuf], aphase ^ 1, a.err, abort_flag)) break;
                tc::mbar_expect_tx(&a_full[abuf], 2 * kABytes);
                const int row0 = it.b * a.T * a.G + it.mt * kRowsPerItem;
                for (int half = 0; half < 2; ++half)
                    for (int at = 0; at < kAtoms; ++at)
                        tc::tma_load_2d(sA + (abuf * 2 + half) * kABytes + at * kM * 128, &tm_q,
                                        &a_full[abuf], at * 64, row0 + half * kM);
                if (++abuf == 2) { abuf = 0; aphase ^= 1; }
                for (int kt = it.kt0; kt < it.kt1; ++kt) {
                    if (!tc::mbar_wait(&b_empty[stage], bphase ^ 1, a.err, abort_flag)) break;
                    tc::mbar_expect_tx(&b_full[stage], kBBytes);
                    const int key0 = it.b * a.S + kt * kN;
                    for (int at = 0; at < kAtoms; ++at)
                        tc::tma_load_2d(sB + stage * kBBytes + at * kN * 128, &tm_k,
                                        &b_full[stage], at * 64, key0);
                    if (++stage == STAGES) { stage = 0; bphase ^= 1; }
                }
            }
        }
    } else if (warp == 1 || warp == 10) {
        // ------------------------------------------------ MMA issuers
        // Key tiles are numbered across the CTA's items; issuer `par` takes
        // the tiles of its parity, which use accumulator buffer `par` and the
        // ring stages of that parity (STAGES is even).
        if (lane == 0) {
            const int par = warp == 1 ? 0 : 1;
            constexpr uint32_t idesc = tc::idesc_bf16(kM, kN, 0, 0);
            int j = 0, abuf = 0, aphase = 0;
            bool ok = true;
            for (int k = 0, i = cta_item(0); i < a.items && ok; i = cta_item(++k)) {
                const Item it = decode_item(a, i);
                if (!it.valid) continue;
                if (!tc::mbar_wait(&a_full[abuf], aphase, a.err, abort_flag)) break;
                const uint32_t a_base = tc::smem_u32(sA + abuf * 2 * kABytes);
                for (int kt = it.kt0; kt < it.kt1; ++kt) {
                    const int jj = j++;
                    if ((jj & 1) != par) continue;
                    const int stage = jj % STAGES, acc = jj & 1;
                    if (!tc::mbar_wait(&acc_empty[acc], ((jj >> 1) & 1) ^ 1, a.err, abort_flag) ||
                        !tc::mbar_wait(&b_full[stage], (jj / STAGES) & 1, a.err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t b_base = tc::smem_u32(sB + stage * kBBytes);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
#pragma unroll
                        for (int ks = 0; ks < DIDX / 16; ++ks) {
                            const uint32_t off_a = half * kABytes + (ks / 4) * kM * 128 + (ks % 4) * 32;
                            const uint32_t off_b = (ks / 4) * kN * 128 + (ks % 4) * 32;
                            tc::mma_ss(tmem + acc * 2 * kN + half * kN,
                                       tc::sdesc_sw128(a_base + off_a, 16, 1024),
                                       tc::sdesc_sw128(b_base + off_b, 16, 1024), idesc, ks > 0);
                        }
                    }
                    tc::mma_commit(&b_empty[stage]);
                    tc::mma_commit(&acc_full[acc]);
                }
                if (!ok) break;
                tc::mma_commit(&a_empty[abuf]);
                if (++abuf == 2) { abuf = 0; aphase ^= 1; }
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        // Two groups of four warps; on every key tile group `grp` reads the
        // 128 columns of A tile `grp` (one row per thread, one TMEM round
        // trip) and the accumulator buffer is released after one read per
        // group.  Warp w reads TMEM lanes 32*(w%4) .. +31.
        const int grp = (warp - 2) / 4;
        const int quad = warp % 4;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int nbpt = kN / a.block;                    // blocks per key tile (1 or 2)
        int acc = 0, accphase = 0;
        for (int k = 0, i = cta_item(0); i < a.items && !*abort_flag; i = cta_item(++k)) {
            const Item it = decode_item(a, i);
            if (!it.valid) continue;
            const int r = it.mt * kRowsPerItem + grp * kM + quad * 32 + lane;
            const bool row_ok = r < a.T * a.G;
            const int64_t p = (int64_t)a.S - a.T + r / a.G;
            float *out = a.bs + ((int64_t)it.b * a.T * a.G + r) * a.NB;
            for (int kt = it.kt0; kt < it.kt1; ++kt) {
                const int my_acc = acc, my_phase = accphase;
                if (++acc == 2) { acc = 0; accphase ^= 1; }
                if (!tc::mbar_wait(&acc_full[my_acc], my_phase, a.err, abort_flag)) break;
                tc::tc_fence_after();
                uint32_t v[4][32];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    tc::tmem_ld32(tmem + my_acc * 2 * kN + grp * kN + lane_off + u * 32, v[u]);
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                __syncwarp();                             // every lane's read is done
                if (lane == 0) tc::mbar_arrive(&acc_empty[my_acc]);
                const int64_t j0 = (int64_t)kt * kN;
                float cm[2];                                  // per 64-column chunk
                if (j0 + kN - 1 <= p) {                       // no causal mask needed
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
                        for (int q = 0; q < 32; q += 2) {
                            m0 = tc::fmax3(m0, __uint_as_float(v[2 * c][q]),
                                           __uint_as_float(v[2 * c][q + 1]));
                            m1 = tc::fmax3(m1, __uint_as_float(v[2 * c + 1][q]),
                                           __uint_as_float(v[2 * c + 1][q + 1]));
                        }
                        cm[c] = fmaxf(m0, m1);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            const int64_t j = j0 + c * 64 + q;
                            if (j <= p) m0 = fmaxf(m0, __uint_as_float(v[2 * c][q]));
                            if (j + 32 <= p) m1 = fmaxf(m1, __uint_as_float(v[2 * c + 1][q]));
                        }
                        cm[c] = fmaxf(m0, m1);
                    }
                }
                cm[0] = canon_zero(cm[0]);
                cm[1] = canon_zero(cm[1]);
                if (row_ok) {
                    if (nbpt == 1) {
                        out[kt] = fmaxf(cm[0], cm[1]);
                    } else if ((a.NB & 1) == 0) {             // rows start 8-byte aligned
                        *(float2 *)(out + 2 * kt) = make_float2(cm[0], cm[1]);
                    } else {                                  // an odd number of 64-key blocks
                        out[2 * kt] = cm[0];
                        if (2 * kt + 1 < a.NB) out[2 * kt + 1] = cm[1];
                    }
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_free(tmem, 512);
    }
}

// Blocks that start after the query's position hold no causal key and score
// -inf.  The scoring kernel writes every block up to the last key tile its
// rows need; this kernel writes blocks cb(t) + 1 .. NB - 1 of every row (the
// overlap is -inf on both sides), one warp per (token, group) row with
// 16-byte stores.  Only the standalone index call needs it: the forward
// pass's Top-k never reads past cb(t).
__global__ void fill_noncausal_kernel(float *__restrict__ bs, int64_t rows, int T, int S, int G,
                                      int NB, int block) {
    const int64_t x = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (x >= rows) return;
    const int t = (int)((x / G) % T);
    const int n0 = (int)(((int64_t)S - T + t) / block) + 1;
    if (n0 >= NB) return;
    const int64_t base = x * NB;
    float *out = bs + base;
    const int n_al = min(NB, n0 + (int)((4 - ((base + n0) & 3)) & 3));   // first 16-byte boundary
    const int n_end = n_al + ((NB - n_al) & ~3);
    if (lane < n_al - n0) out[n0 + lane] = -INFINITY;
    const float4 ninf = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    for (int n = n_al + 4 * lane; n < n_end; n += 128) *(float4 *)(out + n) = ninf;
    if (lane < NB - n_end) out[n_end + lane] = -INFINITY;
}

template <int DIDX, int STAGES>
cudaError_t launch_tc(const Shape &s, const void *q_idx, const void *k_idx, float *bs,
                      bool fill_noncausal, uint32_t *err, cudaStream_t st) {
    if (fill_noncausal) {
        const int64_t rows = s.index_rows();
        fill_noncausal_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(
            bs, rows, s.T, s.S, s.G, s.NB, s.block);
        count_launches(1);
        const cudaError_t ef = cudaGetLastError();
        if (ef != cudaSuccess) return ef;
    }
    CUtensorMap tq, tk;
    const uint64_t qd[2] = {(uint64_t)s.d_idx, (uint64_t)s.B * s.T * s.G};
    const uint64_t qs[1] = {(uint64_t)s.d_idx * 2};
    const uint32_t qb[2] = {64, kM};
    const uint64_t kd[2] = {(uint64_t)s.d_idx, (uint64_t)s.B * s.S};
    const uint32_t kb[2] = {64, kN};
    if (!make_tmap_bf16(&tq, q_idx, 2, qd, qs, qb)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&tk, k_idx, 2, kd, qs, kb)) return cudaErrorInvalidValue;
    IndexArgs a{};
    a.bs = bs; a.err = err;
    a.B = s.B; a.T = s.T; a.S = s.S; a.G = s.G; a.NB = s.NB; a.block = s.block; a.d_idx = s.d_idx;
    a.MT = (s.T * s.G + kRowsPerItem - 1) / kRowsPerItem;
    const int nkt_max = (s.S - 1) / kN + 1;
    a.CPT = (nkt_max + kKtChunk - 1) / kKtChunk;
    a.items = s.B * a.MT * a.CPT;
    const size_t smem = 1024 + 4 * (size_t)kM * DIDX * 2 + (size_t)STAGES * kN * DIDX * 2 + 256;
    auto k = index_tc_kernel<DIDX, STAGES>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = a.items < sms ? a.items : sms;
    k<<<grid, kThreads, smem, st>>>(tq, tk, a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

bool index_tc_supported(const Shape &s) {
    return s.dtype == MSA_BF16 && (s.d_idx == 64 || s.d_idx == 128) && s.T * s.G >= kM &&
           (s.block == 64 || s.block == 128);
}

cudaError_t launch_index_scores_tc(const Shape &s, const void *q_idx, const void *k_idx,
                                   float *bs, bool fill_noncausal, uint32_t *err,
                                   cudaStream_t st) {
    if (s.d_idx == 64) return launch_tc<64, 8>(s, q_idx, k_idx, bs, fill_noncausal, err, st);
    return launch_tc<128, 2>(s, q_idx, k_idx, bs, fill_noncausal, err, st);
}

}  // namespace msa
