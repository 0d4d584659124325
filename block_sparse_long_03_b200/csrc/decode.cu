// decode.cu -- the forward pass for few query tokens per sequence (decode).
//
// Same definitions as the prefill path ("MiniMax Sparse Attention", Summary,
// second paragraph; Key points: decoding and the two-phase combine):
//   index   bs[b, t, g, n] = max_{j in block n, j <= p(t)} q_idx[b, t, g, :] . k_idx[b, j, :]
//   attend  per kept block a partial softmax (normalised O and its LSE), then
//           the LSE-weighted combine shared with the prefill path.
//
// With one query per sequence the index contraction is a matrix-vector
// product per sequence: the whole of k_idx is streamed from HBM once and
// scored against the T*G index queries of its sequence, so the index kernel
// is HBM-bound.  It uses warp-level mma.sync (16 keys x 8 query columns x 16
// channels per instruction, fp32 accumulation; exact on the 1/4-grid inputs):
// the N = 8 shape matches the 8 (token, group) columns of a decode step,
// which is too narrow for a tcgen05 tile.  Keys are staged in shared memory
// with 16-byte cp.async copies into a XOR-swizzled layout and read back with
// ldmatrix without bank conflicts.
//
// The attention kernel runs one small CTA per (query row, group, kept slot):
// it stages the block's K and V rows (cp.async, swizzled), computes
// S^T = K Q^T and O^T = V^T P with mma.sync, and writes the block's partial
// in the same layout as the prefill kernel, so one combine kernel serves
// both paths.  The work is spread over B * T * G * topk CTAs, enough to keep
// HBM busy with a single kept block per CTA.
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
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(p)));
}
// D = A (16x16, row) * B (16x8, col) + C, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk `c` of row `r` in a row-major tile whose rows
// are `row_bytes` long, with the chunk index XOR-ed by (r % 8) so that the 8
// row addresses of one ldmatrix hit 8 different bank groups.
__device__ __forceinline__ int swz(int r, int c, int row_bytes) {
    return r * row_bytes + ((c ^ (r & 7)) << 4);
}

// ---------------------------------------------------------------- index

// One warp scores whole KV blocks of one sequence, 64 keys (a "sub-block")
// at a time, against up to 8*NCG (token, group) columns; sub-blocks are
// double-buffered in shared memory.  Key rows are found through `rows`
// (dense or paged); keys at or past the sequence's length L are never read
// (zero in shared memory, and masked: every query sits before L).
template <int DIDX, int NCG, int WARPS, bool kPaged>
__global__ void __launch_bounds__(WARPS * 32)
decode_index_kernel(const __nv_bfloat16 *__restrict__ q_idx, const __nv_bfloat16 *__restrict__ k_idx,
                    float *__restrict__ bs, int T_, int S, int G, int NB, int block,
                    int blocks_per_warp, KeyRows rows, const int32_t *__restrict__ lens,
                    int64_t kv_rows) {
    constexpr int kRowBytes = DIDX * 2;
    constexpr int kChunks = DIDX / 8;
    constexpr int kSub = 64;                               // keys per staged sub-block
    constexpr int kTileBytes = kSub * kRowBytes;
    extern __shared__ __align__(128) uint8_t sm[];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int b = blockIdx.y;
    const int TG = T_ * G;
    uint8_t *buf0 = sm + (size_t)warp * 2 * kTileBytes;
    const int g4 = lane / 4, t4 = lane % 4;
    const int64_t L = seq_len(lens, b, S);
    const int first_blk = (blockIdx.x * WARPS + warp) * blocks_per_warp;
    const int last_blk = min(NB, first_blk + blocks_per_warp);
    if ((int64_t)first_blk * block >= L) {                 // no key of these blocks exists
        for (int i = lane; i < (last_blk - first_blk) * TG; i += 32) {
            const int col = i % TG, n = first_blk + i / TG;
            bs[((int64_t)b * TG + col) * NB + n] = -INFINITY;
        }
        return;
    }

    // B fragments: column n = 8 * cg + g4 is (token, group) pair n of this sequence
    uint32_t bq[NCG][DIDX / 16][2];
#pragma unroll
    for (int cg = 0; cg < NCG; ++cg) {
        const int n = cg * 8 + g4;
#pragma unroll
        for (int ks = 0; ks < DIDX / 16; ++ks) {
            if (n < TG) {
                const __nv_bfloat16 *q = q_idx + ((int64_t)b * TG + n) * DIDX + ks * 16 + 2 * t4;
                bq[cg][ks][0] = *(const uint32_t *)q;
                bq[cg][ks][1] = *(const uint32_t *)(q + 8);
            } else {
                bq[cg][ks][0] = bq[cg][ks][1] = 0u;
            }
        }
    }
    // causal position of the two columns this thread holds in each column group
    int64_t pcol[NCG][2];
#pragma unroll
    for (int cg = 0; cg < NCG; ++cg)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = cg * 8 + 2 * t4 + e;
            pcol[cg][e] = L - T_ + (n < TG ? n / G : 0);
        }

    const int spb = block / kSub;                          // sub-blocks per block
    const int first = first_blk * spb, last = last_blk * spb;
    auto stage = [&](int sb, uint8_t *dst) {
        if (!kPaged) {                                     // whole sequences of S keys
            const __nv_bfloat16 *src = k_idx + ((int64_t)b * S + (int64_t)sb * kSub) * DIDX;
            for (int c = lane; c < kSub * kChunks; c += 32) {
                const int r = c / kChunks, ch = c % kChunks;
                cp_async16(dst + swz(r, ch, kRowBytes), src + (int64_t)r * DIDX + ch * 8);
            }
        } else {
            // one page-table lookup per key row (lane l: rows l and l + 32),
            // handed to the lanes copying that row's chunks by a shuffle
            static_assert(kSub == 64, "two key rows per lane");
            const int64_t j0 = (int64_t)sb * kSub;
            int64_t rw0, rw1;
            if (rows.page_size % kSub == 0) {              // the sub-block lies in one page
                const int64_t base = rows.row(b, j0);      // one lookup, the same in every lane
                rw0 = j0 + lane < L && base >= 0 ? base + lane : -1;
                rw1 = j0 + lane + 32 < L && base >= 0 ? base + lane + 32 : -1;
            } else {
                rw0 = j0 + lane < L ? rows.row(b, j0 + lane) : -1;
                rw1 = j0 + lane + 32 < L ? rows.row(b, j0 + lane + 32) : -1;
            }
            for (int c = lane; c < kSub * kChunks; c += 32) {
                const int r = c / kChunks, ch = c % kChunks;     // r < 32 is uniform per step
                const int64_t row = __shfl_sync(0xffffffffu, r < 32 ? rw0 : rw1, r & 31);
                if (row >= 0 && MSA_IN_BOUNDS(row, kv_rows))
                    cp_async16(dst + swz(r, ch, kRowBytes), k_idx + row * DIDX + ch * 8);
                else
                    *(uint4 *)(dst + swz(r, ch, kRowBytes)) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        cp_async_commit();
    };
    float best[NCG][2];
#pragma unroll
    for (int cg = 0; cg < NCG; ++cg) best[cg][0] = best[cg][1] = -INFINITY;
    if (first < last) stage(first, buf0);
    for (int sb = first; sb < last; ++sb) {
        uint8_t *cur = buf0 + ((sb - first) & 1) * kTileBytes;
        if (sb + 1 < last) {
            stage(sb + 1, buf0 + ((sb + 1 - first) & 1) * kTileBytes);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
#pragma unroll
        for (int mt = 0; mt < kSub / 16; ++mt) {
            float acc[NCG][4];
#pragma unroll
            for (int cg = 0; cg < NCG; ++cg) acc[cg][0] = acc[cg][1] = acc[cg][2] = acc[cg][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < DIDX / 16; ++ks) {
                uint32_t a[4];
                const int r = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                ldmatrix_x4(a, cur + swz(r, 2 * ks + (lane >> 4), kRowBytes));
#pragma unroll
                for (int cg = 0; cg < NCG; ++cg) mma_bf16_16816(acc[cg], a, bq[cg][ks][0], bq[cg][ks][1]);
            }
            const int64_t j0 = (int64_t)sb * kSub + mt * 16 + g4;   // key of acc[.][0..1]
#pragma unroll
            for (int cg = 0; cg < NCG; ++cg)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    if (j0 <= pcol[cg][e]) best[cg][e] = fmaxf(best[cg][e], acc[cg][e]);
                    if (j0 + 8 <= pcol[cg][e]) best[cg][e] = fmaxf(best[cg][e], acc[cg][2 + e]);
                }
        }
        __syncwarp();                                      // buffer free for the next stage
        if ((sb + 1) % spb == 0) {                         // block complete: reduce and write
            const int n = sb / spb;
#pragma unroll
            for (int cg = 0; cg < NCG; ++cg)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = best[cg][e];
                    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                    const int col = cg * 8 + 2 * t4 + e;
                    if (g4 == 0 && col < TG) bs[((int64_t)b * TG + col) * NB + n] = canon_zero(v);
                    best[cg][e] = -INFINITY;
                }
        }
    }
}

// ---------------------------------------------------------------- attention

constexpr int kAttnThreads = 128;

// One CTA = one kept slot of one (query row, group) and up to 8 of the
// group's query heads (the width of one mma tile): the partial softmax of
// those heads over that block's causal keys.  With R = 16 two CTAs share a
// slot, heads 0-7 and 8-15.
template <int D, int BLOCK, bool kPaged>
__global__ void __launch_bounds__(kAttnThreads)
decode_block_kernel(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
                    const __nv_bfloat16 *__restrict__ V, const int32_t *__restrict__ ids,
                    __nv_bfloat16 *__restrict__ part_o, float *__restrict__ part_lse, uint32_t *err,
                    int T_, int S, int Hq, int Hkv, int R, int NB, int topk, float scale_log2,
                    float scale, int64_t n_prows, KeyRows rows, const int32_t *__restrict__ lens,
                    int64_t kv_rows) {
    constexpr int kRowBytes = D * 2;
    constexpr int kChunks = D / 8;
    extern __shared__ __align__(128) uint8_t sm[];
    uint8_t *sK = sm;                                      // [BLOCK][D] swizzled
    uint8_t *sV = sK + BLOCK * kRowBytes;                  // [BLOCK][D] swizzled
    __nv_bfloat16 *sP = (__nv_bfloat16 *)(sV + BLOCK * kRowBytes);   // [8 heads][BLOCK]
    float *sRed = (float *)(sP + 8 * BLOCK);               // [4 warps][8] maxima, then sums
    float *sMax = sRed + 4 * 8;                            // [8] per-head maximum
    __nv_bfloat16 *sO = (__nv_bfloat16 *)(sMax + 8);       // [8 heads][D]

    const int nhalf = (R + 7) / 8;                         // CTAs per kept slot
    const int h0 = (int)(blockIdx.x % nhalf) * 8;          // first head of this CTA
    const int Rh = R - h0 < 8 ? R - h0 : 8;                // heads of this CTA
    const int slot = (int)((blockIdx.x / nhalf) % topk);
    const int64_t rg = blockIdx.x / nhalf / topk;          // (b * T + t) * G + g
    const int g = (int)(rg % Hkv);
    const int64_t bt = rg / Hkv;
    const int b = (int)(bt / T_), t = (int)(bt % T_);
    const int64_t p = seq_len(lens, b, S) - T_ + t;
    if (p < 0) return;                                     // a sequence marked as doing no work
    const int cb = (int)(p / BLOCK);
    const int32_t *row = ids + rg * topk;
    // validity of this slot (same rule as every other phase): the range is
    // checked before the block's copies are issued, repeats while they fly
    const int n = row[slot];
    if (n < 0) return;
    if (n >= NB) {
        if (threadIdx.x == 0 && h0 == 0) record_error(err, MSA_ERR_BAD_BLOCK_IDS, 1);
        return;
    }
    const int64_t j0 = (int64_t)n * BLOCK;
    const int nk = (int)((p - j0 + 1 < BLOCK) ? (p - j0 + 1) : BLOCK);   // <= 0 past cb

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int g4 = lane / 4, t4 = lane % 4;
    // stage K and V rows of the block (zero rows past the last causal key);
    // a paged cache takes one page-table lookup per key row, shared through
    // shared memory
    int64_t *s_rows = nullptr;
    int64_t page_base = -1;                            // a block inside one page: its first row
    const bool one_page = kPaged && rows.page_size % BLOCK == 0;
    if constexpr (kPaged) {
        if (one_page) {
            page_base = nk > 0 ? rows.row(b, j0) : -1;
        } else {
            __shared__ int64_t s_rows_buf[BLOCK];
            for (int r = tid; r < BLOCK; r += kAttnThreads)
                s_rows_buf[r] = r < nk ? rows.row(b, j0 + r) : -1;
            __syncthreads();
            s_rows = s_rows_buf;
        }
    }
    for (int c = tid; c < BLOCK * kChunks; c += kAttnThreads) {
        const int r = c / kChunks, ch = c % kChunks;
        const int64_t kr = r >= nk ? -1
                           : !kPaged ? (int64_t)b * S + j0 + r
                           : one_page ? (page_base >= 0 ? page_base + r : -1) : s_rows[r];
        if (kr >= 0 && MSA_IN_BOUNDS(kr, kv_rows)) {
            const int64_t src = (kr * Hkv + g) * D + ch * 8;
            cp_async16(sK + swz(r, ch, kRowBytes), K + src);
            cp_async16(sV + swz(r, ch, kRowBytes), V + src);
        } else {
            *(uint4 *)(sK + swz(r, ch, kRowBytes)) = make_uint4(0, 0, 0, 0);
            *(uint4 *)(sV + swz(r, ch, kRowBytes)) = make_uint4(0, 0, 0, 0);
        }
    }
    cp_async_commit();
    // an id repeated within the row counts once: later slots are reported and skipped
    bool repeat = false;
    for (int i0 = 0; i0 < slot; i0 += 32) {
        const int i = i0 + lane;
        repeat |= __any_sync(0xffffffffu, i < slot && row[i] == n);
    }
    if (repeat || n > cb) {                                // n > cb: no causal token
        cp_async_wait<0>();                                // this CTA's copies land first
        if (threadIdx.x == 0 && h0 == 0) record_error(err, MSA_ERR_BAD_BLOCK_IDS, 1);
        return;
    }
    // B fragments of Q^T: column g4 = head (zero past R)
    uint32_t bq[D / 16][2];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        if (g4 < Rh) {
            const __nv_bfloat16 *q =
                Q + (bt * Hq + (int64_t)g * R + h0 + g4) * D + ks * 16 + 2 * t4;
            bq[ks][0] = *(const uint32_t *)q;
            bq[ks][1] = *(const uint32_t *)(q + 8);
        } else {
            bq[ks][0] = bq[ks][1] = 0u;
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // S^T = K Q^T: warp w owns key rows [16 w, 16 w + 16) (+ 64 for BLOCK = 128)
    constexpr int kMT = BLOCK / 16 / 4;                    // key m-tiles per warp
    float s[kMT][4];
#pragma unroll
    for (int mi = 0; mi < kMT; ++mi) {
        s[mi][0] = s[mi][1] = s[mi][2] = s[mi][3] = 0.f;
        const int mt = warp + 4 * mi;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4];
            const int r = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
            ldmatrix_x4(a, sK + swz(r, 2 * ks + (lane >> 4), kRowBytes));
            mma_bf16_16816(s[mi], a, bq[ks][0], bq[ks][1]);
        }
    }
    // row max per head (columns 2 t4, 2 t4 + 1), masked past the causal end
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mi = 0; mi < kMT; ++mi) {
        const int key = (warp + 4 * mi) * 16 + g4;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (key < nk) mx[e] = fmaxf(mx[e], s[mi][e]);
            if (key + 8 < nk) mx[e] = fmaxf(mx[e], s[mi][2 + e]);
        }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 4));
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 8));
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 16));
    }
    if (g4 == 0) { sRed[warp * 8 + 2 * t4] = mx[0]; sRed[warp * 8 + 2 * t4 + 1] = mx[1]; }
    __syncthreads();
    float m[2], lsum[2] = {0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int h = 2 * t4 + e;
        m[e] = fmaxf(fmaxf(sRed[h], sRed[8 + h]), fmaxf(sRed[16 + h], sRed[24 + h]));
        if (warp == 0 && g4 == 0) sMax[h] = m[e];
    }
    // P = exp(scale * (s - m)) as bf16 into sP[head][key]
#pragma unroll
    for (int mi = 0; mi < kMT; ++mi) {
        const int key = (warp + 4 * mi) * 16 + g4;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 2 * t4 + e;
            const float p0 = key < nk ? exp2f((s[mi][e] - m[e]) * scale_log2) : 0.f;
            const float p1 = key + 8 < nk ? exp2f((s[mi][2 + e] - m[e]) * scale_log2) : 0.f;
            lsum[e] += p0 + p1;
            sP[h * BLOCK + key] = __float2bfloat16_rn(p0);
            sP[h * BLOCK + key + 8] = __float2bfloat16_rn(p1);
        }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        lsum[e] += __shfl_xor_sync(0xffffffffu, lsum[e], 4);
        lsum[e] += __shfl_xor_sync(0xffffffffu, lsum[e], 8);
        lsum[e] += __shfl_xor_sync(0xffffffffu, lsum[e], 16);
    }
    __syncthreads();                                       // sP complete; sRed reads done
    if (g4 == 0) { sRed[warp * 8 + 2 * t4] = lsum[0]; sRed[warp * 8 + 2 * t4 + 1] = lsum[1]; }
    // O^T = V^T P: warp w owns channel m-tiles [2 w, 2 w + 2) (D = 128)
    constexpr int kDT = D / 16 / 4;
    float o[kDT][4];
#pragma unroll
    for (int di = 0; di < kDT; ++di) {
        o[di][0] = o[di][1] = o[di][2] = o[di][3] = 0.f;
        const int dt = warp * kDT + di;
#pragma unroll
        for (int ks = 0; ks < BLOCK / 16; ++ks) {
            uint32_t a[4];
            const int key = ks * 16 + (lane & 7) + 8 * (lane >> 4);
            ldmatrix_x4_trans(a, sV + swz(key, 2 * dt + ((lane >> 3) & 1), kRowBytes));
            const __nv_bfloat16 *pp = sP + g4 * BLOCK + ks * 16 + 2 * t4;
            mma_bf16_16816(o[di], a, *(const uint32_t *)pp, *(const uint32_t *)(pp + 8));
        }
    }
    __syncthreads();                                       // sRed (sums) complete
    // normalise and stage O[head][channel] as bf16
#pragma unroll
    for (int di = 0; di < kDT; ++di) {
        const int d0 = (warp * kDT + di) * 16 + g4;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 2 * t4 + e;
            const float l = sRed[h] + sRed[8 + h] + sRed[16 + h] + sRed[24 + h];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            sO[h * D + d0] = __float2bfloat16_rn(o[di][e] * inv);
            sO[h * D + d0 + 8] = __float2bfloat16_rn(o[di][2 + e] * inv);
        }
    }
    __syncthreads();
    // write this CTA's Rh partial rows in the blocked chunk layout
    // (partial_chunk) and their LSE
    const int64_t prow0 = (rg * topk + slot) * R + h0;
    for (int c = tid; c < Rh * kChunks; c += kAttnThreads) {
        const int h = c % Rh, ch = c / Rh;
        if (MSA_IN_BOUNDS(prow0 + h, n_prows))
            ((uint4 *)part_o)[partial_chunk(prow0 + h, ch, D)] = *(const uint4 *)(sO + h * D + ch * 8);
    }
    if (tid < Rh && MSA_IN_BOUNDS(prow0 + tid, n_prows)) {
        const int h = tid;
        const float l = sRed[h] + sRed[8 + h] + sRed[16 + h] + sRed[24 + h];
        part_lse[prow0 + h] = sMax[h] * scale + logf(l);
    }
}

template <int DIDX, int NCG>
cudaError_t launch_index_t(const Shape &s, const void *q_idx, const void *k_idx, float *bs,
                           cudaStream_t st, const KeyRows &rows, const int32_t *lens) {
    constexpr int W = DIDX == 64 ? 8 : 4;
    const size_t smem = (size_t)W * 2 * 64 * DIDX * 2;
    auto k = rows.table ? decode_index_kernel<DIDX, NCG, W, true>
                        : decode_index_kernel<DIDX, NCG, W, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int bpw = 4;                                     // blocks per warp
    const dim3 grid((unsigned)((s.NB + W * bpw - 1) / (W * bpw)), (unsigned)s.B);
    k<<<grid, W * 32, smem, st>>>((const __nv_bfloat16 *)q_idx, (const __nv_bfloat16 *)k_idx, bs,
                                  s.T, s.S, s.G, s.NB, s.block, bpw, rows, lens,
                                  rows.table ? (int64_t)rows.num_pages * rows.page_size
                                             : (int64_t)s.B * s.S);
    count_launches(1);
    return cudaGetLastError();
}

template <int DIDX>
cudaError_t launch_index_d(const Shape &s, const void *q, const void *k, float *bs, cudaStream_t st,
                           const KeyRows &rows, const int32_t *lens) {
    const int ncg = (s.T * s.G + 7) / 8;
    switch (ncg) {
        case 1: return launch_index_t<DIDX, 1>(s, q, k, bs, st, rows, lens);
        case 2: return launch_index_t<DIDX, 2>(s, q, k, bs, st, rows, lens);
        case 3: return launch_index_t<DIDX, 3>(s, q, k, bs, st, rows, lens);
        default: return launch_index_t<DIDX, 4>(s, q, k, bs, st, rows, lens);
    }
}

template <int BLOCK>
cudaError_t launch_block_t(const Shape &s, const void *Q, const void *K, const void *V,
                           const int32_t *ids, __nv_bfloat16 *part_o, float *part_lse, uint32_t *err,
                           cudaStream_t st, const KeyRows &rows, const int32_t *lens) {
    constexpr int D = 128;
    const size_t smem = 2 * (size_t)BLOCK * D * 2 + 8 * BLOCK * 2 + 40 * 4 + 8 * D * 2;
    auto k = rows.table ? decode_block_kernel<D, BLOCK, true> : decode_block_kernel<D, BLOCK, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t ctas = s.index_rows() * s.topk * ((s.R + 7) / 8);
    const float scale_log2 = s.scale * 1.4426950408889634f;
    k<<<(unsigned)ctas, kAttnThreads, smem, st>>>(
        (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K, (const __nv_bfloat16 *)V, ids, part_o,
        part_lse, err, s.T, s.S, s.Hq, s.Hkv, s.R, s.NB, s.topk, scale_log2, s.scale,
        (int64_t)s.index_rows() * s.topk * s.R, rows, lens,
        rows.table ? (int64_t)rows.num_pages * rows.page_size : (int64_t)s.B * s.S);
    count_launches(1);
    return cudaGetLastError();
}

// One warp per sequence of a paged call.
__global__ void paged_check_kernel(const int32_t *__restrict__ lens, KeyRows rows,
                                   int32_t *__restrict__ lens_ok, uint32_t *err, int B, int T_,
                                   int64_t S) {
    const int b = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32);
    const int lane = threadIdx.x % 32;
    if (b >= B) return;
    const int64_t L = lens[b];
    bool ok = L >= T_ && L <= S;
    bool bad_page = false;
    if (ok) {
        const int64_t npages = (L + rows.page_size - 1) / rows.page_size;   // <= max_pages
        for (int64_t i = lane; i < npages; i += 32) {
            const int pg = rows.table[(int64_t)b * rows.max_pages + i];
            bad_page |= pg < 0 || pg >= rows.num_pages;
        }
    }
    ok = ok && !__any_sync(0xffffffffu, bad_page);
    if (lane == 0) {
        lens_ok[b] = ok ? (int32_t)L : 0;
        if (!ok) record_error(err, MSA_ERR_BAD_PAGE_TABLE, 3);
    }
}

size_t part_bytes_o(const Shape &s) {
    const size_t rows = ((size_t)s.index_rows() * s.topk * s.R + 31) / 32 * 32;
    return ((rows * s.d * 2) + 255) / 256 * 256;
}

}  // namespace

cudaError_t launch_paged_check(const Shape &s, const int32_t *lens, const KeyRows &rows,
                               int32_t *lens_ok, uint32_t *err, cudaStream_t st) {
    paged_check_kernel<<<(unsigned)((s.B * 32 + 255) / 256), 256, 0, st>>>(lens, rows, lens_ok,
                                                                          err, s.B, s.T, s.S);
    count_launches(1);
    return cudaGetLastError();
}

bool decode_index_supported(const Shape &s) {
    return s.dtype == MSA_BF16 && (s.d_idx == 64 || s.d_idx == 128) && s.T * s.G <= 32 &&
           (s.block == 64 || s.block == 128);
}

cudaError_t launch_decode_index(const Shape &s, const void *q_idx, const void *k_idx, float *bs,
                                cudaStream_t st, const KeyRows *rows, const int32_t *lens) {
    const KeyRows r = rows ? *rows : dense_rows(s.S);
    if (s.d_idx == 64) return launch_index_d<64>(s, q_idx, k_idx, bs, st, r, lens);
    return launch_index_d<128>(s, q_idx, k_idx, bs, st, r, lens);
}

bool decode_attn_supported(const Shape &s) {
    return s.dtype == MSA_BF16 && s.d == 128 && s.R <= 16 && (s.block == 64 || s.block == 128) &&
           s.index_rows() * s.topk * ((s.R + 7) / 8) < (1ll << 31) && combine_supported(s);
}

size_t decode_attn_workspace(const Shape &s) {
    return part_bytes_o(s) + (((size_t)s.index_rows() * s.topk * s.R * 4) + 255) / 256 * 256;
}

cudaError_t launch_decode_attn(const Shape &s, const void *Q, const void *K, const void *V,
                               const int32_t *ids, void *O, float *lse, uint32_t *err, void *ws,
                               cudaStream_t st, float *mass, const KeyRows *rows,
                               const int32_t *lens) {
    __nv_bfloat16 *part_o = (__nv_bfloat16 *)ws;
    float *part_lse = (float *)((char *)ws + part_bytes_o(s));
    const KeyRows r = rows ? *rows : dense_rows(s.S);
    cudaError_t e = s.block == 64
                        ? launch_block_t<64>(s, Q, K, V, ids, part_o, part_lse, err, st, r, lens)
                        : launch_block_t<128>(s, Q, K, V, ids, part_o, part_lse, err, st, r, lens);
    if (e != cudaSuccess) return e;
    return launch_combine(s, ids, part_o, part_lse, O, lse, 0, s.rows(), st, mass, lens);
}

}  // namespace msa
