// attn_tc.cu -- sparse attention over the kept blocks on the tensor cores
// (bf16 prefill), KV-block-outer.
//
// Main branch ("MiniMax Sparse Attention", Summary, second paragraph: exact
// softmax attention restricted to the kept blocks; Key points, kernel design:
// pre-scheduled chunks, a two-phase combine, and the LSE produced by the
// forward pass).  For query (b, t), head h in group g, over the causal
// tokens j <= p(t) of the kept blocks:
//   O = sum_j softmax(scale * Q.K_j) V_j,   lse = log sum_j exp(scale * Q.K_j).
//
// Each (query, group) keeps its own blocks, so the query heads that share a
// kept block are only the R = Hq/Hkv heads of one token -- too few rows for
// a tensor-core tile.  The work is therefore turned around: for every
// (batch, group, block n) the tokens that kept n are listed (a CSR built on
// the device), and a tile is up to 128/R of those tokens times their R
// heads = 128 rows, against the 128 (or 64) keys of block n:
//   phase 1  S = Q K_n^T (tcgen05, SS), block-local softmax in registers,
//            P (bf16) to TMEM, O_n = P V_n (tcgen05, A from TMEM), written as
//            a normalised bf16 partial plus its LSE, one per (query, head,
//            kept slot);
//   phase 2  per (query, head): LSE-weighted combine of the partials of its
//            kept slots -> O (bf16) and lse (fp32).
// Work is chunked over query rows so the partial buffer stays bounded.
#include <math.h>

#include <algorithm>

#include "tc.cuh"

namespace msa {
namespace {

constexpr int kRows = 128;           // tile rows = tokens_per_tile * R
constexpr int kThreads = 512;        // four warpgroups: loads + MMA, two softmax, epilogue
constexpr int kRun = 8;              // consecutive tiles per CTA turn (K/V reuse)
constexpr float kLog2e = 1.4426950408889634f;

// Validity of the kept slots lane and lane + 32 of a row (topk <= 64; the
// hot merge path, which keeps these few values in registers), computed by
// one warp: in range, holding a causal token, and not a repeat
// (a strictly ascending row, the form msa_topk_blocks writes, cannot repeat;
// otherwise earlier slots are scanned).  bad = an id >= NB, an id above cb
// (a block with no causal token) or a repeat; bad slots are skipped and
// counted in the error word.
struct SlotPair {
    int id0, id1;
    bool ok0, ok1, bad0, bad1;
};
__device__ __forceinline__ SlotPair warp_slots2(const int32_t *row, int topk, int NB, int cb,
                                               int lane) {
    SlotPair r;
    r.id0 = lane < topk ? row[lane] : -1;
    r.id1 = lane + 32 < topk ? row[lane + 32] : -1;
    int pm0 = r.id0;
    for (int off = 1; off < 32; off *= 2) {
        const int o = __shfl_up_sync(0xffffffffu, pm0, off);
        if (lane >= off) pm0 = max(pm0, o);
    }
    const int before0 = __shfl_up_sync(0xffffffffu, pm0, 1);
    const int max_first = __shfl_sync(0xffffffffu, pm0, 31);
    int pm1 = r.id1;
    for (int off = 1; off < 32; off *= 2) {
        const int o = __shfl_up_sync(0xffffffffu, pm1, off);
        if (lane >= off) pm1 = max(pm1, o);
    }
    const int before1 = max(max_first, __shfl_up_sync(0xffffffffu, pm1, 1));
    const bool dis0 = r.id0 >= 0 && lane > 0 && r.id0 <= before0;
    const bool dis1 = r.id1 >= 0 && (lane > 0 ? r.id1 <= before1 : r.id1 <= max_first);
    const bool asc = !__any_sync(0xffffffffu, dis0 || dis1);
    bool rep0 = false, rep1 = false;
    if (!asc) {
        for (int q = 0; q < lane && r.id0 >= 0; ++q) rep0 |= row[q] == r.id0;
        for (int q = 0; q < lane + 32 && r.id1 >= 0; ++q) rep1 |= row[q] == r.id1;
    }
    r.bad0 = r.id0 >= NB || r.id0 > cb || (r.id0 >= 0 && rep0);
    r.bad1 = r.id1 >= NB || r.id1 > cb || (r.id1 >= 0 && rep1);
    r.ok0 = r.id0 >= 0 && !r.bad0;
    r.ok1 = r.id1 >= 0 && !r.bad1;
    return r;
}

// The same for the kept slots lane + 32 k (k < kPer, topk <= 32 kPer) of a
// row, computed by one warp: in range, holding a causal token, and not a
// repeat (a strictly ascending row, the form msa_topk_blocks writes, cannot
// repeat; otherwise earlier slots are scanned).  bad = an id >= NB, an id
// above cb (a block with no causal token) or a repeat; bad slots are skipped
// and counted in the error word.  okmask[k] bit l: slot 32 k + l is valid.
template <int kPer>
struct SlotSet {
    int id[kPer];
    bool ok[kPer], bad[kPer];
    uint32_t okmask[kPer];
    __device__ __forceinline__ bool valid(int sl) const {      // slot sl of the row
        uint32_t m = 0;
#pragma unroll
        for (int k = 0; k < kPer; ++k)
            if (k == (sl >> 5)) m = okmask[k];
        return (m >> (sl & 31)) & 1u;
    }
};
template <int kPer>
__device__ __forceinline__ SlotSet<kPer> warp_slots(const int32_t *row, int topk, int NB, int cb,
                                                    int lane) {
    SlotSet<kPer> r;
    int carry = -1;                               // largest id of the earlier 32-slot groups
    bool dis = false;                             // some slot not above every earlier one
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int id = 32 * k + lane < topk ? row[32 * k + lane] : -1;
        r.id[k] = id;
        int pm = id;                              // inclusive prefix max over the lanes
        for (int off = 1; off < 32; off *= 2) {
            const int o = __shfl_up_sync(0xffffffffu, pm, off);
            if (lane >= off) pm = max(pm, o);
        }
        const int up = __shfl_up_sync(0xffffffffu, pm, 1);
        const int before = lane > 0 ? max(carry, up) : carry;
        dis |= id >= 0 && (32 * k + lane > 0) && id <= before;
        carry = max(carry, __shfl_sync(0xffffffffu, pm, 31));
    }
    const bool asc = !__any_sync(0xffffffffu, dis);
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int id = r.id[k];
        bool rep = false;
        if (!asc)
            for (int q = 0; q < 32 * k + lane && id >= 0; ++q) rep |= row[q] == id;
        r.bad[k] = id >= NB || id > cb || (id >= 0 && rep);
        r.ok[k] = id >= 0 && !r.bad[k];
        r.okmask[k] = __ballot_sync(0xffffffffu, r.ok[k]);
    }
    return r;
}

// ---------------------------------------------------------------- CSR build

// counts[(b*G + g)*NB + n] += 1 for every valid kept slot of the chunk's rows;
// one warp per (row, group), one lane per slot.
template <int kPer>
__global__ void csr_count_kernel(const int32_t *__restrict__ ids, int *__restrict__ counts,
                                 uint32_t *err, int64_t r0, int64_t rc, int T_, int S, int G,
                                 int NB, int block, int topk) {
    const int64_t x = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (x >= rc * G) return;
    const int64_t r = r0 + x / G;                 // b * T + t
    const int g = (int)(x % G);
    const int b = (int)(r / T_), t = (int)(r % T_);
    const int cb = (int)(((int64_t)S - T_ + t) / block);
    const SlotSet<kPer> sp = warp_slots<kPer>(ids + (r * G + g) * topk, topk, NB, cb, lane);
    int *base = counts + ((int64_t)b * G + g) * NB;
    bool bad = false;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        if (sp.ok[k]) atomicAdd(base + sp.id[k], 1);
        bad |= sp.bad[k];
    }
    if (bad) record_error(err, MSA_ERR_BAD_BLOCK_IDS, 1);
}

// Single-CTA exclusive scan: tile_offs = scan(ceil(counts / tpt)); tile_offs[L]
// holds the number of tiles.
__global__ void csr_scan_kernel(const int *__restrict__ counts, int *__restrict__ tile_offs, int L,
                                int tpt) {
    __shared__ int s_b[1024];
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (L + nt - 1) / nt;
    const int lo = min(L, tid * per), hi = min(L, lo + per);
    int b = 0;
    for (int i = lo; i < hi; ++i) b += (counts[i] + tpt - 1) / tpt;
    s_b[tid] = b;
    __syncthreads();
    for (int off = 1; off < nt; off *= 2) {       // inclusive Hillis-Steele scan
        const int vb = tid >= off ? s_b[tid - off] : 0;
        __syncthreads();
        s_b[tid] += vb;
        __syncthreads();
    }
    int eb = s_b[tid] - b;                         // exclusive
    for (int i = lo; i < hi; ++i) {
        tile_offs[i] = eb;
        eb += (counts[i] + tpt - 1) / tpt;
    }
    if (tid == nt - 1) tile_offs[L] = s_b[nt - 1];
}

// Tile records: record k of a chunk is rec_ints(tpt) ints, {list, tokens in
// the tile, 0, 0, entry[0 .. tpt)} with entry = (row - r0) << 8 | slot, so a
// tile's description is one contiguous read with no dependent load.
__host__ __device__ constexpr int rec_ints(int tpt) { return 4 + tpt; }

// Every valid kept slot of the chunk's rows into its list's next free record
// entry; one warp per (row, group), one lane per slot.
template <int kPer>
__global__ void csr_fill_kernel(const int32_t *__restrict__ ids,
                                const int *__restrict__ tile_offs, int *__restrict__ cursor,
                                int *__restrict__ recs, int64_t r0, int64_t rc, int T_, int S,
                                int G, int NB, int block, int topk, int tpt, int64_t rec_cap) {
    const int64_t x = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (x >= rc * G) return;
    const int64_t r = r0 + x / G;
    const int g = (int)(x % G);
    const int b = (int)(r / T_), t = (int)(r % T_);
    const int cb = (int)(((int64_t)S - T_ + t) / block);
    const SlotSet<kPer> sp = warp_slots<kPer>(ids + (r * G + g) * topk, topk, NB, cb, lane);
    const int64_t lbase = ((int64_t)b * G + g) * NB;
    const int tag = (int)((r - r0) << 8);
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        if (sp.ok[k]) {
            const int64_t list = lbase + sp.id[k];
            const int pos = atomicAdd(&cursor[list], 1);
            const int64_t at = (int64_t)(tile_offs[list] + pos / tpt) * rec_ints(tpt) + 4 + pos % tpt;
            if (MSA_IN_BOUNDS(at, rec_cap)) recs[at] = tag | (32 * k + lane);
        }
    }
}

// Record headers {list, tokens in the tile, 0, 0} for every tile of every list.
__global__ void csr_tiles_kernel(const int *__restrict__ counts, const int *__restrict__ tile_offs,
                                 int *__restrict__ recs, int L, int tpt) {
    const int list = blockIdx.x * blockDim.x + threadIdx.x;
    if (list >= L) return;
    const int cnt = counts[list];
    const int nt = (cnt + tpt - 1) / tpt;
    const int base = tile_offs[list];
    for (int c = 0; c < nt; ++c)
        *(int4 *)(recs + (int64_t)(base + c) * rec_ints(tpt)) =
            make_int4(list, min(tpt, cnt - c * tpt), 0, 0);
}

}  // namespace
}  // namespace msa

namespace msa {
namespace {

// Phase 2: the LSE-weighted merge of a (query row, group)'s partials over
// its valid kept slots, for each of the group's R heads: weights
// exp(lse_i - max lse) give the softmax over the union of the slots' keys.
// Four warps share a (row, group), each merging a quarter of the d/8 16-byte
// channel chunks.  Lane l owns head l % R and slots l / R, l / R + 32 / R, ...;
// with the blocked chunk layout every load of the warp is 512 contiguous
// bytes, and all loads of a warp are independent (issued together).
// Needs R | 32 and kPer >= topk / 32; lanes take their slots in batches of
// kMaxPer.  Run by combine_kernel after each row chunk's attention kernel.
struct CombineArgs {
    const int32_t *ids;
    const __nv_bfloat16 *part_o;
    const float *part_lse;
    __nv_bfloat16 *O;
    float *lse;
    int64_t r0, rc;                               // the chunk's query rows
    int T_, S, Hq, G, R, NB, block, topk;
    const int32_t *lens;
};

constexpr int kCombineChunksPerWarp = 4;          // 16-byte channel chunks per warp
// Warps that merge one (row, group).
template <int D> constexpr int combine_warps_per_row() { return D / 8 / kCombineChunksPerWarp; }

// The merge of one (row, group) quarter: warp unit `wid` of the chunk
// (wid < rc * G * combine_warps_per_row<D>()).  kMaxPer: slots per lane,
// >= topk * R / 32.
template <int D, int kMaxPer>
__device__ __forceinline__ void combine_unit(const CombineArgs &c, int64_t wid, int lane) {
    constexpr int kChunksPerWarp = kCombineChunksPerWarp;
    constexpr int kWarpsPerRow = combine_warps_per_row<D>();
    const int32_t *__restrict__ ids = c.ids;
    const __nv_bfloat16 *__restrict__ part_o = c.part_o;
    const float *__restrict__ part_lse = c.part_lse;
    __nv_bfloat16 *__restrict__ O = c.O;
    float *__restrict__ lse = c.lse;
    const int64_t r0 = c.r0;
    const int T_ = c.T_, S = c.S, Hq = c.Hq, G = c.G, R = c.R, NB = c.NB, block = c.block;
    const int topk = c.topk;
    const int32_t *__restrict__ lens = c.lens;
    const int part = (int)(wid % kWarpsPerRow);
    const int64_t rgl = wid / kWarpsPerRow;
    const int64_t rl = rgl / G;                   // row within the chunk
    const int g = (int)(rgl % G);
    const int64_t r = r0 + rl;
    const int t = (int)(r % T_);
    const int64_t p = seq_len(lens, (int)(r / T_), S) - T_ + t;
    const int cb = p < 0 ? -1 : (int)(p / block);
    const SlotPair sp = warp_slots2(ids + (r * G + g) * topk, topk, NB, cb, lane);
    const int h = lane % R, s0 = lane / R, sstep = 32 / R;
    const int per = (topk + sstep - 1) / sstep;
    const int64_t base = (rl * G + g) * topk * R;
    float li[kMaxPer], m = -INFINITY;
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        const int sl = s0 + k * sstep;
        const bool okk = __shfl_sync(0xffffffffu, sl < 32 ? sp.ok0 : sp.ok1, sl & 31);
        const bool ok = k < per && sl < topk && okk;
        li[k] = ok ? part_lse[base + (int64_t)sl * R + h] : -INFINITY;
        m = fmaxf(m, li[k]);
    }
    for (int off = R; off < 32; off *= 2) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float w[kMaxPer], lsum = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        w[k] = li[k] == -INFINITY ? 0.f : expf(li[k] - m);
        lsum += w[k];
    }
    for (int off = R; off < 32; off *= 2) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    const uint4 *src = (const uint4 *)part_o;
    __nv_bfloat16 *dst = O + (r * Hq + (int64_t)g * R + h) * D;
    float acc[kChunksPerWarp][8];
#pragma unroll
    for (int c = 0; c < kChunksPerWarp; ++c)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[c][q] = 0.f;
    // k < per is uniform across the warp, so the loads are issued together;
    // a slot that holds no partial (weight 0) issues no load and adds 0
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        if (k < per) {
            const int64_t prow = base + (int64_t)(s0 + k * sstep) * R + h;
            const bool use = w[k] > 0.f && MSA_IN_BOUNDS(prow, c.rc * G * topk * R);
#pragma unroll
            for (int c = 0; c < kChunksPerWarp; ++c) {
                uint4 u = make_uint4(0u, 0u, 0u, 0u);
                if (use) u = src[partial_chunk(prow, part * kChunksPerWarp + c, D)];
                const __nv_bfloat162 *hp = (const __nv_bfloat162 *)&u;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __bfloat1622float2(hp[q]);
                    acc[c][2 * q] = fmaf(w[k], f.x, acc[c][2 * q]);
                    acc[c][2 * q + 1] = fmaf(w[k], f.y, acc[c][2 * q + 1]);
                }
            }
        }
    }
#pragma unroll
    for (int c = 0; c < kChunksPerWarp; ++c) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
            for (int off = R; off < 32; off *= 2)
                acc[c][q] += __shfl_xor_sync(0xffffffffu, acc[c][q], off);
        if (s0 == 0) {
            __nv_bfloat162 o2[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                o2[q] = __floats2bfloat162_rn(acc[c][2 * q] * inv, acc[c][2 * q + 1] * inv);
            *(uint4 *)(dst + (part * kChunksPerWarp + c) * 8) = *(const uint4 *)o2;
        }
    }
    if (part == 0 && s0 == 0) lse[r * Hq + (int64_t)g * R + h] = lsum > 0.f ? m + logf(lsum) : -INFINITY;
}

// The merge for rows of more than 64 kept blocks: slots taken in batches of
// kMaxPer per lane; pass 1 finds the maximum LSE, pass 2 weighs and adds.
template <int D, int kMaxPer, int kPer>
__device__ __forceinline__ void combine_unit_batched(const CombineArgs &c, int64_t wid, int lane) {
    constexpr int kChunksPerWarp = kCombineChunksPerWarp;
    constexpr int kWarpsPerRow = combine_warps_per_row<D>();
    const int32_t *__restrict__ ids = c.ids;
    const __nv_bfloat16 *__restrict__ part_o = c.part_o;
    const float *__restrict__ part_lse = c.part_lse;
    __nv_bfloat16 *__restrict__ O = c.O;
    float *__restrict__ lse = c.lse;
    const int64_t r0 = c.r0;
    const int T_ = c.T_, S = c.S, Hq = c.Hq, G = c.G, R = c.R, NB = c.NB, block = c.block;
    const int topk = c.topk;
    const int32_t *__restrict__ lens = c.lens;
    const int part = (int)(wid % kWarpsPerRow);
    const int64_t rgl = wid / kWarpsPerRow;
    const int64_t rl = rgl / G;                   // row within the chunk
    const int g = (int)(rgl % G);
    const int64_t r = r0 + rl;
    const int t = (int)(r % T_);
    const int64_t p = seq_len(lens, (int)(r / T_), S) - T_ + t;
    const int cb = p < 0 ? -1 : (int)(p / block);
    const SlotSet<kPer> sp = warp_slots<kPer>(ids + (r * G + g) * topk, topk, NB, cb, lane);
    const int h = lane % R, s0 = lane / R, sstep = 32 / R;
    const int per = (topk + sstep - 1) / sstep;   // slots per lane (uniform across the warp)
    const int64_t base = (rl * G + g) * topk * R;
    float li0[kMaxPer], m = -INFINITY;            // the first batch's LSEs stay in registers
    for (int k0 = 0; k0 < per; k0 += kMaxPer) {
#pragma unroll
        for (int k = 0; k < kMaxPer; ++k) {
            const int sl = s0 + (k0 + k) * sstep;
            const bool ok = k0 + k < per && sl < topk && sp.valid(sl);
            const float l = ok ? part_lse[base + (int64_t)sl * R + h] : -INFINITY;
            if (k0 == 0) li0[k] = l;
            m = fmaxf(m, l);
        }
    }
    for (int off = R; off < 32; off *= 2) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const uint4 *src = (const uint4 *)part_o;
    __nv_bfloat16 *dst = O + (r * Hq + (int64_t)g * R + h) * D;
    float acc[kChunksPerWarp][8];
#pragma unroll
    for (int c = 0; c < kChunksPerWarp; ++c)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[c][q] = 0.f;
    float lsum = 0.f;
    for (int k0 = 0; k0 < per; k0 += kMaxPer) {
        float w[kMaxPer];
#pragma unroll
        for (int k = 0; k < kMaxPer; ++k) {
            float l = li0[k];
            if (k0 > 0) {
                const int sl = s0 + (k0 + k) * sstep;
                const bool ok = k0 + k < per && sl < topk && sp.valid(sl);
                l = ok ? part_lse[base + (int64_t)sl * R + h] : -INFINITY;
            }
            w[k] = l == -INFINITY ? 0.f : expf(l - m);
            lsum += w[k];
        }
        // k0 + k < per is uniform across the warp, so the loads are issued
        // together; a slot that holds no partial (weight 0) issues no load
#pragma unroll
        for (int k = 0; k < kMaxPer; ++k) {
            if (k0 + k < per) {
                const int64_t prow = base + (int64_t)(s0 + (k0 + k) * sstep) * R + h;
                const bool use = w[k] > 0.f && MSA_IN_BOUNDS(prow, c.rc * G * topk * R);
#pragma unroll
                for (int c = 0; c < kChunksPerWarp; ++c) {
                    uint4 u = make_uint4(0u, 0u, 0u, 0u);
                    if (use) u = src[partial_chunk(prow, part * kChunksPerWarp + c, D)];
                    const __nv_bfloat162 *hp = (const __nv_bfloat162 *)&u;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = __bfloat1622float2(hp[q]);
                        acc[c][2 * q] = fmaf(w[k], f.x, acc[c][2 * q]);
                        acc[c][2 * q + 1] = fmaf(w[k], f.y, acc[c][2 * q + 1]);
                    }
                }
            }
        }
    }
    for (int off = R; off < 32; off *= 2) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
    for (int c = 0; c < kChunksPerWarp; ++c) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
            for (int off = R; off < 32; off *= 2)
                acc[c][q] += __shfl_xor_sync(0xffffffffu, acc[c][q], off);
        if (s0 == 0) {
            __nv_bfloat162 o2[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                o2[q] = __floats2bfloat162_rn(acc[c][2 * q] * inv, acc[c][2 * q + 1] * inv);
            *(uint4 *)(dst + (part * kChunksPerWarp + c) * 8) = *(const uint4 *)o2;
        }
    }
    if (part == 0 && s0 == 0) lse[r * Hq + (int64_t)g * R + h] = lsum > 0.f ? m + logf(lsum) : -INFINITY;
}

// kPer == 0: rows of at most 64 kept blocks and at most kMaxPer slots per
// lane, one batch; otherwise batches of kMaxPer over up to 32 kPer kept blocks.
template <int D, int kMaxPer, int kPer>
__global__ void __launch_bounds__(256, kMaxPer <= 8 ? 3 : 2)
combine_kernel(CombineArgs c) {
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    if (wid >= c.rc * c.G * combine_warps_per_row<D>()) return;
    if (kPer == 0) combine_unit<D, kMaxPer>(c, wid, threadIdx.x % 32);
    else combine_unit_batched<D, kMaxPer, (kPer > 0 ? kPer : 1)>(c, wid, threadIdx.x % 32);
}

// The merge in two passes, for R * d >= 256 (a warp's 32 lanes then cover
// whole heads): pass 1 turns each (row, group)'s slot LSEs into normalised
// weights w = exp(lse_i - lse) (0 for a slot no tile served), written over
// the LSEs, and writes the row's final LSE; pass 2 streams the partials with
// lanes = (head, 16-byte channel chunk), each lane summing w * O_i over the
// slots for its own 8 output channels (no cross-lane reduction, no per-warp
// LSE work).  Lanes of pass 1 are laid out as in the single-pass merge (head
// l % R, slots l / R + k * 32 / R); kMaxPer (8 or 16) >= slots per lane.
template <int kMaxPer>
__global__ void __launch_bounds__(256) merge_weights_kernel(CombineArgs c, float *wts) {
    const int64_t x = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (x >= c.rc * c.G) return;
    const int64_t rl = x / c.G, r = c.r0 + rl;
    const int g = (int)(x % c.G);
    const int t = (int)(r % c.T_);
    const int64_t p = seq_len(c.lens, (int)(r / c.T_), c.S) - c.T_ + t;
    const int cb = p < 0 ? -1 : (int)(p / c.block);
    const SlotPair sp = warp_slots2(c.ids + (r * c.G + g) * c.topk, c.topk, c.NB, cb, lane);
    const int R = c.R, h = lane % R, s0 = lane / R, sstep = 32 / R;
    const int per = (c.topk + sstep - 1) / sstep;        // slots per lane
    const int64_t base = x * c.topk * R;
    float li[kMaxPer], m = -INFINITY;                    // every load issued before any use
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        const int sl = s0 + k * sstep;
        const bool okk = __shfl_sync(0xffffffffu, sl < 32 ? sp.ok0 : sp.ok1, sl & 31);
        const bool ok = k < per && sl < c.topk && okk;
        li[k] = ok ? c.part_lse[base + (int64_t)sl * R + h] : -INFINITY;
        m = fmaxf(m, li[k]);
    }
    for (int off = R; off < 32; off *= 2) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float lsum = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        li[k] = li[k] == -INFINITY ? 0.f : expf(li[k] - m);
        lsum += li[k];
    }
    for (int off = R; off < 32; off *= 2) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        const int sl = s0 + k * sstep;
        if (k < per && sl < c.topk) wts[base + (int64_t)sl * R + h] = li[k] * inv;
    }
    if (s0 == 0) c.lse[r * c.Hq + (int64_t)g * R + h] = lsum > 0.f ? m + logf(lsum) : -INFINITY;
}

template <int D, int R>
__global__ void __launch_bounds__(256) merge_apply_kernel(CombineArgs c, const float *wts) {
    constexpr int C = 32 / R;                            // chunks per head in one warp
    constexpr int W = D / 8 / C;                         // warps per (row, group)
    static_assert(W >= 1, "the group's heads must fill a warp");
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (wid >= c.rc * c.G * W) return;
    const int part = (int)(wid % W);
    const int64_t x = wid / W;                           // (row in chunk, group)
    const int64_t rl = x / c.G;
    const int g = (int)(x % c.G);
    const int h = lane / C, ch = part * C + lane % C;    // head, 16-byte channel chunk
    const int64_t base = x * c.topk * R;
    const uint4 *src = (const uint4 *)c.part_o;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int s0 = 0; s0 < c.topk; s0 += 8) {
        // a batch's weights, then its loads (a zero weight: no partial, no load)
        float w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            w[k] = s0 + k < c.topk ? __ldg(wts + base + (int64_t)(s0 + k) * R + h) : 0.f;
        uint4 u[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int64_t prow = base + (int64_t)(s0 + k) * R + h;
            u[k] = make_uint4(0u, 0u, 0u, 0u);
            if (w[k] != 0.f && MSA_IN_BOUNDS(prow, c.rc * c.G * c.topk * R))
                u[k] = src[partial_chunk(prow, ch, D)];
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const __nv_bfloat162 *hp = (const __nv_bfloat162 *)&u[k];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __bfloat1622float2(hp[q]);
                acc[2 * q] = fmaf(w[k], f.x, acc[2 * q]);
                acc[2 * q + 1] = fmaf(w[k], f.y, acc[2 * q + 1]);
            }
        }
    }
    const int64_t r = c.r0 + rl;
    __nv_bfloat162 o2[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) o2[q] = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
    *(uint4 *)(c.O + (r * c.Hq + (int64_t)g * R + h) * D + ch * 8) = *(const uint4 *)o2;
}

struct AttnArgs {
    const __nv_bfloat16 *Q;     // [B, T, Hq, D]
    const int *recs;            // tile records (rec_ints(tpt) ints each)
    const int *n_tiles;         // device-side tile count
    __nv_bfloat16 *part_o;      // normalised partial O, blocked chunks (partial_chunk)
    float *part_lse;            // [n_prows]
    int64_t n_prows;            // rc * G * topk * R
    int64_t q_rows;             // B * T (rows of Q)
    uint32_t *err;
    int64_t r0;
    int T, S, Hq, G, R, NB, topk, tpt;
    int q_box4;                 // Q tensor map is 4-D: one box = both channel atoms
    float scale, scale_log2;
};

// The CTA's i-th tile: runs of kRun consecutive tiles dealt round-robin
// over the CTAs.
__device__ __forceinline__ int run_tile(const AttnArgs &, int i) {
    return (i / kRun) * (gridDim.x * kRun) + blockIdx.x * kRun + (i % kRun);
}

// Header {list, count} of a CTA's i-th tile ({-1, 0} past the end) and entry
// k (< tpt) of its record (0 past the end); independent loads.
__device__ __forceinline__ int2 load_head(const AttnArgs &a, int i, int total) {
    const int tile = run_tile(a, i);
    return tile < total ? __ldg((const int2 *)(a.recs + (int64_t)tile * rec_ints(a.tpt)))
                        : make_int2(-1, 0);
}
__device__ __forceinline__ int load_ent(const AttnArgs &a, int i, int total, int k) {
    const int tile = run_tile(a, i);
    return tile < total && k < a.tpt ? __ldg(a.recs + (int64_t)tile * rec_ints(a.tpt) + 4 + k) : 0;
}

// Warp roles (four warpgroups, 512 threads):
//   warpgroup 0     warp 0 loads the K/V blocks, warps 0 and 3 the Q rows
//                   (TMA boxes, half the tokens each; for fewer than 8 heads
//                   per token, a cp.async gather), warp 1 issues the S
//                   products, warp 2 the PV products;
//   warpgroups 1-2  softmax, tiles 0, 2, 4, ... and 1, 3, 5, ...;
//   warpgroup 3     epilogue of every tile: O from TMEM to a bf16 partial.
// TMEM: three S/P buffers (S: BLOCK fp32 columns; P: bf16 pairs in the first
// BLOCK/2 of them; partial row, row max m and row sum l in the last three) at
// columns 0, 128, 256 and one O accumulator at 384.  The epilogue divides O
// by l, converts and stores it with the LSE, so no global store is issued by
// the softmax warps; an S/P buffer is free again once PV has read P and the
// epilogue has read m and l.
constexpr int kRegsLoad = 88, kRegsSoftmax = 136, kRegsEpilogue = 152;
static_assert(kRegsLoad + 2 * kRegsSoftmax + kRegsEpilogue <= 4 * (65536 / kThreads),
              "warpgroup register budgets exceed the launch's registers");

template <int D, int BLOCK>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, AttnArgs a) {
    constexpr int kAtoms = D / 64;
    constexpr int kQBuf = 3;                      // Q tiles in flight = S/P buffers
    constexpr uint32_t kQBytes = kRows * D * 2;
    constexpr uint32_t kKBytes = BLOCK * D * 2;
    // A Q tile is 16 groups of 8 rows; a group holds its kAtoms 64-channel
    // swizzle atoms (8 rows x 128 bytes each) back to back, so 8 heads of a
    // token are one contiguous 2-KB TMA box.
    constexpr uint32_t kGroupBytes = 8 * D * 2;
    constexpr uint32_t kSCols = 128, kOCol = 384;
    static_assert(BLOCK <= (int)kSCols && D <= 128, "TMEM budget");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = smem;                           // [3][16 row groups][kAtoms][8][64]
    uint8_t *sK = sQ + kQBuf * kQBytes;           // [2][kAtoms][BLOCK][64]
    uint8_t *sV = sK + 2 * kKBytes;               // [2][kAtoms][BLOCK][64]
    uint64_t *bar = (uint64_t *)(sV + 2 * kKBytes);
    // A Q buffer is free again when the S product that read it completes
    // (s_full); an S/P buffer when the epilogue has read m and l, after PV.
    uint64_t *q_full = bar;                       // [3]
    uint64_t *kv_full = bar + 3, *kv_empty = bar + 5;        // [2] each
    uint64_t *s_full = bar + 7, *p_full = bar + 10, *s_free = bar + 13;   // [3] each
    uint64_t *o_full = bar + 16, *o_empty = bar + 17;
    uint32_t *tmem_slot = (uint32_t *)(bar + 18);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kQBuf; ++i) {
            tc::mbar_init(&q_full[i], a.R >= 8 ? 2 : 64);   // TMA: one per warp; cp.async: per thread
            tc::mbar_init(&s_full[i], 1);
            tc::mbar_init(&p_full[i], 128);
            tc::mbar_init(&s_free[i], 128);        // epilogue threads, after PV
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&kv_full[i], 1);
            tc::mbar_init(&kv_empty[i], 1);
        }
        tc::mbar_init(o_full, 1);
        tc::mbar_init(o_empty, 128);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = *a.n_tiles;
    const int wg = warp / 4;

    // Each role sets its warpgroup's register budget first.
    if (wg == 0) {
        tc::regs_dec<kRegsLoad>();
        if (warp == 0 || warp == 3) {
            // ------------------------------------------------ loads
            // K/V blocks by TMA (warp 0, lane 0) whenever the list changes, and
            // the tile's Q rows by warps 0 and 3: TMA boxes for 8 or more heads
            // per token, else 16-byte cp.async copies straight into the
            // 128-byte-swizzled K-major
            // layout the MMA reads.  Each warp instruction copies kRPI whole
            // rows of D / 8 16-byte chunks (two rows for D = 128, four for
            // D = 64); lane l always copies chunk l % (D / 8).  A
            // thread's copies arrive on q_full when they complete
            // (cp.async.mbarrier.arrive.noinc), so no warp waits for its own
            // copies and loads run up to three tiles ahead.
            constexpr int kCPR = D / 8, kRPI = 32 / kCPR;   // chunks per row, rows per instruction
            const int gw = warp == 0 ? 0 : 1;          // gather warp 0..1
            const int cc = lane % kCPR;
            const uint32_t q_swz = (uint32_t)(cc / 8) * 1024;
            const int lr = __ffs(a.R) - 1;             // log2 R
            // A token's Q rows are read once per kept block: keep them in L2
            // ahead of the partials streaming out.
            const uint64_t q_pol = tc::policy_evict_last();
            int kvb = -1, cur_list = -1;
            uint32_t kv_ph = 0;                        // per K/V buffer phase bits
            // Records of the next two tiles in flight: lane l holds entries
            // l, l + 32, l + 64, l + 96 of a record.
            int2 h1 = load_head(a, 0, total), h2 = load_head(a, 1, total);
            int e1[4], e2[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                e1[k] = load_ent(a, 0, total, lane + 32 * k);
                e2[k] = load_ent(a, 1, total, lane + 32 * k);
            }
            for (int i = 0;; ++i) {
                const int2 d = h1;
                int e[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) e[k] = e1[k];
                if (d.x < 0) break;
                h1 = h2;
                h2 = load_head(a, i + 2, total);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    e1[k] = e2[k];
                    e2[k] = load_ent(a, i + 2, total, lane + 32 * k);
                }
                const int list = d.x, count = d.y;
                const int n = list % a.NB, g = (list / a.NB) % a.G, b = list / (a.NB * a.G);
                if (list != cur_list) {
                    kvb = (kvb + 1) & 1;
                    cur_list = list;
                    if (warp == 0 && lane == 0 &&
                        tc::mbar_wait(&kv_empty[kvb], ((kv_ph >> kvb) & 1) ^ 1, a.err, abort_flag)) {
                        tc::mbar_expect_tx(&kv_full[kvb], 2 * kKBytes);
                        const int key0 = b * a.S + n * BLOCK;
#pragma unroll
                        for (int at = 0; at < kAtoms; ++at) {
                            tc::tma_load_3d(sK + kvb * kKBytes + at * BLOCK * 128, &tm_k,
                                            &kv_full[kvb], at * 64, g, key0);
                            tc::tma_load_3d(sV + kvb * kKBytes + at * BLOCK * 128, &tm_v,
                                            &kv_full[kvb], at * 64, g, key0);
                        }
                    }
                    kv_ph ^= 1u << kvb;
                }
                const int qb = i % kQBuf;
                if (!tc::mbar_wait(&s_full[qb], ((i / kQBuf) & 1) ^ 1, a.err, abort_flag)) break;
                if (a.R >= 8) {
                    // 8 or more heads per token: the token's heads in groups of 8
                    // rows, one TMA box per group holding both 64-channel atoms
                    // (or one box per atom).  Warps 0 and 3 take the first and
                    // the second half of the tile's tokens: one thread issues a
                    // box every ~100 cycles, so two issuing warps halve the
                    // time a tile's Q takes to leave.  Lane k holds token k's
                    // entry; a shuffle hands each lane its token's.
                    const int half = (count + 1) / 2;
                    const int t0 = warp == 0 ? 0 : half, nt = warp == 0 ? half : count - half;
                    const int ent_t = __shfl_sync(0xffffffffu, e[0], min(t0 + lane, 31));
                    if (lane == 0)
                        tc::mbar_expect_tx(&q_full[qb], (uint32_t)nt * a.R * D * 2);
                    __syncwarp();
                    if (lane < nt) {
                        const int grow = (int)(a.r0 + (ent_t >> 8));
                        for (int j = 0; j < a.R / 8; ++j) {
                            uint8_t *grp8 =
                                sQ + qb * kQBytes + ((t0 + lane) * (a.R / 8) + j) * kGroupBytes;
                            if (a.q_box4) {
                                tc::tma_load_4d_hint(grp8, &tm_q, &q_full[qb], 0, g * a.R + j * 8, 0,
                                                     grow, q_pol);
                            } else {
#pragma unroll
                                for (int at = 0; at < kAtoms; ++at)
                                    tc::tma_load_3d_hint(grp8 + at * 1024, &tm_q, &q_full[qb],
                                                         at * 64, g * a.R + j * 8, grow, q_pol);
                            }
                        }
                    }
                    continue;
                }
                const uint32_t dst = tc::smem_u32(sQ + qb * kQBytes) + q_swz;
                const int rows = count << lr;
                const int64_t head0 = (int64_t)g * a.R;
                // row group q = rows kRPI q .. kRPI q + kRPI - 1 (lane / kCPR);
                // their tokens sit in the same 32-token block, so one register
                // holds their entries and a shuffle hands each lane its token's
                // entry
                for (int q = gw; kRPI * q < rows; q += 2) {
                    const int r = kRPI * q + lane / kCPR;
                    const int tk = r >> lr, hh = r & (a.R - 1);
                    const int kk = (kRPI * q) >> (lr + 5);
                    const int ev = kk == 0 ? e[0] : kk == 1 ? e[1] : kk == 2 ? e[2] : e[3];
                    const int ent = __shfl_sync(0xffffffffu, ev, tk & 31);
                    if (r < rows && MSA_IN_BOUNDS(a.r0 + (ent >> 8), a.q_rows)) {
                        const __nv_bfloat16 *src =
                            a.Q + ((a.r0 + (ent >> 8)) * a.Hq + head0 + hh) * D + cc * 8;
                        const uint32_t sa = dst + (r / 8) * kGroupBytes + (r % 8) * 128 +
                                            (((cc % 8) ^ (r % 8)) * 16);
                        asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;"
                                     ::"r"(sa), "l"(src), "l"(q_pol)
                                     : "memory");
                    }
                }
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];"
                             ::"r"(tc::smem_u32(&q_full[qb])) : "memory");
            }
            // the last copies must land before the CTA can retire
            asm volatile("cp.async.wait_all;" ::: "memory");
        } else if (warp == 1 && lane == 0) {
            // ------------------------------------------------ S issuer: S(t) = Q K^T
            // into S/P buffer t % 3, once Q(t) has landed, the buffer is free
            // (the epilogue has read tile t - 3's row sums, after its PV) and,
            // at a list change, the list's K/V block has landed.
            constexpr uint32_t idesc_s = tc::idesc_bf16(kRows, BLOCK, 0, 0);
            int kvb = -1, cur_list = -1;
            uint32_t kv_ph = 0;
            int next_list = load_head(a, 0, total).x, next_list2 = load_head(a, 1, total).x;
            for (int t = 0;; ++t) {
                const int list = next_list;
                if (list < 0) break;
                next_list = next_list2;
                next_list2 = load_head(a, t + 2, total).x;
                const bool new_list = list != cur_list;
                if (new_list) {
                    kvb = (kvb + 1) & 1;
                    cur_list = list;
                    kv_ph ^= 1u << kvb;
                }
                const int bs = t % kQBuf;
                if (t >= kQBuf &&
                    !tc::mbar_wait(&s_free[bs], ((t / kQBuf) - 1) & 1, a.err, abort_flag))
                    break;
                if (!tc::mbar_wait(&q_full[bs], (t / kQBuf) & 1, a.err, abort_flag)) break;
                if (new_list &&
                    !tc::mbar_wait(&kv_full[kvb], ((kv_ph >> kvb) & 1) ^ 1, a.err, abort_flag))
                    break;
                tc::tc_fence_after();
                const uint32_t qa = tc::smem_u32(sQ + bs * kQBytes);
                const uint32_t ka = tc::smem_u32(sK + kvb * kKBytes);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t ad =
                        tc::sdesc_sw128(qa + (ks / 4) * 1024 + (ks % 4) * 32, 16, kGroupBytes);
                    const uint64_t bd =
                        tc::sdesc_sw128(ka + (ks / 4) * BLOCK * 128 + (ks % 4) * 32, 16, 1024);
                    tc::mma_ss(tmem + bs * kSCols, ad, bd, idesc_s, ks > 0);
                }
                tc::mma_commit(&s_full[bs]);
            }
        } else if (warp == 2 && lane == 0) {
            // ------------------------------------------------ PV issuer: O = P V
            // once P(t) is in TMEM and the epilogue has read O(t - 1).  After a
            // list's last tile its K/V buffer is released to the loads.  The two
            // issuers are independent, so neither waits behind the other.
            constexpr uint32_t idesc_o = tc::idesc_bf16(kRows, D, 0, 1);
            int kvb = -1, cur_list = -1;
            int next_list = load_head(a, 0, total).x, next_list2 = load_head(a, 1, total).x;
            for (int t = 0;; ++t) {
                const int list = next_list;
                if (list < 0) break;
                next_list = next_list2;
                next_list2 = load_head(a, t + 2, total).x;
                if (list != cur_list) {
                    kvb = (kvb + 1) & 1;
                    cur_list = list;
                }
                const int bp = t % kQBuf;
                if (!tc::mbar_wait(&p_full[bp], (t / kQBuf) & 1, a.err, abort_flag)) break;
                if (t >= 1 && !tc::mbar_wait(o_empty, (t - 1) & 1, a.err, abort_flag)) break;
                tc::tc_fence_after();
                const uint32_t va = tc::smem_u32(sV + kvb * kKBytes);
#pragma unroll
                for (int ks = 0; ks < BLOCK / 16; ++ks) {
                    const uint64_t bd = tc::sdesc_sw128(va + ks * 2048, BLOCK * 128, 1024);
                    tc::mma_ts(tmem + kOCol, tmem + bp * kSCols + ks * 8, bd, idesc_o, ks > 0);
                }
                tc::mma_commit(o_full);
                if (next_list != list) tc::mma_commit(&kv_empty[kvb]);
            }
        }
    } else if (wg == 1 || wg == 2) {
        tc::regs_inc<kRegsSoftmax>();
        // ------------------------------------------------ softmax (two groups)
        // Group g takes tiles g, g + 2, ...; S/P buffer t % 3.  Row maximum,
        // P = 2^((s - m) * scale * log2 e) on the special-function unit packed
        // to bf16 into TMEM for the PV product, and the partial's row, m and
        // the fp32 row sum l into the buffer's last columns for the epilogue.
        const int grp = wg - 1;
        const int quad = warp % 4;
        const int tt = (quad * 32 + lane) / a.R;      // the row's token in the tile
        const int h = (quad * 32 + lane) % a.R;       // and its head in the group
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        // records of this group's next two tiles in flight
        int2 nh = load_head(a, grp, total), nh2 = load_head(a, grp + 2, total);
        int nent = load_ent(a, grp, total, tt), nent2 = load_ent(a, grp + 2, total, tt);
        for (int i = grp;; i += 2) {
            const int2 d = nh;
            const int ent = nent;
            if (d.x < 0) break;
            nh = nh2;
            nent = nent2;
            nh2 = load_head(a, i + 4, total);
            nent2 = load_ent(a, i + 4, total, tt);
            const int list = d.x;
            const int n = list % a.NB;
            const bool valid = tt < d.y;
            const int rl = ent >> 8;                           // row within the chunk
            const int p = a.S - a.T + (int)((a.r0 + rl) % a.T);   // query position
            const int j_base = n * BLOCK;
            // the partial's row in the chunk (-1: no query)
            const int prow =
                valid ? ((rl * a.G + (list / a.NB) % a.G) * a.topk + (ent & 255)) * a.R + h : -1;
            const int bsel = i % kQBuf;
            const uint32_t tS = tmem + bsel * kSCols + lane_off;
            if (!tc::mbar_wait(&s_full[bsel], (i / kQBuf) & 1, a.err, abort_flag)) break;
            tc::tc_fence_after();
            const bool masked = valid && (j_base + BLOCK - 1 > p);
            // S is read from TMEM twice, 32 columns at a time, in rolled loops:
            // the code every warp of the sub-partition runs stays small enough
            // for its instruction cache (the unrolled passes were not; a TMEM
            // read is cheap).  Causal mask (only in a token's own block): keys
            // past the query position read as -inf.
            // Pass 1: row maximum.
            float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll 1
            for (int h0 = 0; h0 < BLOCK; h0 += 32) {
                uint32_t v[32];
                tc::tmem_ld32(tS + h0, v);
                tc::tmem_ld_wait();
                if (masked) {
                    const int lim = p - (j_base + h0);     // columns above lim are not causal
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (c > lim) v[c] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int c = 0; c < 32; c += 8) {
                    m0 = tc::fmax3(m0, __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
                    m1 = tc::fmax3(m1, __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
                    m2 = tc::fmax3(m2, __uint_as_float(v[c + 4]), __uint_as_float(v[c + 5]));
                    m3 = tc::fmax3(m3, __uint_as_float(v[c + 6]), __uint_as_float(v[c + 7]));
                }
            }
            float m = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
            if (!valid) m = 0.f;
            const float mb = m * a.scale_log2;
            // Pass 2: 2^x, packed to bf16 pairs and written over the S columns
            // already read, with four partial row sums.  Rows past the tile's
            // tokens hold no query and are never stored.
            float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll 1
            for (int h0 = 0; h0 < BLOCK; h0 += 32) {
                uint32_t v[32];
                tc::tmem_ld32(tS + h0, v);
                tc::tmem_ld_wait();
                if (masked) {
                    const int lim = p - (j_base + h0);
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (c > lim) v[c] = __float_as_uint(-INFINITY);
                }
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float e0 = tc::ex2_approx(fmaf(__uint_as_float(v[c]), a.scale_log2, -mb));
                    const float e1 = tc::ex2_approx(fmaf(__uint_as_float(v[c + 1]), a.scale_log2, -mb));
                    const float e2 = tc::ex2_approx(fmaf(__uint_as_float(v[c + 2]), a.scale_log2, -mb));
                    const float e3 = tc::ex2_approx(fmaf(__uint_as_float(v[c + 3]), a.scale_log2, -mb));
                    l0 += e0; l1 += e1; l2 += e2; l3 += e3;
                    __nv_bfloat162 b0 = __floats2bfloat162_rn(e0, e1);
                    __nv_bfloat162 b1 = __floats2bfloat162_rn(e2, e3);
                    pk[c / 2] = *(uint32_t *)&b0;
                    pk[c / 2 + 1] = *(uint32_t *)&b1;
                }
                tc::tmem_st16(tS + h0 / 2, pk);
            }
            const float l = (l0 + l1) + (l2 + l3);
            // the partial's row, m and l for the epilogue
            tc::tmem_st4(tS + (kSCols - 4), 0u, (uint32_t)prow, __float_as_uint(m),
                         __float_as_uint(l));
            tc::tmem_st_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(&p_full[bsel]);
        }
    } else {
        tc::regs_inc<kRegsEpilogue>();
        // ------------------------------------------------ epilogue
        // Every tile in order: wait for its PV product, read the O row and the
        // softmax's partial row, m and l from TMEM (which frees the accumulator
        // for the next PV and, with PV done, the tile's S/P buffer), then O / l
        // to bf16 (the range of fp32: no V the inputs can hold overflows it),
        // stored in 32-row blocked chunk planes (partial_chunk) so that
        // the rows of a warp store to consecutive addresses, and
        // LSE = m * scale + ln l.  No tile metadata is read from memory.
        const int quad = warp % 4;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tO = tmem + kOCol + lane_off;
        // partials are read back only by the combine: first out of L2
        const uint64_t st_pol = tc::policy_evict_first();
        for (int i = 0; run_tile(a, i) < total; ++i) {
            if (!tc::mbar_wait(o_full, i & 1, a.err, abort_flag)) break;
            tc::tc_fence_after();
            uint32_t ov[D];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) tc::tmem_ld32(tO + c0, *(uint32_t(*)[32])(ov + c0));
            const int bsel = i % kQBuf;
            uint32_t meta[4];                         // -, partial row, m, l
            tc::tmem_ld4(tmem + bsel * kSCols + lane_off + (kSCols - 4), meta);
            tc::tmem_ld_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(o_empty);
            tc::mbar_arrive(&s_free[bsel]);
            const int prow = (int)meta[1];
            const float m = __uint_as_float(meta[2]), l = __uint_as_float(meta[3]);
            const float inv = 1.f / l;
#pragma unroll
            for (int c = 0; c < D; c += 2) {
                __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(ov[c]) * inv,
                                                          __uint_as_float(ov[c + 1]) * inv);
                ov[c / 2] = *(uint32_t *)&hv;
            }
            if (prow >= 0 && MSA_IN_BOUNDS(prow, a.n_prows)) {
                uint4 *dst = (uint4 *)a.part_o + partial_chunk(prow, 0, D);
#pragma unroll
                for (int c = 0; c < D / 2; c += 4)
                    tc::st_global_v4_hint(dst + (c / 4) * 32,
                                          make_uint4(ov[c], ov[c + 1], ov[c + 2], ov[c + 3]), st_pol);
                tc::st_global_f32_hint(a.part_lse + prow, m * a.scale + logf(l), st_pol);
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

}  // namespace
}  // namespace msa

namespace msa {
namespace {

// The indexer's KL target for query rows [r0, r0 + rc), run after their
// merge: slot sl's share of head h's softmax is exp(part_lse - lse) of that
// slot (0 for slots no tile served), averaged over the group's R heads; after
// the two-pass merge (weights = true) part_lse already holds those shares.  One
// warp per (row, group), lanes laid out as in the merge (head l % R, slots
// l / R + k * 32 / R), so the head average is a shuffle over R lanes.
__global__ void __launch_bounds__(256)
block_mass_kernel(const int32_t *__restrict__ ids, const float *__restrict__ part_lse,
                  const float *__restrict__ lse, float *__restrict__ mass, int64_t r0, int64_t rc,
                  int T_, int S, int Hq, int G, int R, int NB, int block, int topk,
                  const int32_t *__restrict__ lens, bool weights) {
    const int64_t x = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (x >= rc * G) return;
    const int64_t rl = x / G, r = r0 + rl;
    const int g = (int)(x % G);
    const int t = (int)(r % T_);
    const int64_t p = seq_len(lens, (int)(r / T_), S) - T_ + t;
    const int cb = p < 0 ? -1 : (int)(p / block);
    const SlotPair sp = warp_slots2(ids + (r * G + g) * topk, topk, NB, cb, lane);
    const int h = lane % R, s0 = lane / R, sstep = 32 / R;
    const int per = (topk + sstep - 1) / sstep;
    const float l = lse[r * Hq + (int64_t)g * R + h];
    const int64_t base = x * topk * R;
    float *mrow = mass + (r * G + g) * topk;
    constexpr int kMaxPer = 16;                     // per <= 16 wherever the merge runs
    float li[kMaxPer];                              // every load issued before any use
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        const int sl = s0 + k * sstep;
        const bool okk = __shfl_sync(0xffffffffu, sl < 32 ? sp.ok0 : sp.ok1, sl & 31);
        li[k] = (k < per && sl < topk && okk) ? part_lse[base + (int64_t)sl * R + h] : -INFINITY;
    }
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
        if (k >= per) break;                        // per is uniform across the warp
        const int sl = s0 + k * sstep;
        float share = weights ? (li[k] == -INFINITY ? 0.f : li[k])
                              : (li[k] != -INFINITY && l != -INFINITY) ? expf(li[k] - l) : 0.f;
        for (int off = 1; off < R; off *= 2) share += __shfl_xor_sync(0xffffffffu, share, off);
        if (h == 0 && sl < topk) mrow[sl] = share / (float)R;
    }
}

// More than 64 kept blocks or 16 slots per lane: the same, slots taken in
// batches of 16 per lane.
__global__ void __launch_bounds__(256)
block_mass_wide_kernel(const int32_t *__restrict__ ids, const float *__restrict__ part_lse,
                  const float *__restrict__ lse, float *__restrict__ mass, int64_t r0, int64_t rc,
                  int T_, int S, int Hq, int G, int R, int NB, int block, int topk,
                  const int32_t *__restrict__ lens, bool weights) {
    const int64_t x = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (x >= rc * G) return;
    const int64_t rl = x / G, r = r0 + rl;
    const int g = (int)(x % G);
    const int t = (int)(r % T_);
    const int64_t p = seq_len(lens, (int)(r / T_), S) - T_ + t;
    const int cb = p < 0 ? -1 : (int)(p / block);
    const SlotSet<8> sp = warp_slots<8>(ids + (r * G + g) * topk, topk, NB, cb, lane);
    const int h = lane % R, s0 = lane / R, sstep = 32 / R;
    const int per = (topk + sstep - 1) / sstep;
    const float l = lse[r * Hq + (int64_t)g * R + h];
    const int64_t base = x * topk * R;
    float *mrow = mass + (r * G + g) * topk;
    constexpr int kMaxPer = 16;                     // slots per lane and batch
    for (int k0 = 0; k0 < per; k0 += kMaxPer) {
        float li[kMaxPer];                          // every load of a batch issued before any use
#pragma unroll
        for (int k = 0; k < kMaxPer; ++k) {
            const int sl = s0 + (k0 + k) * sstep;
            li[k] = (k0 + k < per && sl < topk && sp.valid(sl))
                        ? part_lse[base + (int64_t)sl * R + h] : -INFINITY;
        }
#pragma unroll
        for (int k = 0; k < kMaxPer; ++k) {
            if (k0 + k >= per) break;               // per is uniform across the warp
            const int sl = s0 + (k0 + k) * sstep;
            float share = weights ? (li[k] == -INFINITY ? 0.f : li[k])
                                  : (li[k] != -INFINITY && l != -INFINITY) ? expf(li[k] - l) : 0.f;
            for (int off = 1; off < R; off *= 2) share += __shfl_xor_sync(0xffffffffu, share, off);
            if (h == 0 && sl < topk) mrow[sl] = share / (float)R;
        }
    }
}

int combine_per(const Shape &s) { return (s.topk + 32 / s.R - 1) / (32 / s.R); }  // slots per lane
bool combine_wide(const Shape &s) { return combine_per(s) > 8; }
// More than 64 kept blocks, or more than 16 slots per merging lane: batches.
bool combine_batched(const Shape &s) { return s.topk > 64 || combine_per(s) > 16; }

CombineArgs combine_args(const Shape &s, const int32_t *ids, const __nv_bfloat16 *part_o,
                         const float *part_lse, void *O, float *lse, int64_t r0, int64_t rc,
                         const int32_t *lens) {
    CombineArgs c;
    c.ids = ids; c.part_o = part_o; c.part_lse = part_lse; c.O = (__nv_bfloat16 *)O; c.lse = lse;
    c.r0 = r0; c.rc = rc;
    c.T_ = s.T; c.S = s.S; c.Hq = s.Hq; c.G = s.G; c.R = s.R; c.NB = s.NB; c.block = s.block;
    c.topk = s.topk; c.lens = lens;
    return c;
}

constexpr size_t kPartialBudget = (size_t)4 << 30;   // bytes of partials per chunk
constexpr size_t kA = 256;
size_t al(size_t x) { return (x + kA - 1) / kA * kA; }

struct Plan {
    int64_t rows_per_chunk;
    int tpt;
    int64_t L;
    size_t counts, cursor, toffs, recs, part_o, part_lse, total;
};

Plan make_plan(const Shape &s) {
    Plan p;
    p.tpt = kRows / s.R;
    p.L = (int64_t)s.B * s.G * s.NB;
    const size_t per_row = (size_t)s.G * s.topk * s.R * (2 * (size_t)s.d + 4);
    int64_t rc = (int64_t)(kPartialBudget / per_row);
    if (rc < 1) rc = 1;
    if (rc > s.rows()) rc = s.rows();
    p.rows_per_chunk = rc;
    const size_t slots = (size_t)rc * s.G * s.topk;
    size_t o = 0;
    p.counts = o;   o += al(sizeof(int) * p.L);
    p.cursor = o;   o += al(sizeof(int) * p.L);
    p.toffs = o;    o += al(sizeof(int) * (p.L + 1));
    // at most ceil(slots / tpt) full tiles plus one partial tile per list
    p.recs = o;     o += al(sizeof(int) * rec_ints(p.tpt) * ((slots + p.tpt - 1) / p.tpt + p.L));
    p.part_o = o;   o += al(sizeof(__nv_bfloat16) * ((slots * s.R + 31) / 32 * 32) * s.d);
    p.part_lse = o; o += al(sizeof(float) * slots * s.R);
    p.total = o;
    return p;
}

template <int D, int BLOCK>
cudaError_t run_chunks(const Shape &s, const void *Q, const void *K, const void *V,
                       const int32_t *ids, void *O, float *lse, uint32_t *err, char *ws,
                       cudaStream_t st, float *mass) {
    const Plan pl = make_plan(s);
    CUtensorMap tq, tk, tv;
    const uint64_t dims[3] = {(uint64_t)s.d, (uint64_t)s.Hkv, (uint64_t)s.B * s.S};
    const uint64_t strides[2] = {(uint64_t)s.d * 2, (uint64_t)s.Hkv * s.d * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)BLOCK};
    if (!make_tmap_bf16(&tk, K, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&tv, V, 3, dims, strides, box)) return cudaErrorInvalidValue;
    // Q as [B*T][atom][Hq][64] (atoms of 64 channels, stride 128 bytes): one box =
    // 8 heads of one token, both atoms, atom-major in shared memory.  Where the
    // encoder rejects that stride order, Q as [B*T][Hq][d] with one box per atom.
    int q_box4 = 1;
    {
        const uint64_t qdims[4] = {64, (uint64_t)s.Hq, (uint64_t)s.d / 64, (uint64_t)s.B * s.T};
        const uint64_t qstrides[3] = {(uint64_t)s.d * 2, 128, (uint64_t)s.Hq * s.d * 2};
        const uint32_t qbox[4] = {64, 8, (uint32_t)s.d / 64, 1};
        if (!make_tmap_bf16(&tq, Q, 4, qdims, qstrides, qbox)) {
            q_box4 = 0;
            const uint64_t qdims3[3] = {(uint64_t)s.d, (uint64_t)s.Hq, (uint64_t)s.B * s.T};
            const uint64_t qstrides3[2] = {(uint64_t)s.d * 2, (uint64_t)s.Hq * s.d * 2};
            const uint32_t qbox3[3] = {64, 8, 1};
            if (s.R >= 8 && !make_tmap_bf16(&tq, Q, 3, qdims3, qstrides3, qbox3))
                return cudaErrorInvalidValue;
        }
    }
    int *counts = (int *)(ws + pl.counts), *cursor = (int *)(ws + pl.cursor);
    int *toffs = (int *)(ws + pl.toffs);
    int *recs = (int *)(ws + pl.recs);
    __nv_bfloat16 *part_o = (__nv_bfloat16 *)(ws + pl.part_o);
    float *part_lse = (float *)(ws + pl.part_lse);
    const size_t smem = 1024 + 3 * (size_t)kRows * D * 2 + 4 * (size_t)BLOCK * D * 2 + 256;
    auto kern = attn_tc_kernel<D, BLOCK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int L = (int)pl.L;
    for (int64_t r0 = 0; r0 < s.rows(); r0 += pl.rows_per_chunk) {
        const int64_t rc = std::min<int64_t>(pl.rows_per_chunk, s.rows() - r0);
        e = cudaMemsetAsync(counts, 0, pl.toffs - pl.counts, st);   // counts and cursor
        if (e != cudaSuccess) return e;
        const int64_t nrow = rc * s.G;                      // one warp each
        const unsigned g1 = (unsigned)((nrow * 32 + 255) / 256);
        auto count_k = s.topk > 64 ? csr_count_kernel<8> : csr_count_kernel<2>;
        auto fill_k = s.topk > 64 ? csr_fill_kernel<8> : csr_fill_kernel<2>;
        count_k<<<g1, 256, 0, st>>>(ids, counts, err, r0, rc, s.T, s.S, s.G, s.NB, s.block,
                                    s.topk);
        csr_scan_kernel<<<1, 1024, 0, st>>>(counts, toffs, L, pl.tpt);
        fill_k<<<g1, 256, 0, st>>>(ids, toffs, cursor, recs, r0, rc, s.T, s.S, s.G, s.NB,
                                   s.block, s.topk, pl.tpt, (int64_t)(pl.part_o - pl.recs) / 4);
        csr_tiles_kernel<<<(L + 255) / 256, 256, 0, st>>>(counts, toffs, recs, L, pl.tpt);
        AttnArgs a{};
        a.Q = (const __nv_bfloat16 *)Q;
        a.recs = recs;
        a.n_tiles = toffs + L;
        a.part_o = part_o; a.part_lse = part_lse; a.err = err; a.r0 = r0;
        a.n_prows = rc * s.G * s.topk * s.R;
        a.q_rows = s.rows();
        a.T = s.T; a.S = s.S; a.Hq = s.Hq; a.G = s.G; a.R = s.R; a.NB = s.NB; a.topk = s.topk;
        a.tpt = pl.tpt;
        a.q_box4 = q_box4;
        a.scale = s.scale;
        a.scale_log2 = s.scale * kLog2e;
        if ((e = prof_mark(st, kProfAttn, false)) != cudaSuccess) return e;
        kern<<<sms, kThreads, smem, st>>>(tq, tk, tv, a);
        if ((e = prof_mark(st, kProfAttn, true)) != cudaSuccess) return e;
        if ((e = prof_mark(st, kProfMerge, false)) != cudaSuccess) return e;
        e = launch_combine(s, ids, part_o, part_lse, O, lse, r0, rc, st, mass);
        if (e != cudaSuccess) return e;
        if ((e = prof_mark(st, kProfMerge, true)) != cudaSuccess) return e;
        count_launches(5);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

// The two-pass merge serves prefill-shaped calls (64 or more queries per
// sequence) whose group's heads fill whole warps; a decode step's few rows are
// bound by launch latency, where one pass is faster.  The choice depends on
// the call's shape only, never on how its rows are chunked, so a call split
// into pieces gives the same bits as the whole call.
bool merge_two_pass(const Shape &s) {
    return s.R * s.d >= 256 && !combine_batched(s) && s.T >= 64;
}

template <int D>
cudaError_t launch_merge_apply(const Shape &s, const CombineArgs &ca, const float *wts,
                               int64_t rc, cudaStream_t st) {
    const int64_t warps = rc * s.G * (D / 8 / (32 / s.R));
    const unsigned grid = (unsigned)((warps * 32 + 255) / 256);
    switch (s.R) {
        case 2: if constexpr (D / 8 >= 16) merge_apply_kernel<D, 2><<<grid, 256, 0, st>>>(ca, wts); break;
        case 4: if constexpr (D / 8 >= 8) merge_apply_kernel<D, 4><<<grid, 256, 0, st>>>(ca, wts); break;
        case 8: merge_apply_kernel<D, 8><<<grid, 256, 0, st>>>(ca, wts); break;
        case 16: merge_apply_kernel<D, 16><<<grid, 256, 0, st>>>(ca, wts); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaSuccess;
}

cudaError_t launch_block_mass(const Shape &s, const int32_t *ids, const float *part_lse,
                              const float *lse, float *mass, int64_t r0, int64_t rc,
                              cudaStream_t st, const int32_t *lens) {
    const unsigned mgrid = (unsigned)((rc * s.G * 32 + 255) / 256);
    auto k = combine_batched(s) ? block_mass_wide_kernel : block_mass_kernel;
    k<<<mgrid, 256, 0, st>>>(ids, part_lse, lse, mass, r0, rc, s.T, s.S, s.Hq, s.G, s.R, s.NB,
                             s.block, s.topk, lens, merge_two_pass(s));
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_combine(const Shape &s, const int32_t *ids, const __nv_bfloat16 *part_o,
                           float *part_lse, void *O, float *lse, int64_t r0, int64_t rc,
                           cudaStream_t st, float *mass, const int32_t *lens) {
    if (merge_two_pass(s)) {
        const CombineArgs ca = combine_args(s, ids, part_o, part_lse, O, lse, r0, rc, lens);
        const unsigned g1 = (unsigned)((rc * s.G * 32 + 255) / 256);
        if (combine_wide(s)) merge_weights_kernel<16><<<g1, 256, 0, st>>>(ca, part_lse);
        else merge_weights_kernel<8><<<g1, 256, 0, st>>>(ca, part_lse);
        const cudaError_t e = s.d == 64 ? launch_merge_apply<64>(s, ca, part_lse, rc, st)
                                        : launch_merge_apply<128>(s, ca, part_lse, rc, st);
        if (e != cudaSuccess) return e;
        count_launches(2);
        if (mass != nullptr) {
            const cudaError_t e2 = cudaGetLastError();
            if (e2 != cudaSuccess) return e2;
            return launch_block_mass(s, ids, part_lse, lse, mass, r0, rc, st, lens);
        }
        return cudaGetLastError();
    }
    const int64_t warps = rc * s.G * (s.d / 8 / kCombineChunksPerWarp);
    const unsigned grid = (unsigned)((warps * 32 + 255) / 256);
    // slots per merging lane: one batch of 8 or 16, or batches of 8 past 64 kept blocks
    const bool batched = combine_batched(s);
    auto kern = s.d == 64 ? (batched ? combine_kernel<64, 8, 8>
                             : combine_wide(s) ? combine_kernel<64, 16, 0>
                                               : combine_kernel<64, 8, 0>)
                          : (batched ? combine_kernel<128, 8, 8>
                             : combine_wide(s) ? combine_kernel<128, 16, 0>
                                               : combine_kernel<128, 8, 0>);
    kern<<<grid, 256, 0, st>>>(combine_args(s, ids, part_o, part_lse, O, lse, r0, rc, lens));
    count_launches(1);
    if (mass != nullptr) {
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return launch_block_mass(s, ids, part_lse, lse, mass, r0, rc, st, lens);
    }
    return cudaGetLastError();
}

cudaError_t launch_slot_csr(const Shape &s, const int32_t *ids, int tpt, int64_t r0, int64_t rc,
                            int *counts, int *cursor, int *toffs, int *recs, uint32_t *err,
                            cudaStream_t st) {
    const int L = s.B * s.G * s.NB;
    cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)L, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(cursor, 0, sizeof(int) * (size_t)L, st);
    if (e != cudaSuccess) return e;
    const unsigned g1 = (unsigned)((rc * s.G * 32 + 255) / 256);
    auto count_k = s.topk > 64 ? csr_count_kernel<8> : csr_count_kernel<2>;
    auto fill_k = s.topk > 64 ? csr_fill_kernel<8> : csr_fill_kernel<2>;
    count_k<<<g1, 256, 0, st>>>(ids, counts, err, r0, rc, s.T, s.S, s.G, s.NB, s.block, s.topk);
    csr_scan_kernel<<<1, 1024, 0, st>>>(counts, toffs, L, tpt);
    fill_k<<<g1, 256, 0, st>>>(ids, toffs, cursor, recs, r0, rc, s.T, s.S, s.G, s.NB, s.block,
                               s.topk, tpt,
                               (int64_t)(slot_csr_records(s, rc, tpt) * rec_ints(tpt)));
    csr_tiles_kernel<<<(L + 255) / 256, 256, 0, st>>>(counts, toffs, recs, L, tpt);
    count_launches(4);
    return cudaGetLastError();
}

size_t slot_csr_records(const Shape &s, int64_t rc, int tpt) {
    const size_t slots = (size_t)rc * s.G * s.topk;
    return (slots + tpt - 1) / tpt + (size_t)s.B * s.G * s.NB;
}

int slot_csr_record_ints(int tpt) { return rec_ints(tpt); }

bool combine_supported(const Shape &s) {
    return (s.R == 1 || s.R == 2 || s.R == 4 || s.R == 8 || s.R == 16 || s.R == 32) &&
           s.topk <= 256;
}

bool attn_tc_supported(const Shape &s) {
    return s.dtype == MSA_BF16 && (s.d == 128 || s.d == 64) && (s.block == 128 || s.block == 64) &&
           s.R <= 16 && combine_supported(s);
}

size_t attn_tc_workspace(const Shape &s) { return make_plan(s).total; }

int64_t attn_tc_rows_per_pass(const Shape &s) { return make_plan(s).rows_per_chunk; }

cudaError_t launch_attn_tc(const Shape &s, const void *Q, const void *K, const void *V,
                           const int32_t *ids, void *O, float *lse, uint32_t *err, void *ws,
                           cudaStream_t st, float *mass) {
    if (s.d == 64)
        return s.block == 128 ? run_chunks<64, 128>(s, Q, K, V, ids, O, lse, err, (char *)ws, st, mass)
                              : run_chunks<64, 64>(s, Q, K, V, ids, O, lse, err, (char *)ws, st, mass);
    if (s.block == 128)
        return run_chunks<128, 128>(s, Q, K, V, ids, O, lse, err, (char *)ws, st, mass);
    return run_chunks<128, 64>(s, Q, K, V, ids, O, lse, err, (char *)ws, st, mass);
}

}  // namespace msa
