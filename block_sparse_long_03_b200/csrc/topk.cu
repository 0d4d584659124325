// topk.cu -- per-group Top-k over blocks with the current block forced.
//
// ("MiniMax Sparse Attention", Summary, second paragraph: each GQA group
// picks its own Top-k blocks and the block containing the current position
// is always kept; Key points, benchmark configuration: the current block is
// one of the k.)
//
// For row (b, t, g) with cb = p(t) / block, the kept set is cb plus the
// M = topk - 1 best candidates n < cb, ranked by (score descending, id
// ascending).  Scores are compared as fp32 bit patterns mapped to an
// order-preserving uint32 -- nothing is exponentiated.
//
// One warp per row.  The candidates' ordered keys are staged in shared
// memory.  For M <= 64 a lower bound of the M-th largest score (the M-th
// largest of the lanes' top-2 keys) usually leaves at most 128 candidates;
// those are compacted in id order and the M-th largest score u* among them
// is found bit by bit with warp ballots.  Otherwise a 4-pass radix select
// (8 bits per pass, warp-private histogram) over all candidates finds u*.
// Every candidate above u* is kept, and of the candidates equal to u* the
// lowest ids are kept until M is reached.  The kept ids are emitted in
// ascending id order with ballots, so the output needs no sort; cb is
// appended last (it is larger than every candidate) and unused slots get -1.
// Rows of more than 2048 blocks are too long to stage per warp; their warp
// streams the row from memory instead (topk_long_kernel), unless there are
// too few rows to fill the GPU that way (decode), where a CTA of 256
// threads takes each row (topk_cta_kernel).
#include "msa_internal.cuh"

namespace msa {
namespace {

// Scores compare as numbers: -0.0 and +0.0 are equal (the lower id wins the
// tie), so -0.0 takes the key of +0.0.
__device__ __forceinline__ uint32_t ordered_key(float f) {
    const uint32_t u = __float_as_uint(canon_zero(f));
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Of C <= kMaxCand candidates (ordered keys ck, ids ci, in ascending id
// order, with every one of the row's M best among them) keep the M best and
// write them in ascending id order, then cb.  One warp, two or four
// candidates per lane (candidate 32 q + lane in slot q): the M-th largest key u* is found
// bit by bit with ballots below the bits all candidates share; every
// candidate above u* is kept, then the ties at u* with the lowest ids.
constexpr int kMaxCand = 128;

template <int kSlots>
__device__ __forceinline__ void select_slots(const uint32_t *ck, const uint32_t *ci, int C, int M,
                                             int cb, int32_t *out, int lane) {
    const unsigned lt_mask = (1u << lane) - 1u;
    bool ok[kSlots];
    uint32_t k[kSlots];
    uint32_t all1 = 0xffffffffu, any1 = 0u;
#pragma unroll
    for (int q = 0; q < kSlots; ++q) {
        ok[q] = 32 * q + lane < C;
        k[q] = ok[q] ? ck[32 * q + lane] : 0u;
        all1 &= __reduce_and_sync(0xffffffffu, ok[q] ? k[q] : 0xffffffffu);
        any1 |= __reduce_or_sync(0xffffffffu, ok[q] ? k[q] : 0u);
    }
    const uint32_t diff = all1 ^ any1;
    const int top = diff ? 31 - __clz((int)diff) : -1;
    uint32_t u = top >= 0 ? all1 & ~((2u << top) - 1u) : all1;
    for (int bit = top; bit >= 0; --bit) {
        const uint32_t c = u | (1u << bit);
        int cnt = 0;
#pragma unroll
        for (int q = 0; q < kSlots; ++q)
            cnt += __popc(__ballot_sync(0xffffffffu, ok[q] && k[q] >= c));
        if (cnt >= M) u = c;
    }
    int gt = 0;
#pragma unroll
    for (int q = 0; q < kSlots; ++q) gt += __popc(__ballot_sync(0xffffffffu, ok[q] && k[q] > u));
    const int need = M - gt;
    int eq_before = 0, taken_before = 0;          // over the slots before slot q
#pragma unroll
    for (int q = 0; q < kSlots; ++q) {
        const unsigned eb = __ballot_sync(0xffffffffu, ok[q] && k[q] == u);
        const bool take = ok[q] && (k[q] > u || (k[q] == u && eq_before + __popc(eb & lt_mask) < need));
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        if (take) out[taken_before + __popc(tb & lt_mask)] = (int32_t)ci[32 * q + lane];
        eq_before += __popc(eb);
        taken_before += __popc(tb);
    }
    if (lane == 0) out[M] = cb;
}

__device__ __forceinline__ void select_candidates(const uint32_t *ck, const uint32_t *ci, int C,
                                                  int M, int cb, int32_t *out, int lane) {
    if (C <= 64)                                  // C is the same in every lane
        select_slots<2>(ck, ci, C, M, cb, out, lane);
    else
        select_slots<4>(ck, ci, C, M, cb, out, lane);
}

__global__ void topk_kernel(const float *__restrict__ bs, int32_t *__restrict__ ids,
                            int64_t nrows, int T_, int S, int G, int NB, int block, int topk,
                            int warps_per_cta, const int32_t *__restrict__ lens) {
    extern __shared__ uint32_t sm[];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t r = (int64_t)blockIdx.x * warps_per_cta + warp;
    if (r >= nrows) return;
    uint32_t *keys = sm + (size_t)warp * (NB + 256);
    uint32_t *hist = keys + NB;
    const int t = (int)((r / G) % T_);
    const int64_t p = seq_len(lens, (int)(r / G / T_), S) - T_ + t;
    const int cb = (int)(p / block);
    const int M = topk - 1;
    int32_t *out = ids + r * topk;
    const unsigned lt_mask = (1u << lane) - 1u;

    if (p < 0) {                      // a sequence marked as doing no work
        for (int i = lane; i < topk; i += 32) out[i] = -1;
        return;
    }
    if (M == 0) {                     // only the forced block
        if (lane == 0) out[0] = cb;
        return;
    }
    if (cb <= M) {                    // every causal block is kept
        for (int i = lane; i < topk; i += 32) out[i] = (i <= cb) ? i : -1;
        return;
    }
    const float *row = bs + r * NB;
    uint32_t b1 = 0u, b2 = 0u;        // this lane's two largest keys (0: none)
    for (int n0 = lane; n0 < cb; n0 += 128) {
        float f[4];                   // four loads in flight per lane
#pragma unroll
        for (int u = 0; u < 4; ++u) f[u] = n0 + 32 * u < cb ? row[n0 + 32 * u] : -INFINITY;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (n0 + 32 * u < cb) {
                const uint32_t v = ordered_key(f[u]);
                keys[n0 + 32 * u] = v;
                b2 = max(b2, min(v, b1));
                b1 = max(b1, v);
            }
        }
    }
    __syncwarp();

    if (M <= 64) {
        // A lower bound tau of the M-th largest key: the M-th largest of the 64
        // per-lane top-2 keys (a subset of the candidates), found on its top 16
        // bits (truncating only lowers it).  Every one of the M best candidates
        // has key >= tau, and on these scores few others do.
        uint32_t tau = 0u;
        for (int bit = 31; bit >= 16; --bit) {
            const uint32_t c = tau | (1u << bit);
            const int cnt = __popc(__ballot_sync(0xffffffffu, b1 >= c)) +
                            __popc(__ballot_sync(0xffffffffu, b2 >= c));
            if (cnt >= M) tau = c;
        }
        // candidates with key >= tau, compacted in ascending id order
        uint32_t *ck = hist, *ci = hist + kMaxCand;
        int C = 0;
        for (int base = 0; base < cb; base += 32) {
            const int n = base + lane;
            const uint32_t v = n < cb ? keys[n] : 0u;
            const bool f = n < cb && v >= tau;
            const unsigned fb = __ballot_sync(0xffffffffu, f);
            const int pos = C + __popc(fb & lt_mask);
            if (f && pos < kMaxCand) {
                ck[pos] = v;
                ci[pos] = (uint32_t)n;
            }
            C += __popc(fb);
        }
        __syncwarp();
        if (C <= kMaxCand) {
            select_candidates(ck, ci, C, M, cb, out, lane);
            return;
        }
        __syncwarp();                 // the radix select below reuses hist
    }

    uint32_t prefix = 0, mask = 0;
    int remaining = M;                // how many still to take at or below prefix
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        for (int n = lane; n < cb; n += 32) {
            const uint32_t v = keys[n];
            if ((v & mask) == prefix) atomicAdd(&hist[(v >> shift) & 255u], 1u);
        }
        __syncwarp();
        // lane L owns digits [8L, 8L + 8); suffix sums over digits, high to low
        uint32_t c[8], lane_sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { c[i] = hist[lane * 8 + i]; lane_sum += c[i]; }
        uint32_t above = 0;           // count in lanes > this lane
        {
            uint32_t incl = lane_sum; // inclusive suffix sum over lanes >= lane
#pragma unroll
            for (int off = 1; off < 32; off *= 2) {
                const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
                if (lane + off < 32) incl += o;
            }
            above = incl - lane_sum;
        }
        // the digit D where the running count from the top first reaches `remaining`
        int found = -1;
        uint32_t gt_count = 0;
        if (above < (uint32_t)remaining && above + lane_sum >= (uint32_t)remaining) {
            uint32_t acc = above;
            for (int i = 7; i >= 0; --i) {
                if (acc + c[i] >= (uint32_t)remaining) { found = lane * 8 + i; gt_count = acc; break; }
                acc += c[i];
            }
        }
        const unsigned who = __ballot_sync(0xffffffffu, found >= 0);
        const int src = __ffs(who) - 1;
        const int digit = __shfl_sync(0xffffffffu, found, src);
        gt_count = __shfl_sync(0xffffffffu, gt_count, src);
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
        remaining -= (int)gt_count;
        __syncwarp();
    }
    // prefix == u*, `remaining` ties at u* are to be taken, lowest ids first
    int ties_seen = 0, written = 0;
    for (int base = 0; base < cb; base += 32) {
        const int n = base + lane;
        const uint32_t v = (n < cb) ? keys[n] : 0u;
        const bool eq = (n < cb) && v == prefix;
        const unsigned eq_b = __ballot_sync(0xffffffffu, eq);
        const int tie_rank = ties_seen + __popc(eq_b & lt_mask);
        const bool take = (n < cb) && (v > prefix || (eq && tie_rank < remaining));
        const unsigned tk_b = __ballot_sync(0xffffffffu, take);
        const int pos = written + __popc(tk_b & lt_mask);
        if (take && pos < M) out[pos] = n;
        ties_seen += __popc(eq_b);
        written += __popc(tk_b);
    }
    if (lane == 0) out[M] = cb;
}

// Rows with many candidates (NB > kWarpRowMaxNB, the 1M-token context): one
// warp per row, nothing staged in shared memory.  Pass 1 streams the row's
// candidate scores from memory with 16-byte loads (four in flight per lane)
// and keeps each lane's two largest keys; their M-th largest, on its top 16
// bits, is a lower bound tau of the M-th largest key.  Pass 2 streams the
// row again (now mostly from L2) and compacts the candidates >= tau in id
// order into the warp's shared buffer; with at most 128 of them the
// ballot selection of the warp kernel finishes the row.  Otherwise (heavy
// ties, or M > 64) a radix select runs over the row in memory, one pass per
// 8 bits, and the ordered emission reads it once more.  There are no block
// barriers: every warp works alone.
constexpr int kLongWarps = 8;

// Four consecutive scores n .. n + 3 of a row (kVec: one 16-byte load, rows
// 16-byte aligned; otherwise four scalar loads); past the row's end: 0.
template <bool kVec>
__device__ __forceinline__ float4 load4(const float *row, int n, int limit) {
    if (n >= limit) return make_float4(0.f, 0.f, 0.f, 0.f);
    if (kVec) return __ldg((const float4 *)(row + n));
    return make_float4(__ldg(row + n), n + 1 < limit ? __ldg(row + n + 1) : 0.f,
                       n + 2 < limit ? __ldg(row + n + 2) : 0.f,
                       n + 3 < limit ? __ldg(row + n + 3) : 0.f);
}

// kTop: keys each lane keeps in pass 1 (2, or 4 when M > 32, so that the
// threshold of the M-th largest stays close to it and few candidates pass).
template <bool kVec, int kTop>
__global__ void __launch_bounds__(kLongWarps * 32)
topk_long_kernel(const float *__restrict__ bs, int32_t *__restrict__ ids, int64_t nrows, int T_,
                 int S, int G, int NB, int block, int topk, const int32_t *__restrict__ lens) {
    __shared__ uint32_t s_buf[kLongWarps][2 * kMaxCand];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t r = (int64_t)blockIdx.x * kLongWarps + warp;
    if (r >= nrows) return;
    uint32_t *ck = s_buf[warp], *ci = s_buf[warp] + kMaxCand;
    const int t = (int)((r / G) % T_);
    const int64_t p = seq_len(lens, (int)(r / G / T_), S) - T_ + t;
    const int cb = (int)(p / block);
    const int M = topk - 1;
    int32_t *out = ids + r * topk;
    const unsigned lt_mask = (1u << lane) - 1u;
    if (p < 0) {
        for (int i = lane; i < topk; i += 32) out[i] = -1;
        return;
    }
    if (M == 0) {
        if (lane == 0) out[0] = cb;
        return;
    }
    if (cb <= M) {
        for (int i = lane; i < topk; i += 32) out[i] = (i <= cb) ? i : -1;
        return;
    }
    const float *row = bs + r * NB;                 // kVec: NB % 4 == 0, aligned rows
    const int nchunk = (cb + 3) / 4;                // chunks holding a candidate
    auto key_of = [&](float f, int n) -> uint32_t { return n < cb ? ordered_key(f) : 0u; };

    if (M <= 64) {
        uint32_t bt[kTop];                          // this lane's largest keys, descending
#pragma unroll
        for (int q = 0; q < kTop; ++q) bt[q] = 0u;
        for (int c0 = lane; c0 < nchunk; c0 += 128) {
            float4 f[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) f[u] = load4<kVec>(row, 4 * (c0 + 32 * u), cb);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int n = 4 * (c0 + 32 * u);
                const uint32_t k4[4] = {key_of(f[u].x, n), key_of(f[u].y, n + 1),
                                        key_of(f[u].z, n + 2), key_of(f[u].w, n + 3)};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
#pragma unroll
                    for (int q = kTop - 1; q > 0; --q) bt[q] = max(bt[q], min(k4[e], bt[q - 1]));
                    bt[0] = max(bt[0], k4[e]);
                }
            }
        }
        uint32_t tau = 0u;
        for (int bit = 31; bit >= 16; --bit) {
            const uint32_t c = tau | (1u << bit);
            int cnt = 0;
#pragma unroll
            for (int q = 0; q < kTop; ++q) cnt += __popc(__ballot_sync(0xffffffffu, bt[q] >= c));
            if (cnt >= M) tau = c;
        }
        // candidates >= tau in ascending id order: lane l owns ids 4l .. 4l + 3
        // of each 128-id round; its base is the count of the lanes before it
        int C = 0;
        for (int c0 = 0; c0 < nchunk; c0 += 32) {
            const int c = c0 + lane;
            const float4 f = load4<kVec>(row, 4 * c, cb);
            const int n = 4 * c;
            const uint32_t k4[4] = {key_of(f.x, n), key_of(f.y, n + 1), key_of(f.z, n + 2),
                                    key_of(f.w, n + 3)};
            int mine = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) mine += (n + e < cb && k4[e] >= tau) ? 1 : 0;
            int incl = mine;
#pragma unroll
            for (int off = 1; off < 32; off *= 2) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            int pos = C + incl - mine;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (n + e < cb && k4[e] >= tau) {
                    if (pos < kMaxCand) {
                        ck[pos] = k4[e];
                        ci[pos] = (uint32_t)(n + e);
                    }
                    ++pos;
                }
            }
            C += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncwarp();
        if (C <= kMaxCand) {
            select_candidates(ck, ci, C, M, cb, out, lane);
            return;
        }
        __syncwarp();                               // the radix select reuses the buffer
    }

    // radix select over the row in memory, 8 bits per pass
    uint32_t *hist = s_buf[warp];                   // 256 counters
    uint32_t prefix = 0, mask = 0;
    int remaining = M;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        for (int n = lane; n < cb; n += 32) {
            const uint32_t v = ordered_key(row[n]);
            if ((v & mask) == prefix) atomicAdd(&hist[(v >> shift) & 255u], 1u);
        }
        __syncwarp();
        uint32_t c[8], lane_sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { c[i] = hist[lane * 8 + i]; lane_sum += c[i]; }
        uint32_t incl = lane_sum;
#pragma unroll
        for (int off = 1; off < 32; off *= 2) {
            const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
            if (lane + off < 32) incl += o;
        }
        const uint32_t above = incl - lane_sum;
        int found = -1;
        uint32_t gt_count = 0;
        if (above < (uint32_t)remaining && above + lane_sum >= (uint32_t)remaining) {
            uint32_t acc = above;
            for (int i = 7; i >= 0; --i) {
                if (acc + c[i] >= (uint32_t)remaining) { found = lane * 8 + i; gt_count = acc; break; }
                acc += c[i];
            }
        }
        const unsigned who = __ballot_sync(0xffffffffu, found >= 0);
        const int src = __ffs(who) - 1;
        const int digit = __shfl_sync(0xffffffffu, found, src);
        gt_count = __shfl_sync(0xffffffffu, gt_count, src);
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
        remaining -= (int)gt_count;
        __syncwarp();
    }
    int ties_seen = 0, written = 0;
    for (int base = 0; base < cb; base += 32) {
        const int n = base + lane;
        const uint32_t v = n < cb ? ordered_key(row[n]) : 0u;
        const bool eq = n < cb && v == prefix;
        const unsigned eq_b = __ballot_sync(0xffffffffu, eq);
        const int tie_rank = ties_seen + __popc(eq_b & lt_mask);
        const bool take = n < cb && (v > prefix || (eq && tie_rank < remaining));
        const unsigned tk_b = __ballot_sync(0xffffffffu, take);
        const int pos = written + __popc(tk_b & lt_mask);
        if (take && pos < M) out[pos] = n;
        ties_seen += __popc(eq_b);
        written += __popc(tk_b);
    }
    if (lane == 0) out[M] = cb;
}

constexpr int kWarpRowMaxNB = 2048;       // beyond: topk_long_kernel, or
constexpr int kLongMinRows = 4096;        // topk_cta_kernel for fewer rows than this

// Last step of the coarse-to-fine selection: row r's candidates cand[r, 0..kc)
// (ascending block ids, the current block last, -1 padding) with their
// exact block scores fine[r, 0..kc).  Keeps the current block and the
// topk - 1 best candidates below it, by (score descending, id ascending),
// written ascending and -1 padded.  One warp per row, through the same
// ballot selection as the Top-k kernels (kc <= 64 candidates).
constexpr int kSelWarps = 8;

__global__ void __launch_bounds__(kSelWarps * 32)
select_among_kernel(const int32_t *__restrict__ cand, const float *__restrict__ fine,
                    int32_t *__restrict__ ids, int64_t nrows, int T_, int S, int G, int block,
                    int kc, int topk) {
    __shared__ uint32_t s_buf[kSelWarps][2 * kMaxCand];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t r = (int64_t)blockIdx.x * kSelWarps + warp;
    if (r >= nrows) return;
    uint32_t *ck = s_buf[warp], *ci = s_buf[warp] + kMaxCand;
    const int t = (int)((r / G) % T_);
    const int cb = (int)(((int64_t)S - T_ + t) / block);
    const int M = topk - 1;
    int32_t *out = ids + r * topk;
    const unsigned lt_mask = (1u << lane) - 1u;
    int C = 0;
    for (int c0 = 0; c0 < kc; c0 += 32) {
        const int c = c0 + lane;
        const int n = c < kc ? cand[r * kc + c] : -1;
        const bool ok = n >= 0 && n < cb;
        const unsigned fb = __ballot_sync(0xffffffffu, ok);
        const int pos = C + __popc(fb & lt_mask);
        if (ok) {
            ck[pos] = ordered_key(fine[r * kc + c]);
            ci[pos] = (uint32_t)n;
        }
        C += __popc(fb);
    }
    __syncwarp();
    if (C <= M) {                     // every candidate is kept
        for (int i = lane; i < topk; i += 32)
            out[i] = i < C ? (int32_t)ci[i] : (i == C ? cb : -1);
        return;
    }
    select_candidates(ck, ci, C, M, cb, out, lane);
}

// Few rows with many candidates (decode at the 1M context: too few rows to
// fill the GPU one warp per row): one CTA of kCtaThreads
// threads per row runs the same selection (the threshold filter first, the
// radix select when it leaves more than 128 candidates), the histogram and the
// ordered emission shared by its warps; leading bits shared by every
// candidate need no radix pass.
constexpr int kCtaThreads = 256;

__global__ void __launch_bounds__(kCtaThreads)
topk_cta_kernel(const float *__restrict__ bs, int32_t *__restrict__ ids, int T_, int S, int G,
                int NB, int block, int topk, const int32_t *__restrict__ lens) {
    extern __shared__ uint32_t sm[];
    constexpr int kWarps = kCtaThreads / 32;
    uint32_t *keys = sm;                          // [NB]
    uint32_t *hist = keys + NB;                   // [256]
    uint32_t *red = hist + 256;                   // [2 * kWarps] reductions / warp counts
    int *sel = (int *)(red + 2 * kWarps);         // [3]: digit, gt_count, (spare)
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int64_t r = blockIdx.x;
    const int t = (int)((r / G) % T_);
    const int64_t p = seq_len(lens, (int)(r / G / T_), S) - T_ + t;
    const int cb = (int)(p / block);
    const int M = topk - 1;
    int32_t *out = ids + r * topk;
    const unsigned lt_mask = (1u << lane) - 1u;
    if (p < 0) {
        for (int i = tid; i < topk; i += kCtaThreads) out[i] = -1;
        return;
    }
    if (M == 0) {
        if (tid == 0) out[0] = cb;
        return;
    }
    if (cb <= M) {
        for (int i = tid; i < topk; i += kCtaThreads) out[i] = (i <= cb) ? i : -1;
        return;
    }
    const float *row = bs + r * NB;
    uint32_t all_and = 0xffffffffu, all_or = 0u;
    uint32_t b1 = 0u, b2 = 0u;                    // this thread's two largest keys (0: none)
    for (int n = tid; n < cb; n += kCtaThreads) {
        const uint32_t v = ordered_key(row[n]);
        keys[n] = v;
        all_and &= v;
        all_or |= v;
        b2 = max(b2, min(v, b1));
        b1 = max(b1, v);
    }
    all_and = __reduce_and_sync(0xffffffffu, all_and);
    all_or = __reduce_or_sync(0xffffffffu, all_or);
    if (lane == 0) { red[warp] = all_and; red[kWarps + warp] = all_or; }
    __syncthreads();
    all_and = 0xffffffffu; all_or = 0u;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) { all_and &= red[w]; all_or |= red[kWarps + w]; }
    if (M <= 64) {
        // As in the warp kernel: a lower bound tau of the M-th largest key
        // (the M-th largest of the threads' top-2 keys, on its top 16 bits),
        // the candidates >= tau compacted in id order, and if at most 128,
        // warp 0 selects among them.  Counts cross the warps through a
        // double-buffered shared array (one barrier per step).
        __shared__ int cnt[2][kWarps];
        uint32_t tau = 0u;
        for (int bit = 31, it = 0; bit >= 16; --bit, ++it) {
            const uint32_t c = tau | (1u << bit);
            const int n_ge = __popc(__ballot_sync(0xffffffffu, b1 >= c)) +
                             __popc(__ballot_sync(0xffffffffu, b2 >= c));
            if (lane == 0) cnt[it & 1][warp] = n_ge;
            __syncthreads();
            int total = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) total += cnt[it & 1][w];
            if (total >= M) tau = c;
        }
        uint32_t *ck = hist, *ci = hist + kMaxCand;   // the radix path re-zeroes hist
        int C = 0;
        for (int base = 0, it = 0; base < cb; base += kCtaThreads, ++it) {
            const int n = base + tid;
            const uint32_t v = n < cb ? keys[n] : 0u;
            const bool f = n < cb && v >= tau;
            const unsigned fb = __ballot_sync(0xffffffffu, f);
            if (lane == 0) cnt[it & 1][warp] = __popc(fb);
            __syncthreads();
            int before = C, total = C;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                before += w < warp ? cnt[it & 1][w] : 0;
                total += cnt[it & 1][w];
            }
            const int pos = before + __popc(fb & lt_mask);
            if (f && pos < kMaxCand) {
                ck[pos] = v;
                ci[pos] = (uint32_t)n;
            }
            C = total;
        }
        __syncthreads();
        if (C <= kMaxCand) {                      // C is the same in every thread
            if (warp == 0) select_candidates(ck, ci, C, M, cb, out, lane);
            return;
        }
        __syncthreads();                          // hist is reused below
    }
    const uint32_t diff = all_and ^ all_or;
    const int top = diff ? 31 - __clz(diff) : -1;
    uint32_t prefix = 0, mask = 0;
    int first_shift = 24;
    while (first_shift > 0 && first_shift > top) first_shift -= 8;
    if (first_shift + 8 <= 31) {
        mask = 0xffffffffu << (first_shift + 8);
        prefix = all_and & mask;
    }
    int remaining = M;
    for (int shift = first_shift; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kCtaThreads) hist[i] = 0;
        __syncthreads();
        for (int base = 0; base < cb; base += kCtaThreads) {
            const int n = base + tid;
            const uint32_t v = n < cb ? keys[n] : 0u;
            const bool in = n < cb && (v & mask) == prefix;
            if (in) atomicAdd(&hist[(v >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t c[8], lane_sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) { c[i] = hist[lane * 8 + i]; lane_sum += c[i]; }
            uint32_t incl = lane_sum;
#pragma unroll
            for (int off = 1; off < 32; off *= 2) {
                const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
                if (lane + off < 32) incl += o;
            }
            const uint32_t above = incl - lane_sum;
            int found = -1;
            uint32_t gt_count = 0;
            if (above < (uint32_t)remaining && above + lane_sum >= (uint32_t)remaining) {
                uint32_t acc = above;
                for (int i = 7; i >= 0; --i) {
                    if (acc + c[i] >= (uint32_t)remaining) { found = lane * 8 + i; gt_count = acc; break; }
                    acc += c[i];
                }
            }
            if (found >= 0) { sel[0] = found; sel[1] = (int)gt_count; }
        }
        __syncthreads();
        prefix |= (uint32_t)sel[0] << shift;
        mask |= 255u << shift;
        remaining -= sel[1];
        __syncthreads();                              // sel and hist are reused
    }
    // ordered emission: per chunk of kCtaThreads ids, ranks from the warps'
    // ballot counts
    int ties_seen = 0, written = 0;
    for (int base = 0; base < cb; base += kCtaThreads) {
        const int n = base + tid;
        const uint32_t v = (n < cb) ? keys[n] : 0u;
        const bool eq = (n < cb) && v == prefix;
        const unsigned eq_b = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) red[warp] = __popc(eq_b);
        __syncthreads();
        int eq_before = ties_seen, eq_total = ties_seen;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            eq_before += w < warp ? (int)red[w] : 0;
            eq_total += (int)red[w];
        }
        const int tie_rank = eq_before + __popc(eq_b & lt_mask);
        const bool take = (n < cb) && (v > prefix || (eq && tie_rank < remaining));
        const unsigned tk_b = __ballot_sync(0xffffffffu, take);
        if (lane == 0) red[kWarps + warp] = __popc(tk_b);
        __syncthreads();
        int tk_before = written, tk_total = written;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            tk_before += w < warp ? (int)red[kWarps + w] : 0;
            tk_total += (int)red[kWarps + w];
        }
        const int pos = tk_before + __popc(tk_b & lt_mask);
        if (take && pos < M) out[pos] = n;
        ties_seen = eq_total;
        written = tk_total;
        __syncthreads();                              // red is reused
    }
    if (tid == 0) out[M] = cb;
}

}  // namespace

cudaError_t launch_topk(const Shape &s, const float *bs, int32_t *ids, cudaStream_t st,
                        const int32_t *lens) {
    const int64_t nrows = s.index_rows();
    if (s.NB > kWarpRowMaxNB && nrows < kLongMinRows) {
        const size_t smem = sizeof(uint32_t) * ((size_t)s.NB + 256 + 2 * (kCtaThreads / 32) + 4);
        if (smem > 220 * 1024) return cudaErrorInvalidConfiguration;
        cudaFuncSetAttribute(topk_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        topk_cta_kernel<<<(unsigned)nrows, kCtaThreads, smem, st>>>(bs, ids, s.T, s.S, s.G, s.NB,
                                                                     s.block, s.topk, lens);
        count_launches(1);
        return cudaGetLastError();
    }
    if (s.NB > kWarpRowMaxNB) {
        const unsigned grid = (unsigned)((nrows + kLongWarps - 1) / kLongWarps);
        const bool vec = (s.NB & 3) == 0 && ((uintptr_t)bs & 15) == 0, wide = s.topk - 1 > 32;
        auto k = vec ? (wide ? topk_long_kernel<true, 4> : topk_long_kernel<true, 2>)
                     : (wide ? topk_long_kernel<false, 4> : topk_long_kernel<false, 2>);
        k<<<grid, kLongWarps * 32, 0, st>>>(bs, ids, nrows, s.T, s.S, s.G, s.NB, s.block, s.topk,
                                            lens);
        count_launches(1);
        return cudaGetLastError();
    }
    const size_t per_warp = sizeof(uint32_t) * ((size_t)s.NB + 256);
    int warps = 8;
    while (warps > 1 && per_warp * warps > 200 * 1024) warps /= 2;
    if (per_warp * warps > 220 * 1024) return cudaErrorInvalidConfiguration;
    const size_t smem = per_warp * warps;
    cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int64_t grid = (nrows + warps - 1) / warps;
    topk_kernel<<<(unsigned)grid, warps * 32, smem, st>>>(bs, ids, nrows, s.T, s.S, s.G, s.NB,
                                                          s.block, s.topk, warps, lens);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_select_among(const Shape &s, const int32_t *cand, const float *fine, int kc,
                                int32_t *ids, cudaStream_t st) {
    if (kc > 2 * 32 || kc < s.topk) return cudaErrorInvalidValue;
    const int64_t nrows = s.index_rows();
    select_among_kernel<<<(unsigned)((nrows + kSelWarps - 1) / kSelWarps), kSelWarps * 32, 0, st>>>(
        cand, fine, ids, nrows, s.T, s.S, s.G, s.block, kc, s.topk);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
