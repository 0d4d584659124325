/*
 * msa_oracle.c -- plain, slow, fp64 CPU oracle for the forward pass of
 * MiniMax-Sparse-Attention-style block-sparse GQA attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this library.  The product path
 * (the CUDA library) never calls it, and it shares no code, header, table or
 * helper with the CUDA library.
 *
 * Source of the method: "MiniMax Sparse Attention -- paper by Lai et al.
 * (2026)", section "Summary" (second paragraph) and section "Key points"
 * (benchmark configuration; kernel design).  Restated in our own words:
 *   - a light index branch produces an index query per (token, GQA group) and
 *     an index key per token;
 *   - a KV block is scored by max-pooling the token-level dot products of the
 *     index query with the index keys of the block's tokens;
 *   - every GQA group keeps its own Top-k blocks; the block that holds the
 *     current position is always kept;
 *   - exact softmax attention then runs over the kept blocks only, and the
 *     log-sum-exp (LSE) of that softmax is an output of the forward pass.
 *
 * Readings of points the page leaves open (each is listed in the design
 * notes of the repository):
 *   - the forced current block counts as one of the k ("k = 16, B_k = 128
 *     gives 2,048 attended tokens per query");
 *   - inside a block only causal tokens (position j <= p(t)) are scored and
 *     attended; blocks with no causal token score -infinity;
 *   - ties in block score are broken toward the lower block id;
 *   - the softmax scale is 1/sqrt(d) unless the caller passes another;
 *   - LSE uses the natural logarithm of sum_j exp(scale * q.k_j);
 *   - with T query tokens against S keys, query t sits at absolute position
 *     p(t) = S - T + t (bottom-right causal alignment);
 *   - the kept block ids are written in ascending order, padded with -1;
 *   - the index score is the plain dot product (no weights, no ReLU), one
 *     index head per GQA group; KV head g is group g.
 *
 * Arithmetic: every input element is widened to double (bf16 and fp32 widen
 * exactly) and all sums, maxima, exponentials and logarithms run in double.
 * Loops are in the order of the definition; rows (b, t) run in parallel with
 * OpenMP, which changes no result.
 *
 * Layouts (dense, row-major, as the library's public header also uses):
 *   q_idx [B, T, G, d_idx]   k_idx [B, S, d_idx]
 *   Q     [B, T, Hq, d]      K, V  [B, S, Hkv, d]     G = Hkv
 * Work is done for a caller-chosen list of rows r = b * T + t, so that large
 * shapes can be checked on a sample of rows.  The query-side inputs are
 * passed already gathered for those rows, q_idx_rows [nrows, G, d_idx] and
 * Q_rows [nrows, Hq, d] (row ri of the list holds query (b, t) with
 * r = rows[ri]); the key-side inputs are the full tensors.  Outputs are
 * indexed by the position ri of the row in the list.
 *
 * Every entry point returns 0 on success and a negative value on a bad
 * argument.  Nothing is allocated that is not freed before return.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F32 0
#define ORACLE_BF16 1

/* Widen element i of a float32 or bfloat16 array to double (exact). */
static double widen(const void *base, int dtype, int64_t i)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* Absolute position of query t: bottom-right causal alignment. */
static int64_t query_pos(int64_t T, int64_t S, int64_t t) { return S - T + t; }

/*
 * Index branch: token-level index scores max-pooled per KV block
 * ("MiniMax Sparse Attention", Summary, second paragraph).
 *
 *   bs[r, g, n] = max over tokens j of block n with j <= p(t) of
 *                 sum_i q_idx[b, t, g, i] * k_idx[b, j, i]
 * (q_idx[b, t] is row ri of q_idx_rows).
 *   bs[r, g, n] = -inf when block n holds no token j <= p(t).
 *
 * Block n covers tokens [n * block, min((n + 1) * block, S)).
 * Output bs has shape [nrows, G, NB] with NB = ceil(S / block).
 */
int oracle_block_scores(int64_t B, int64_t T, int64_t S, int64_t G,
                        int64_t d_idx, int64_t block, int dtype,
                        const void *q_idx_rows, const void *k_idx,
                        const int64_t *rows, int64_t nrows, double *bs)
{
    if (B <= 0 || T <= 0 || S <= 0 || T > S || G <= 0 || d_idx <= 0 ||
        block <= 0 || nrows < 0 || (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
        return -1;
    const int64_t NB = ceil_div(S, block);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t ri = 0; ri < nrows; ++ri) {
        const int64_t r = rows[ri];
        if (r < 0 || r >= B * T) { bad = 1; continue; }
        const int64_t b = r / T, t = r % T;
        const int64_t p = query_pos(T, S, t);
        for (int64_t g = 0; g < G; ++g) {
            double *out = bs + (ri * G + g) * NB;
            for (int64_t n = 0; n < NB; ++n) {
                double best = -INFINITY;
                const int64_t j0 = n * block;
                int64_t j1 = j0 + block;
                if (j1 > S) j1 = S;
                for (int64_t j = j0; j < j1 && j <= p; ++j) {
                    double dot = 0.0;
                    for (int64_t i = 0; i < d_idx; ++i)
                        dot += widen(q_idx_rows, dtype, (ri * G + g) * d_idx + i) *
                               widen(k_idx, dtype, (b * S + j) * d_idx + i);
                    if (dot > best) best = dot;
                }
                out[n] = best;
            }
        }
    }
    return bad ? -2 : 0;
}

/*
 * Per-group Top-k with the current block forced
 * ("MiniMax Sparse Attention", Summary, second paragraph; Key points,
 * benchmark configuration: the k blocks include the current one).
 *
 * For row r (query t at position p) and group g, with cb = floor(p / block):
 *   kept = {cb} united with the k - 1 best blocks n < cb, where "better" is
 *          the larger block score, and on equal scores the lower block id.
 * The number kept is min(k, cb + 1).  Ids are written ascending to
 * ids[ri, g, 0..k-1] and the rest of the k slots is -1.
 *
 * The ranking is done the plain way: sort the candidate ids by
 * (score descending, id ascending), take the first k - 1, then sort those
 * ids ascending and append cb (which is larger than every candidate).
 */
typedef struct { double score; int64_t id; } cand_t;

static int cand_better_first(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

static int id_ascending(const void *a, const void *b)
{
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

int oracle_select_blocks(int64_t T, int64_t S, int64_t G, int64_t block,
                         int64_t topk, const double *bs, const int64_t *rows,
                         int64_t nrows, int32_t *ids)
{
    if (T <= 0 || S <= 0 || T > S || G <= 0 || block <= 0 || topk <= 0 || nrows < 0)
        return -1;
    const int64_t NB = ceil_div(S, block);
    int bad = 0;
#pragma omp parallel
    {
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)NB);
        if (!cand) bad = 1;
#pragma omp for schedule(dynamic, 4)
        for (int64_t ri = 0; ri < nrows; ++ri) {
            if (!cand) continue;
            const int64_t t = rows[ri] % T;
            const int64_t cb = query_pos(T, S, t) / block;
            for (int64_t g = 0; g < G; ++g) {
                const double *score = bs + (ri * G + g) * NB;
                int32_t *out = ids + (ri * G + g) * topk;
                for (int64_t n = 0; n < cb; ++n) {
                    cand[n].score = score[n];
                    cand[n].id = n;
                }
                qsort(cand, (size_t)cb, sizeof(cand_t), cand_better_first);
                const int64_t take = (cb < topk - 1) ? cb : topk - 1;
                for (int64_t i = 0; i < take; ++i) out[i] = (int32_t)cand[i].id;
                qsort(out, (size_t)take, sizeof(int32_t), id_ascending);
                out[take] = (int32_t)cb;
                for (int64_t i = take + 1; i < topk; ++i) out[i] = -1;
            }
        }
        free(cand);
    }
    return bad ? -2 : 0;
}

/*
 * Main branch: exact softmax attention restricted to the kept blocks
 * ("MiniMax Sparse Attention", Summary, second paragraph), with the LSE of
 * that softmax as a second output (Key points, kernel design).
 *
 * For row r (query t at position p), query head h, group g = h / (Hq / Hkv):
 *   J   = tokens j of every kept block n (ids[ri, g, :], entries < 0 are
 *         empty slots) with j <= p
 *   s_j = scale * sum_c Q[b, t, h, c] * K[b, j, g, c]   (Q[b, t] = Q_rows[ri])
 *   m   = max_j s_j
 *   O[ri, h, c] = sum_j exp(s_j - m) V[b, j, g, c] / sum_j exp(s_j - m)
 *   lse[ri, h]  = m + log(sum_j exp(s_j - m))
 * A kept id outside [0, NB) or listed twice is an error (-3): the oracle
 * only attends to a set of blocks.  The order of the kept ids does not
 * matter.  scale <= 0 means 1 / sqrt(d).
 */
int oracle_attention(int64_t B, int64_t T, int64_t S, int64_t Hq, int64_t Hkv,
                     int64_t d, int64_t block, int64_t topk, int dtype,
                     double scale, const void *Q_rows, const void *K, const void *V,
                     const int32_t *ids, const int64_t *rows, int64_t nrows,
                     double *O, double *lse)
{
    if (B <= 0 || T <= 0 || S <= 0 || T > S || Hq <= 0 || Hkv <= 0 ||
        Hq % Hkv != 0 || d <= 0 || block <= 0 || topk <= 0 || nrows < 0 ||
        (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
        return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    const int64_t NB = ceil_div(S, block);
    const int64_t R = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(topk * block));
        int64_t *key = (int64_t *)malloc(sizeof(int64_t) * (size_t)(topk * block));
        unsigned char *seen = (unsigned char *)calloc((size_t)NB, 1);
        if (!s || !key || !seen) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t ri = 0; ri < nrows; ++ri) {
            if (!s || !key || !seen) continue;
            const int64_t r = rows[ri];
            if (r < 0 || r >= B * T) { bad = 1; continue; }
            const int64_t b = r / T, t = r % T;
            const int64_t p = query_pos(T, S, t);
            for (int64_t h = 0; h < Hq; ++h) {
                const int64_t g = h / R;
                const int32_t *kept = ids + (ri * Hkv + g) * topk;
                /* the attended key set J */
                int64_t nkeys = 0;
                memset(seen, 0, (size_t)NB);
                for (int64_t i = 0; i < topk; ++i) {
                    const int64_t n = kept[i];
                    if (n < 0) continue;
                    if (n >= NB || seen[n]) { bad = 3; continue; }
                    seen[n] = 1;
                    for (int64_t j = n * block; j < (n + 1) * block && j < S && j <= p; ++j)
                        key[nkeys++] = j;
                }
                double *o = O + (ri * Hq + h) * d;
                if (nkeys == 0) {
                    /* nothing attended: defined as O = 0, lse = -inf */
                    for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
                    lse[ri * Hq + h] = -INFINITY;
                    continue;
                }
                /* pass 1: scores and their maximum */
                double m = -INFINITY;
                for (int64_t q = 0; q < nkeys; ++q) {
                    const int64_t j = key[q];
                    double dot = 0.0;
                    for (int64_t c = 0; c < d; ++c)
                        dot += widen(Q_rows, dtype, (ri * Hq + h) * d + c) *
                               widen(K, dtype, ((b * S + j) * Hkv + g) * d + c);
                    s[q] = scale * dot;
                    if (s[q] > m) m = s[q];
                }
                /* pass 2: normaliser and weighted sum of values */
                double denom = 0.0;
                for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
                for (int64_t q = 0; q < nkeys; ++q) {
                    const int64_t j = key[q];
                    const double w = exp(s[q] - m);
                    denom += w;
                    for (int64_t c = 0; c < d; ++c)
                        o[c] += w * widen(V, dtype, ((b * S + j) * Hkv + g) * d + c);
                }
                for (int64_t c = 0; c < d; ++c) o[c] /= denom;
                lse[ri * Hq + h] = m + log(denom);
            }
        }
        free(s);
        free(key);
        free(seen);
    }
    return bad ? -bad : 0;
}

/*
 * Target of the indexer's KL objective ("MiniMax Sparse Attention",
 * Summary, second paragraph: the indexer learns to match the Main Branch's
 * distribution averaged over the heads of a GQA group; Key points, kernel
 * design: the LSE that loss needs is a forward output).  For row r (query t
 * at position p), group g and kept slot i holding block n = ids[ri, g, i]:
 *   mass[ri, g, i] = (1 / R) * sum over heads h of g of
 *                    sum over tokens j of block n with j <= p of
 *                    exp(s_hj - lse[ri, h])
 * with s_hj = scale * Q[b, t, h] . K[b, j, g] as in oracle_attention and
 * lse the stored LSE of that row and head.  An empty slot (-1) gets 0, and
 * a head whose lse is -inf adds 0.  With the LSE of the same kept set, a
 * row's masses over its slots sum to 1.  Ids outside [0, NB) or listed
 * twice are an error (-3), as in oracle_attention.
 */
int oracle_block_mass(int64_t B, int64_t T, int64_t S, int64_t Hq, int64_t Hkv,
                      int64_t d, int64_t block, int64_t topk, int dtype, double scale,
                      const void *Q_rows, const void *K, const int32_t *ids,
                      const double *lse, const int64_t *rows, int64_t nrows, double *mass)
{
    if (B <= 0 || T <= 0 || S <= 0 || T > S || Hq <= 0 || Hkv <= 0 ||
        Hq % Hkv != 0 || d <= 0 || block <= 0 || topk <= 0 || nrows < 0 ||
        (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
        return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    const int64_t NB = ceil_div(S, block);
    const int64_t R = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        unsigned char *seen = (unsigned char *)calloc((size_t)NB, 1);
        if (!seen) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t ri = 0; ri < nrows; ++ri) {
            if (!seen) continue;
            const int64_t r = rows[ri];
            if (r < 0 || r >= B * T) { bad = 1; continue; }
            const int64_t b = r / T, t = r % T;
            const int64_t p = query_pos(T, S, t);
            for (int64_t g = 0; g < Hkv; ++g) {
                const int32_t *kept = ids + (ri * Hkv + g) * topk;
                double *out = mass + (ri * Hkv + g) * topk;
                memset(seen, 0, (size_t)NB);
                for (int64_t i = 0; i < topk; ++i) {
                    out[i] = 0.0;
                    const int64_t n = kept[i];
                    if (n < 0) continue;
                    if (n >= NB || seen[n]) { bad = 3; continue; }
                    seen[n] = 1;
                    const int64_t first = n * block;
                    const int64_t stop = (n + 1) * block < S ? (n + 1) * block : S;
                    double head_sum = 0.0;
                    for (int64_t hh = 0; hh < R; ++hh) {
                        const int64_t h = g * R + hh;           /* head hh of group g */
                        const double l = lse[ri * Hq + h];
                        if (l == -INFINITY) continue;
                        for (int64_t j = first; j < stop; ++j) {
                            if (j > p) break;                   /* causal tokens only */
                            double dot = 0.0;
                            for (int64_t c = 0; c < d; ++c)
                                dot += widen(Q_rows, dtype, (ri * Hq + h) * d + c) *
                                       widen(K, dtype, ((b * S + j) * Hkv + g) * d + c);
                            head_sum += exp(scale * dot - l);
                        }
                    }
                    out[i] = head_sum / (double)R;
                }
            }
        }
        free(seen);
    }
    return bad ? -bad : 0;
}

/*
 * The whole forward pass for a list of rows: index scores, selection, then
 * attention.  ids_out [nrows, G, topk] (int32), O [nrows, Hq, d] and
 * lse [nrows, Hq] (double).  bs_out may be NULL; otherwise it receives the
 * block scores [nrows, G, NB].
 */
int oracle_forward(int64_t B, int64_t T, int64_t S, int64_t Hq, int64_t Hkv,
                   int64_t d, int64_t d_idx, int64_t block, int64_t topk,
                   int dtype, double scale, const void *q_idx_rows,
                   const void *k_idx, const void *Q_rows, const void *K,
                   const void *V, const int64_t *rows, int64_t nrows,
                   int32_t *ids_out, double *O, double *lse, double *bs_out)
{
    if (Hkv <= 0 || block <= 0 || S <= 0 || nrows < 0) return -1;
    const int64_t NB = ceil_div(S, block);
    double *bs = bs_out;
    if (!bs) {
        bs = (double *)malloc(sizeof(double) * (size_t)(nrows * Hkv * NB + 1));
        if (!bs) return -2;
    }
    int rc = oracle_block_scores(B, T, S, Hkv, d_idx, block, dtype, q_idx_rows, k_idx,
                                 rows, nrows, bs);
    if (rc == 0)
        rc = oracle_select_blocks(T, S, Hkv, block, topk, bs, rows, nrows, ids_out);
    if (rc == 0)
        rc = oracle_attention(B, T, S, Hq, Hkv, d, block, topk, dtype, scale,
                              Q_rows, K, V, ids_out, rows, nrows, O, lse);
    if (!bs_out) free(bs);
    return rc;
}

/*
 * Hierarchical (coarse-to-fine) block selection, an index-cost reducer
 * ("LongCat Sparse Attention", Abstract, item (3): a coarse-to-fine scoring
 * scheme narrows the candidate set of each query, cutting the indexing
 * work).  The page names no formula; the reading taken here, for MSA's
 * max-pooled block scores, in three steps per (row, group):
 *   1. coarse: block n < cb is scored by the dot product of the index query
 *      with the block's MEAN index key, (1 / block) * sum over the block's
 *      tokens of k_idx[j] -- d_idx multiply-adds per block instead of
 *      block * d_idx;
 *   2. candidates: the kc - 1 best blocks n < cb by coarse score (larger
 *      score first, lower id on ties);
 *   3. fine: each candidate's exact block score (the max-pooled token dot
 *      product of oracle_block_scores); kept = {cb} plus the topk - 1 best
 *      candidates by fine score (same order), written ascending, -1 padded.
 * Candidates are whole blocks before the current one, so every token of a
 * candidate is causal.  With kc - 1 >= cb every earlier block is a
 * candidate and the result is oracle_select_blocks' on the exact scores.
 * Requires 1 <= topk <= kc.  ids [nrows, G, topk].
 */
int oracle_select_hierarchical(int64_t B, int64_t T, int64_t S, int64_t G,
                               int64_t d_idx, int64_t block, int64_t topk, int64_t kc,
                               int dtype, const void *q_idx_rows, const void *k_idx,
                               const int64_t *rows, int64_t nrows, int32_t *ids)
{
    if (B <= 0 || T <= 0 || S <= 0 || T > S || G <= 0 || d_idx <= 0 || block <= 0 ||
        topk <= 0 || kc < topk || nrows < 0 || (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
        return -1;
    const int64_t NB = ceil_div(S, block);
    int bad = 0;
#pragma omp parallel
    {
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)NB);
        double *mean = (double *)malloc(sizeof(double) * (size_t)d_idx);
        if (!cand || !mean) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t ri = 0; ri < nrows; ++ri) {
            if (!cand || !mean) continue;
            const int64_t r = rows[ri];
            if (r < 0 || r >= B * T) { bad = 1; continue; }
            const int64_t b = r / T, t = r % T;
            const int64_t cb = query_pos(T, S, t) / block;
            for (int64_t g = 0; g < G; ++g) {
                const int64_t q0 = (ri * G + g) * d_idx;
                int32_t *out = ids + (ri * G + g) * topk;
                /* 1. coarse scores of the blocks before the current one */
                for (int64_t n = 0; n < cb; ++n) {
                    for (int64_t ii = 0; ii < d_idx; ++ii) {
                        double sum = 0.0;
                        for (int64_t j = n * block; j < (n + 1) * block; ++j)
                            sum += widen(k_idx, dtype, (b * S + j) * d_idx + ii);
                        mean[ii] = sum / (double)block;
                    }
                    double dot = 0.0;
                    for (int64_t ii = 0; ii < d_idx; ++ii)
                        dot += widen(q_idx_rows, dtype, q0 + ii) * mean[ii];
                    cand[n].score = dot;
                    cand[n].id = n;
                }
                /* 2. the kc - 1 best by coarse score */
                qsort(cand, (size_t)cb, sizeof *cand, cand_better_first);
                const int64_t nc = (cb < kc - 1) ? cb : kc - 1;
                /* 3. exact max-pooled scores of the candidates, then the topk - 1 best */
                for (int64_t c = 0; c < nc; ++c) {
                    const int64_t n = cand[c].id;
                    double best = -INFINITY;
                    for (int64_t j = n * block; j < (n + 1) * block; ++j) {
                        double dot = 0.0;
                        for (int64_t ii = 0; ii < d_idx; ++ii)
                            dot += widen(q_idx_rows, dtype, q0 + ii) *
                                   widen(k_idx, dtype, (b * S + j) * d_idx + ii);
                        best = dot > best ? dot : best;
                    }
                    cand[c].score = best;
                }
                qsort(cand, (size_t)nc, sizeof *cand, cand_better_first);
                const int64_t take = (nc < topk - 1) ? nc : topk - 1;
                for (int64_t i = 0; i < take; ++i) out[i] = (int32_t)cand[i].id;
                qsort(out, (size_t)take, sizeof(int32_t), id_ascending);
                out[take] = (int32_t)cb;
                for (int64_t slot = take + 1; slot < topk; ++slot) out[slot] = -1;
            }
        }
        free(cand);
        free(mean);
    }
    return bad ? -2 : 0;
}

/*
 * The forward pass over a PAGED cache with per-sequence lengths (decode
 * steps of a serving batch).  The pages do not describe paging: this is the
 * same method ("MiniMax Sparse Attention", Summary, second paragraph) with
 * each sequence's keys read through a block table.
 *
 * Sequence b has L = seq_lens[b] keys; its key j < L is row j % page_size of
 * page block_table[b * max_pages + j / page_size] of each cache:
 *   k_idx_cache [num_pages, page_size, d_idx]
 *   K_cache, V_cache [num_pages, page_size, Hkv, d]
 * Its T queries (q_idx [B, T, Hkv, d_idx], Q [B, T, Hq, d]) sit at the last
 * T positions L - T + t.  Each sequence is the dense problem with S = L:
 * its keys are copied out of the pages in order, and oracle_forward runs on
 * them (a partial last block is allowed there).  Outputs:
 *   ids [B, T, Hkv, topk] int32, O [B, T, Hq, d], lse [B, T, Hq] (double).
 * A length outside [T, S] or a page id outside [0, num_pages) is an error
 * (-4); nothing is computed for any sequence then.
 */
int oracle_forward_paged(int64_t B, int64_t T, int64_t S, int64_t Hq, int64_t Hkv,
                         int64_t d, int64_t d_idx, int64_t block, int64_t topk,
                         int dtype, double scale, const int32_t *seq_lens,
                         const int32_t *block_table, int64_t page_size,
                         int64_t max_pages, int64_t num_pages, const void *q_idx,
                         const void *k_idx_cache, const void *Q, const void *K_cache,
                         const void *V_cache, int32_t *ids, double *O, double *lse)
{
    if (B <= 0 || T <= 0 || S <= 0 || page_size <= 0 || max_pages <= 0 ||
        num_pages <= 0 || max_pages * page_size < S ||
        (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
        return -1;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t L = seq_lens[b];
        if (L < T || L > S) return -4;
        for (int64_t i = 0; i < (L + page_size - 1) / page_size; ++i) {
            const int64_t pg = block_table[b * max_pages + i];
            if (pg < 0 || pg >= num_pages) return -4;
        }
    }
    const size_t esz = dtype == ORACLE_BF16 ? 2 : 4;
    const size_t ki_row = (size_t)d_idx * esz, kv_row = (size_t)Hkv * d * esz;
    char *ki = (char *)malloc(ki_row * (size_t)S);
    char *kk = (char *)malloc(kv_row * (size_t)S);
    char *vv = (char *)malloc(kv_row * (size_t)S);
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)T);
    int rc = (ki && kk && vv && rows) ? 0 : -2;
    for (int64_t t = 0; t < T && rc == 0; ++t) rows[t] = t;
    for (int64_t b = 0; b < B && rc == 0; ++b) {
        const int64_t L = seq_lens[b];
        /* the sequence's keys, densely: row j of page table entry j / page_size */
        for (int64_t j = 0; j < L; ++j) {
            const int64_t pg = block_table[b * max_pages + j / page_size];
            const int64_t src = pg * page_size + j % page_size;
            memcpy(ki + (size_t)j * ki_row, (const char *)k_idx_cache + (size_t)src * ki_row,
                   ki_row);
            memcpy(kk + (size_t)j * kv_row, (const char *)K_cache + (size_t)src * kv_row, kv_row);
            memcpy(vv + (size_t)j * kv_row, (const char *)V_cache + (size_t)src * kv_row, kv_row);
        }
        rc = oracle_forward(1, T, L, Hq, Hkv, d, d_idx, block, topk, dtype, scale,
                            (const char *)q_idx + (size_t)(b * T * Hkv * d_idx) * esz, ki,
                            (const char *)Q + (size_t)(b * T * Hq * d) * esz, kk, vv, rows, T,
                            ids + b * T * Hkv * topk, O + b * T * Hq * d, lse + b * T * Hq,
                            NULL);
    }
    free(ki);
    free(kk);
    free(vv);
    free(rows);
    return rc;
}

/* Number of OpenMP threads the oracle runs with (for reporting). */
int oracle_num_threads(void)
{
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
