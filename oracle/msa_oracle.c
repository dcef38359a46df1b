/*
 * MSA oracle: a plain, slow, fp64 CPU statement of MiniMax Sparse Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is built into liboracle_msa.so and is
 * called by the tests, by the smoke check and by the CPU-baseline leg of the
 * benchmark.  The product library never includes, links or calls it, and it
 * shares no code, header or table with the CUDA path.
 *
 * What it computes follows "MiniMax wird duenn: M3-Attention anhand eines
 * einzigen Diagramms entschluesselt" (atlascloud.ai), section 1 "Was das
 * Diagramm zeigt", and Figure 1:
 *
 *   Step 1, index branch ("Schritt 1: Index-Branch"):
 *     - each GQA group has one index query; the index key K_idx is a small
 *       per-token vector;                              -> oracle_token_scores
 *     - token scores Q_idx . K_idx^T are reduced to one score per fixed-size
 *       block by taking the block maximum ("Block Max Pool");
 *                                                      -> oracle_block_scores
 *     - TopK keeps the k best blocks for this layer and this group, giving a
 *       short list of block indices (I1, I2).          -> oracle_topk
 *   Step 2, sparse branch ("Schritt 2: Sparse-Branch"):
 *     - every query head of the group uses the group's single list (Q1/Q2/Q3
 *       use I1, Q4/Q5/Q6 use I2, i.e. contiguous grouping), and ordinary
 *       softmax attention runs over only the selected blocks of the full,
 *       uncompressed K and V.                          -> oracle_attention_row
 *   The "MiniMax M3模型发布细节公开" digest (traeai.com), highlight 1, says the
 *   same: real, uncompressed KV with block-level top-K selection.
 *
 * The page's formulas did not survive extraction, so these readings are taken
 * (each is the plainest one the prose supports):
 *   - index score = raw dot product, no scale, no activation;
 *   - a block's score is the max over its causally visible tokens (j <= pos);
 *     a partly visible block is eligible;
 *   - top-k order: higher score first, then lower block id; when fewer than k
 *     blocks are valid, all are taken and the list is padded with -1;
 *   - index-K head for group g is g mod n_idx_k_heads (1 shared head, or one
 *     per KV group);
 *   - softmax scale is a parameter (1/sqrt(head_dim) in every workload);
 *   - the query at position pos sees keys 0..pos (its own K/V included);
 *   - optional forced blocks (off unless force_sink_local is set): the page's
 *     section 2, third point, guesses that an attention sink stands in for the
 *     dropped sliding window; when asked for, block 0 (the sink) and the block
 *     holding pos (the local block) rank above every score, between
 *     themselves by id, and are reported with the score +inf.
 *
 * Layouts (all contiguous, element type f32 or bf16 given by `dtype`):
 *   q      [B, Tq, Hq,  D]       q_idx [B, Tq, G,   di]
 *   k, v   [B, Hkv, Lmax, D]     k_idx [B, Hik, Lmax, di]
 *   ids    [B, Tq, G, k] int32   o [B, Tq, Hq, D] f64   lse [B, Tq, Hq] f64
 * Query position: decode (q_len == 1 and prefill == 0) pos = L_b - 1;
 * prefill pos = q_start + t.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int batch, n_q_heads, n_kv_heads, n_idx_k_heads;
    int head_dim, idx_dim, block_size, top_k;
    int q_len, q_start, max_seq_len;
    int dtype;   /* 0: float32, 1: bfloat16 (raw 16-bit patterns) */
    int dense;   /* 1: select every causally valid block (plain GQA) */
    int prefill; /* 1: pos = q_start + t; 0: pos = seq_len - 1 */
    int force_sink_local; /* 1: block 0 and the query's own block are always selected */
    double softmax_scale;
} oracle_params;

/* One stored element as a double.  bf16 is the top half of an IEEE float. */
static double elem(const void *base, long long i, int dtype)
{
    if (dtype == 0) {
        return (double)((const float *)base)[i];
    } else {
        uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
}

static int n_groups(const oracle_params *p) { return p->n_kv_heads; }

/* Step 1a: s_j = q_idx[b,t,g,:] . k_idx[b, g mod Hik, j, :] for j = 0..pos. */
void oracle_token_scores(const oracle_params *p, const void *q_idx, const void *k_idx,
                         int b, int t, int g, int pos, double *s_out)
{
    const int di = p->idx_dim, G = n_groups(p), hik = g % p->n_idx_k_heads;
    const long long qoff = (((long long)b * p->q_len + t) * G + g) * di;
    const long long koff = ((long long)b * p->n_idx_k_heads + hik) * p->max_seq_len * (long long)di;
    for (int j = 0; j <= pos; ++j) {
        double acc = 0.0;
        for (int d = 0; d < di; ++d)
            acc += elem(q_idx, qoff + d, p->dtype) * elem(k_idx, koff + (long long)j * di + d, p->dtype);
        s_out[j] = acc;
    }
}

/* Step 1b: block max pool over the causally visible tokens of each block.
 * Returns the number of valid blocks, floor(pos / Bk) + 1. */
int oracle_block_scores(const oracle_params *p, const double *s, int pos, double *S_out)
{
    const int bk = p->block_size, nb = pos / bk + 1;
    for (int n = 0; n < nb; ++n) {
        int lo = n * bk, hi = (n + 1) * bk;
        if (hi > pos + 1) hi = pos + 1;
        double m = s[lo];
        for (int j = lo + 1; j < hi; ++j)
            if (s[j] > m) m = s[j];
        S_out[n] = m;
    }
    return nb;
}

typedef struct { double score; int id; } scored_block;

/* Total order of the selection: higher score first, ties to the lower id. */
static int by_score_then_id(const void *a, const void *b)
{
    const scored_block *x = (const scored_block *)a, *y = (const scored_block *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

/* Step 1c: TopK.  Writes k ids (padded with -1) and their scores (padded with
 * -inf), in selection order.  kth / kth_next receive the k-th and (k+1)-th
 * scores of the full ranking (NaN when they do not exist); the tests use
 * them to recognise near-ties, where fp32 and fp64 may legitimately differ. */
void oracle_topk(const oracle_params *p, const double *S, int nb, int *ids_out,
                 double *scores_out, double *kth, double *kth_next)
{
    const int k = p->top_k;
    scored_block *all = (scored_block *)malloc(sizeof(scored_block) * (size_t)(nb > 0 ? nb : 1));
    for (int n = 0; n < nb; ++n) {
        all[n].score = S[n];
        all[n].id = n;
        /* forced blocks: the sink (0) and the query's own block, the last valid one */
        if (p->force_sink_local && (n == 0 || n == nb - 1)) all[n].score = INFINITY;
    }
    qsort(all, (size_t)nb, sizeof(scored_block), by_score_then_id);
    for (int i = 0; i < k; ++i) {
        ids_out[i] = i < nb ? all[i].id : -1;
        if (scores_out) scores_out[i] = i < nb ? all[i].score : -INFINITY;
    }
    if (kth) *kth = (k <= nb) ? all[k - 1].score : NAN;
    if (kth_next) *kth_next = (k + 1 <= nb) ? all[k].score : NAN;
    free(all);
}

/* Step 2 for one query head h: exact softmax attention over the keys of the
 * listed blocks that are visible (j <= pos).  ids entries of -1 are skipped.
 * o_out[D], *lse_out = log of the softmax normaliser of the scaled logits.
 * If w_out is given it receives the weight of every key 0..pos (zero for
 * keys outside the listed blocks). Returns the number of keys attended. */
int oracle_attention_row(const oracle_params *p, const void *q, const void *k, const void *v,
                         int b, int t, int h, int pos, const int *ids, int n_ids,
                         double *o_out, double *lse_out, double *w_out)
{
    const int D = p->head_dim, bk = p->block_size;
    const int r = p->n_q_heads / p->n_kv_heads, kvh = h / r;
    const long long qoff = (((long long)b * p->q_len + t) * p->n_q_heads + h) * D;
    const long long kvoff = ((long long)b * p->n_kv_heads + kvh) * p->max_seq_len * (long long)D;

    int cap = 0;
    for (int i = 0; i < n_ids; ++i) if (ids[i] >= 0) cap += bk;
    int *keys = (int *)malloc(sizeof(int) * (size_t)(cap > 0 ? cap : 1));
    double *z = (double *)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
    int nk = 0;
    for (int i = 0; i < n_ids; ++i) {
        if (ids[i] < 0) continue;
        for (int j = ids[i] * bk; j < (ids[i] + 1) * bk && j <= pos; ++j) keys[nk++] = j;
    }
    double m = -INFINITY;
    for (int a = 0; a < nk; ++a) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += elem(q, qoff + d, p->dtype) * elem(k, kvoff + (long long)keys[a] * D + d, p->dtype);
        z[a] = p->softmax_scale * acc;
        if (z[a] > m) m = z[a];
    }
    double denom = 0.0;
    for (int a = 0; a < nk; ++a) { z[a] = exp(z[a] - m); denom += z[a]; }
    for (int d = 0; d < D; ++d) o_out[d] = 0.0;
    if (w_out) for (int j = 0; j <= pos; ++j) w_out[j] = 0.0;
    for (int a = 0; a < nk; ++a) {
        double w = z[a] / denom;
        if (w_out) w_out[keys[a]] = w;
        for (int d = 0; d < D; ++d)
            o_out[d] += w * elem(v, kvoff + (long long)keys[a] * D + d, p->dtype);
    }
    *lse_out = nk > 0 ? m + log(denom) : -INFINITY;
    free(keys);
    free(z);
    return nk;
}

static int query_pos(const oracle_params *p, const int *seq_lens, int b, int t)
{
    return p->prefill ? p->q_start + t : seq_lens[b] - 1;
}

/* Steps 1 and 2 for a set of (b, t) query rows.  rows[2*i], rows[2*i+1] =
 * (b, t).  For each row and group: ids/top scores/kth/kth_next as in
 * oracle_topk (packed [n_rows, G, k] and [n_rows, G]); for each row and
 * query head: o [n_rows, Hq, D], lse [n_rows, Hq].
 * If ids_in is non-NULL the selection is not computed: the given ids
 * ([n_rows, G, k]) drive Step 2 (used to re-run a near-tie row with another
 * implementation's choice).  With with_attention == 0 only Step 1 runs and
 * o / lse are left untouched. */
void oracle_msa_rows(const oracle_params *p, const int *seq_lens,
                     const void *q, const void *q_idx, const void *k, const void *v,
                     const void *k_idx, int n_rows, const int *rows, const int *ids_in,
                     int *ids_out, double *top_scores_out, double *kth_out,
                     double *kth_next_out, double *o_out, double *lse_out, int with_attention)
{
    const int G = n_groups(p), K = p->top_k, r = p->n_q_heads / p->n_kv_heads;
    const int D = p->head_dim;
#pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_rows * G; ++it) {
        const int i = it / G, g = it % G;
        const int b = rows[2 * i], t = rows[2 * i + 1];
        const int pos = query_pos(p, seq_lens, b, t);
        int *ids = ids_out + ((long long)i * G + g) * K;
        if (ids_in) {
            memcpy(ids, ids_in + ((long long)i * G + g) * K, sizeof(int) * (size_t)K);
            if (kth_out) kth_out[i * G + g] = NAN;
            if (kth_next_out) kth_next_out[i * G + g] = NAN;
        } else {
            const int nb = pos / p->block_size + 1;
            double *s = (double *)malloc(sizeof(double) * (size_t)(pos + 1));
            double *S = (double *)malloc(sizeof(double) * (size_t)nb);
            oracle_token_scores(p, q_idx, k_idx, b, t, g, pos, s);
            oracle_block_scores(p, s, pos, S);
            oracle_topk(p, S, nb, ids, top_scores_out ? top_scores_out + ((long long)i * G + g) * K : NULL,
                        kth_out ? kth_out + i * G + g : NULL,
                        kth_next_out ? kth_next_out + i * G + g : NULL);
            free(s);
            free(S);
        }
        if (!with_attention) continue;
        int *attend = ids;
        int n_attend = K;
        int *all = NULL;
        if (p->dense) {
            n_attend = pos / p->block_size + 1;
            all = (int *)malloc(sizeof(int) * (size_t)n_attend);
            for (int n = 0; n < n_attend; ++n) all[n] = n;
            attend = all;
        }
        for (int hh = 0; hh < r; ++hh) {
            const int h = g * r + hh;
            oracle_attention_row(p, q, k, v, b, t, h, pos, attend, n_attend,
                                 o_out + ((long long)i * p->n_q_heads + h) * D,
                                 lse_out + (long long)i * p->n_q_heads + h, NULL);
        }
        free(all);
    }
}
