/*
 * prr_oracle.c -- plain, slow, fp64 CPU oracle for one PRR decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check of the graft entry
 * point and the CPU-baseline leg of the bench load this library.  The product path
 * (the CUDA library under dynamic_sparse_attention_block_b200/csrc) never calls it,
 * and this file shares no code, header, table or helper with that path.
 *
 * What it computes.  The PRR pages (Predict, Reuse, and Repair: Accelerating
 * Dynamic Sparse Attention for Long-Context LLM Decoding -- abstract, method summary,
 * contribution (3) and the key-result bullet on the repair kernel) state that PRR
 * preserves correctness: repairing the missed blocks restores full top-K coverage,
 * so its output is exactly that of plain top-K dynamic sparse attention.  So the
 * oracle is that plain definition, per decode step
 * and per (sequence b, KV head):
 *   1. per-block key summary: per-channel min and max of the keys of the block
 *      (tokens < n);
 *   2. block score: Quest's channel-wise upper bound of q.k (Quest: Query-Aware
 *      Sparsity for Efficient Long-Context LLM Inference, in PRR's reference list),
 *      U_h(b) = sum_c max(q_hc*min_bc, q_hc*max_bc), computed literally for every
 *      query head h of the GQA group and summed over the group;
 *   3. true selected set S = the first min(K, nb) blocks under (score desc, index asc);
 *   4. out_h = softmax attention of q_h over exactly the tokens of the blocks in S,
 *      with scale 1/sqrt(d); lse_h = ln sum_i exp(scale*q_h.k_i);
 *   5. EMA predictor (PRR abstract: an exponential moving average of past selections):
 *      e_b <- alpha*e_b + (1-alpha)*[b in S], evaluated as alpha*e + beta*ind with
 *      beta = 1 - alpha, no fused multiply-add (build flag -ffp-contract=off);
 *      Pred_{t+1} = first min(P, nb) blocks under (e desc, index asc).
 * A second, PRR-restated path (speculate on Pred, drop Pred \ S, repair M = S \ Pred,
 * merge with online-softmax (m, l, O) statistics in ascending block order) is given
 * for the invariance pin: it must equal step 4 for every predicted set.
 *
 * Readings where the pages are silent (the pages print no formula for any step):
 * GQA heads share one selection per KV head, scored by the sum of the per-head
 * bounds; the tail block (n not a multiple of bs) is scored from its valid tokens and
 * may be selected; no forced sink or local blocks; ties go to the lower block index;
 * e starts at 0; output is fp64 here.
 *
 * bf16 values arrive as raw uint16 bit patterns and are widened exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* exact bf16 -> double: a bf16 is the top half of an IEEE binary32 */
static double bf16_val(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

/* ------------------------------------------------------------------ 1. summaries */

/* Summary of one block: min and max per channel over the block's tokens that are
 * < n.  k is one (sequence, KV head) slice, [tokens][d] bf16 bits. */
void oracle_block_summary(const uint16_t *k, int n, int d, int bs, int blk,
                          double *smin, double *smax)
{
    int t0 = blk * bs, t1 = t0 + bs;
    if (t1 > n) t1 = n;
    for (int c = 0; c < d; ++c) {
        double lo = bf16_val(k[(size_t)t0 * d + c]);
        double hi = lo;
        for (int t = t0 + 1; t < t1; ++t) {
            double x = bf16_val(k[(size_t)t * d + c]);
            if (x < lo) lo = x;
            if (x > hi) hi = x;
        }
        smin[c] = lo;
        smax[c] = hi;
    }
}

/* All ceil(n/bs) summaries of one slice; smin/smax are [nb][d]. */
void oracle_build_summaries(const uint16_t *k, int n, int d, int bs, double *smin, double *smax)
{
    int nb = ceil_div(n, bs);
    for (int b = 0; b < nb; ++b)
        oracle_block_summary(k, n, d, bs, b, smin + (size_t)b * d, smax + (size_t)b * d);
}

/* ------------------------------------------------------------------ 2. scores */

/* s_b = sum over the G query heads of sum_c max(q_hc*min_bc, q_hc*max_bc).
 * q is [G][d] (already widened to double), summaries are [nb][d]. */
void oracle_block_scores(const double *q, int G, int d, const double *smin,
                         const double *smax, int nb, double *s)
{
    for (int b = 0; b < nb; ++b) {
        double total = 0.0;
        for (int h = 0; h < G; ++h) {
            double u = 0.0;
            for (int c = 0; c < d; ++c) {
                double lo = q[h * d + c] * smin[(size_t)b * d + c];
                double hi = q[h * d + c] * smax[(size_t)b * d + c];
                u += (lo > hi) ? lo : hi;
            }
            total += u;
        }
        s[b] = total;
    }
}

/* ------------------------------------------------------------------ 3. top-K */

/* "a before b" under (value desc, index asc) */
static int ranks_before(double va, int ia, double vb, int ib)
{
    if (va != vb) return va > vb;
    return ia < ib;
}

static void sort_ascending(int32_t *x, int n)
{
    for (int i = 1; i < n; ++i) {
        int32_t key = x[i];
        int j = i - 1;
        while (j >= 0 && x[j] > key) { x[j + 1] = x[j]; --j; }
        x[j + 1] = key;
    }
}

/* The first min(K, nb) indices of v[0..nb) under (v desc, index asc), written in
 * ascending index order.  Selection by repeated scan for the best remaining entry.
 * Returns the count. */
int oracle_top_ranked(const double *v, int nb, int K, int32_t *out)
{
    int keff = K < nb ? K : nb;
    if (keff <= 0) return 0;
    unsigned char *taken = (unsigned char *)calloc((size_t)nb, 1);
    for (int r = 0; r < keff; ++r) {
        int best = -1;
        for (int b = 0; b < nb; ++b) {
            if (taken[b]) continue;
            if (best < 0 || ranks_before(v[b], b, v[best], best)) best = b;
        }
        taken[best] = 1;
        out[r] = best;
    }
    free(taken);
    sort_ascending(out, keff);
    return keff;
}

/* ------------------------------------------------------------------ selector variants
 *
 * The abstract measures PRR across "representative DSA methods", whose selectors differ
 * from the one above.  Two of them, as plain definitions (the pages print no formula;
 * readings taken):
 *  - group score as the LARGEST of the per-head bounds instead of their sum;
 *  - forced blocks: the first n_sink blocks (attention sinks) and the last n_local
 *    blocks (the local window) are always in S; the rest of the min(K, nb) budget
 *    goes to the best remaining blocks under (score desc, index asc).  When the forced
 *    blocks alone exceed the budget, sinks are taken first, lowest index first, then
 *    local blocks from the newest backwards, until the budget is full.
 * Per-query-head selection needs nothing new: each head's own bound (G = 1) and top-K. */

/* s_b = max over the G query heads of sum_c max(q_hc*min_bc, q_hc*max_bc). */
void oracle_block_scores_max(const double *q, int G, int d, const double *smin,
                             const double *smax, int nb, double *s)
{
    for (int b = 0; b < nb; ++b) {
        double best = 0.0;
        for (int h = 0; h < G; ++h) {
            double u = 0.0;
            for (int c = 0; c < d; ++c) {
                double lo = q[h * d + c] * smin[(size_t)b * d + c];
                double hi = q[h * d + c] * smax[(size_t)b * d + c];
                u += (lo > hi) ? lo : hi;
            }
            if (h == 0 || u > best) best = u;
        }
        s[b] = best;
    }
}

/* Forced sink and local blocks plus the best of the rest; ascending output; returns
 * the count (min(K, nb)). */
int oracle_top_ranked_forced(const double *v, int nb, int K, int n_sink, int n_local,
                             int32_t *out)
{
    int keff = K < nb ? K : nb;
    if (keff <= 0) return 0;
    unsigned char *taken = (unsigned char *)calloc((size_t)nb, 1);
    int cnt = 0;
    for (int b = 0; b < n_sink && b < nb && cnt < keff; ++b)
        if (!taken[b]) { taken[b] = 1; out[cnt++] = b; }
    for (int i = 0; i < n_local && cnt < keff; ++i) {
        int b = nb - 1 - i;
        if (b < 0) break;
        if (!taken[b]) { taken[b] = 1; out[cnt++] = b; }
    }
    while (cnt < keff) {
        int best = -1;
        for (int b = 0; b < nb; ++b) {
            if (taken[b]) continue;
            if (best < 0 || ranks_before(v[b], b, v[best], best)) best = b;
        }
        taken[best] = 1;
        out[cnt++] = best;
    }
    free(taken);
    sort_ascending(out, keff);
    return keff;
}

/* InfLLM-style representative-key scores (InfLLM: Training-Free Long-Context
 * Extrapolation for LLMs with an Efficient Context Memory, in PRR's reference list;
 * only its title is on the pages).  Each block is represented by r of its own tokens
 * instead of a min/max summary; which tokens is decided when the block is built (an
 * input here, rep [nb][r] offsets inside the block).  The block score is the sum over
 * the group's query heads and the representatives of q_h . k_rep:
 *   s_b = sum_h sum_j q_h . k[b*bs + min(rep[b][j], valid_b - 1)],
 * valid_b = the block's tokens below n (a representative past a ragged tail stands
 * for the block's last token).  q is [G][d] (widened), k one slice [tokens][d] bits. */
void oracle_block_scores_rep(const double *q, int G, int d, const uint16_t *k, int n, int bs,
                             const int32_t *rep, int r, int nb, double *s)
{
    for (int b = 0; b < nb; ++b) {
        int valid = n - b * bs;
        if (valid > bs) valid = bs;
        double total = 0.0;
        for (int h = 0; h < G; ++h) {
            for (int j = 0; j < r; ++j) {
                int off = rep[(size_t)b * r + j];
                if (off > valid - 1) off = valid - 1;
                if (off < 0) off = 0;
                const uint16_t *krow = k + ((size_t)b * bs + off) * d;
                for (int c = 0; c < d; ++c) total += q[h * d + c] * bf16_val(krow[c]);
            }
        }
        s[b] = total;
    }
}

/* Paged KV cache (the PagedAttention / vLLM and FlashInfer layouts in PRR's reference
 * list; only their titles are on the pages): a pool of pages [pages][Hkv][bs][d], one
 * page holding one block of bs tokens of every KV head, and per sequence a block table
 * giving the page of each block.  This gathers tokens [0, n) of KV head h of one
 * sequence (table = that sequence's row) into a contiguous [n][d] slice, on which every
 * function above applies unchanged. */
void oracle_gather_pages(const uint16_t *pool, const int32_t *table, int Hkv, int h, int n, int bs, int d,
                         uint16_t *out)
{
    for (int t = 0; t < n; ++t) {
        const uint16_t *src = pool + (((size_t)table[t / bs] * Hkv + h) * bs + t % bs) * d;
        memcpy(out + (size_t)t * d, src, sizeof(uint16_t) * d);
    }
}

/* ------------------------------------------------------------------ 5. EMA */

/* e_b <- alpha*e_b + beta*[b in S] for every b < nb, beta = 1 - alpha. */
void oracle_ema_update(double *e, int nb, const int32_t *sel, int nsel, double alpha)
{
    double beta = 1.0 - alpha;
    for (int b = 0; b < nb; ++b) {
        double ind = 0.0;
        for (int i = 0; i < nsel; ++i)
            if (sel[i] == b) ind = 1.0;
        double decayed = alpha * e[b];
        double added = beta * ind;
        e[b] = decayed + added;
    }
}

/* ------------------------------------------------------------------ 4. attention */

static double dot_q_k(const double *q, const uint16_t *krow, int d)
{
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q[c] * bf16_val(krow[c]);
    return acc;
}

/* out = softmax attention of q (one head, [d]) over exactly the tokens of the listed
 * blocks (tokens < n), scale applied to q.k; lse = ln sum exp(scale*q.k).
 * Empty list: out = 0, lse = -inf. */
void oracle_attend_blocks(const double *q, const uint16_t *k, const uint16_t *v, int n,
                          int d, int bs, const int32_t *blocks, int nblocks, double scale,
                          double *out, double *lse)
{
    double m = -INFINITY;
    for (int i = 0; i < nblocks; ++i) {
        int t0 = blocks[i] * bs, t1 = t0 + bs < n ? t0 + bs : n;
        for (int t = t0; t < t1; ++t) {
            double s = scale * dot_q_k(q, k + (size_t)t * d, d);
            if (s > m) m = s;
        }
    }
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    if (m == -INFINITY) { *lse = -INFINITY; return; }
    double l = 0.0;
    for (int i = 0; i < nblocks; ++i) {
        int t0 = blocks[i] * bs, t1 = t0 + bs < n ? t0 + bs : n;
        for (int t = t0; t < t1; ++t) {
            double p = exp(scale * dot_q_k(q, k + (size_t)t * d, d) - m);
            l += p;
            for (int c = 0; c < d; ++c) out[c] += p * bf16_val(v[(size_t)t * d + c]);
        }
    }
    for (int c = 0; c < d; ++c) out[c] /= l;
    *lse = m + log(l);
}

/* ------------------------------------------------------------------ PRR restatement */

/* Online-softmax statistics of one block for one head (speculate / repair unit):
 * m = max_i s_i, l = sum_i exp(s_i - m), O = sum_i exp(s_i - m) v_i (unnormalised). */
void oracle_block_partial(const double *q, const uint16_t *k, const uint16_t *v, int n,
                          int d, int bs, int blk, double scale, double *m, double *l,
                          double *O)
{
    int t0 = blk * bs, t1 = t0 + bs < n ? t0 + bs : n;
    double mm = -INFINITY;
    for (int t = t0; t < t1; ++t) {
        double s = scale * dot_q_k(q, k + (size_t)t * d, d);
        if (s > mm) mm = s;
    }
    double ll = 0.0;
    for (int c = 0; c < d; ++c) O[c] = 0.0;
    for (int t = t0; t < t1; ++t) {
        double p = exp(scale * dot_q_k(q, k + (size_t)t * d, d) - mm);
        ll += p;
        for (int c = 0; c < d; ++c) O[c] += p * bf16_val(v[(size_t)t * d + c]);
    }
    *m = mm;
    *l = ll;
}

/* Log-sum-exp merge of cnt partials (m_j, l_j, O_j):
 * m* = max m_j, l* = sum l_j e^(m_j - m*), out = sum O_j e^(m_j - m*) / l*,
 * lse = m* + ln l*.  Entries with m = -inf contribute nothing. */
void oracle_lse_merge(int cnt, const double *m, const double *l, const double *O, int d,
                      double *out, double *lse)
{
    double ms = -INFINITY;
    for (int j = 0; j < cnt; ++j)
        if (m[j] > ms) ms = m[j];
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    if (ms == -INFINITY) { *lse = -INFINITY; return; }
    double ls = 0.0;
    for (int j = 0; j < cnt; ++j) {
        if (m[j] == -INFINITY) continue;
        double w = exp(m[j] - ms);
        ls += l[j] * w;
        for (int c = 0; c < d; ++c) out[c] += O[(size_t)j * d + c] * w;
    }
    for (int c = 0; c < d; ++c) out[c] /= ls;
    *lse = ms + log(ls);
}

static int contains(const int32_t *x, int n, int32_t v)
{
    for (int i = 0; i < n; ++i)
        if (x[i] == v) return 1;
    return 0;
}

/* Missed set M = S \ Pred (ascending, since S is ascending) and the keep mask
 * keep[j] = [Pred_j in S] over the predicted slots.  Returns |M|. */
int oracle_missed_keep(const int32_t *sel, int nsel, const int32_t *pred, int npred,
                       int32_t *missed, uint8_t *keep)
{
    int nm = 0;
    for (int i = 0; i < nsel; ++i)
        if (!contains(pred, npred, sel[i])) missed[nm++] = sel[i];
    for (int j = 0; j < npred; ++j) keep[j] = (uint8_t)contains(sel, nsel, pred[j]);
    return nm;
}

/* PRR-restated attention for one head: speculative partials on every predicted
 * block, drop those not in S (reuse the rest), repair partials on M, merge all
 * kept and repaired partials in ascending block order. */
void oracle_prr_attend(const double *q, const uint16_t *k, const uint16_t *v, int n, int d,
                       int bs, const int32_t *sel, int nsel, const int32_t *pred, int npred,
                       double scale, double *out, double *lse)
{
    int cap = nsel + npred + 1;
    double *pm = (double *)malloc(sizeof(double) * cap);
    double *pl = (double *)malloc(sizeof(double) * cap);
    double *pO = (double *)malloc(sizeof(double) * (size_t)cap * d);
    int32_t *pb = (int32_t *)malloc(sizeof(int32_t) * cap);
    int32_t *missed = (int32_t *)malloc(sizeof(int32_t) * (nsel + 1));
    uint8_t *keep = (uint8_t *)malloc((size_t)npred + 1);
    int cnt = 0;
    /* speculate: one partial per predicted block */
    for (int j = 0; j < npred; ++j) {
        oracle_block_partial(q, k, v, n, d, bs, pred[j], scale, &pm[cnt], &pl[cnt],
                             pO + (size_t)cnt * d);
        pb[cnt++] = pred[j];
    }
    /* reuse: drop predicted blocks that are not in S */
    int nm = oracle_missed_keep(sel, nsel, pred, npred, missed, keep);
    int w = 0;
    for (int j = 0; j < cnt; ++j) {
        if (!keep[j]) continue;
        pm[w] = pm[j]; pl[w] = pl[j]; pb[w] = pb[j];
        memmove(pO + (size_t)w * d, pO + (size_t)j * d, sizeof(double) * d);
        ++w;
    }
    cnt = w;
    /* repair: one partial per missed block */
    for (int i = 0; i < nm; ++i) {
        oracle_block_partial(q, k, v, n, d, bs, missed[i], scale, &pm[cnt], &pl[cnt],
                             pO + (size_t)cnt * d);
        pb[cnt++] = missed[i];
    }
    /* order the partials by block index, then merge */
    for (int i = 1; i < cnt; ++i) {
        for (int j = i; j > 0 && pb[j - 1] > pb[j]; --j) {
            int32_t tb = pb[j]; pb[j] = pb[j - 1]; pb[j - 1] = tb;
            double tm = pm[j]; pm[j] = pm[j - 1]; pm[j - 1] = tm;
            double tl = pl[j]; pl[j] = pl[j - 1]; pl[j - 1] = tl;
            for (int c = 0; c < d; ++c) {
                double to = pO[(size_t)j * d + c];
                pO[(size_t)j * d + c] = pO[(size_t)(j - 1) * d + c];
                pO[(size_t)(j - 1) * d + c] = to;
            }
        }
    }
    oracle_lse_merge(cnt, pm, pl, pO, d, out, lse);
    free(pm); free(pl); free(pO); free(pb); free(missed); free(keep);
}

/* ------------------------------------------------------------------ one decode step */

typedef struct {
    int B, Hq, Hkv, d, bs, cap, K, P;
    double alpha, scale;
} oracle_dims;

/*
 * One decode step over every (sequence, KV head), after the caller has written the
 * new token at position seq_lens[b]-1 of k/v (layout [B][Hkv][cap][d] bf16 bits).
 * State carried between steps: summaries smin/smax [B][Hkv][maxnb][d] (maxnb =
 * ceil(cap/bs)) and ema [B][Hkv][maxnb].
 *   in : q [B][Hq][d] bits, pred [B][Hkv][P] (Pred_t, -1 beyond its count)
 *   out: sel, missed [B][Hkv][K], n_missed [B][Hkv], keep [B][Hkv][P],
 *        pred_next [B][Hkv][P], out [B][Hq][d], lse [B][Hq]
 * Slots beyond a list's count are -1 (keep 0).  The tail summary is recomputed from
 * the block's tokens.  nthreads > 1 spreads (sequence, KV head) units over OpenMP
 * threads; each unit is computed identically either way.
 */
int oracle_decode_step(const oracle_dims *D, const uint16_t *q, const uint16_t *k,
                       const uint16_t *v, const int32_t *seq_lens, const int32_t *pred,
                       double *smin, double *smax, double *ema, int32_t *sel,
                       int32_t *missed, int32_t *n_missed, uint8_t *keep,
                       int32_t *pred_next, double *out, double *lse, int nthreads)
{
    int G = D->Hq / D->Hkv, d = D->d, bs = D->bs;
    int maxnb = ceil_div(D->cap, bs);
    int units = D->B * D->Hkv;
    if (nthreads < 1) nthreads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int u = 0; u < units; ++u) {
        int b = u / D->Hkv, kvh = u % D->Hkv;
        int n = seq_lens[b];
        int nb = ceil_div(n, bs);
        const uint16_t *ku = k + (size_t)u * D->cap * d;
        const uint16_t *vu = v + (size_t)u * D->cap * d;
        double *mn = smin + (size_t)u * maxnb * d, *mx = smax + (size_t)u * maxnb * d;
        double *e = ema + (size_t)u * maxnb;
        const int32_t *pr = pred + (size_t)u * D->P;
        int32_t *su = sel + (size_t)u * D->K, *mu = missed + (size_t)u * D->K;
        uint8_t *kp = keep + (size_t)u * D->P;
        int32_t *pn = pred_next + (size_t)u * D->P;

        /* 1. summary of the block holding the new token */
        int tail = (n - 1) / bs;
        oracle_block_summary(ku, n, d, bs, tail, mn + (size_t)tail * d, mx + (size_t)tail * d);

        /* 2. scores of every block (q of the G heads of this group) */
        double *qg = (double *)malloc(sizeof(double) * G * d);
        for (int h = 0; h < G; ++h)
            for (int c = 0; c < d; ++c)
                qg[h * d + c] = bf16_val(q[((size_t)b * D->Hq + kvh * G + h) * d + c]);
        double *s = (double *)malloc(sizeof(double) * nb);
        oracle_block_scores(qg, G, d, mn, mx, nb, s);

        /* 3. true selected set, missed set, keep mask */
        for (int i = 0; i < D->K; ++i) { su[i] = -1; mu[i] = -1; }
        int nsel = oracle_top_ranked(s, nb, D->K, su);
        int npred = 0;
        while (npred < D->P && pr[npred] >= 0) ++npred;
        for (int j = 0; j < D->P; ++j) kp[j] = 0;
        n_missed[u] = oracle_missed_keep(su, nsel, pr, npred, mu, kp);

        /* 4. attention over exactly the selected tokens, per query head */
        for (int h = 0; h < G; ++h) {
            size_t row = (size_t)b * D->Hq + kvh * G + h;
            oracle_attend_blocks(qg + h * d, ku, vu, n, d, bs, su, nsel, D->scale,
                                 out + row * d, lse + row);
        }

        /* 5. EMA update with S_t, then Pred_{t+1} */
        oracle_ema_update(e, nb, su, nsel, D->alpha);
        for (int j = 0; j < D->P; ++j) pn[j] = -1;
        oracle_top_ranked(e, nb, D->P, pn);

        free(qg);
        free(s);
    }
    return nthreads;
}

/* Number of threads an OpenMP region would use (1 without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
