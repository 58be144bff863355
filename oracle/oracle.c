/*
 * CPU oracle for the DSA sparse-attention layer stack with IndexCache reuse.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library; it is a plain,
 * slow, obviously correct restatement of what the method computes, in fp64.
 *
 * Sources (the pages describing IndexCache, arXiv 2603.12201):
 *  - "IndexCache: Accelerating Sparse Attention via Cross-Layer Index Reuse"
 *    (fugumt digest, Abstract): per query, a lightning indexer ranks the
 *    earlier tokens; core attention then covers only the k best-ranked ones.
 *  - "When the Optimizer Becomes the Bottleneck: A Close Look at IndexCache"
 *    (kualia.ai, Introduction): one indexer pass rates every earlier token
 *    of a query and the k highest-rated are kept.
 *  - "Cross-Layer Index Reuse" (knowledge note, How It Works): the anchor
 *    layer scores the visible positions and stores its k-position set; each
 *    layer after it attends sparsely over that stored set.
 *  The pages print no formula for the indexer score.  The plainest standard
 *  form is used: s[t,s] = sum_j w[t,j] * max(0, q_I[t,j] . k_I[s]), with the
 *  visible set s <= t.
 *
 * Numerics: bf16 inputs are decoded exactly (bits << 16 -> float -> double);
 * every sum is accumulated in double.  OpenMP spreads independent query rows
 * over threads; no loop is blocked, fused or reordered beyond that.
 *
 * Rows: every entry point works on a list of flattened query rows
 * r = b*Lq + i (query i of batch b sits at absolute position t = q_offset+i).
 * rows == NULL means all B*Lq rows in order.  This lets tests and the CPU
 * baseline evaluate a sample of rows of a large problem one by one.
 *
 * Return values: 0 on success, -1 on an argument error, -2 when an index
 * handed to the attention routine lies outside the visible range.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_val(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int64_t row_id(const int64_t *rows, int64_t r) { return rows ? rows[r] : r; }

int or_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the calling host thread's later oracle calls use (OpenMP's
 * per-thread setting); lets a pool of host threads run one row each. */
void or_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Lightning indexer score (Abstract of the IndexCache digest; the
 * score form is the standard one stated in the header above).
 *   qI  [B, Lq, H, dI] bf16 bits      kI [B, Lk, dI] bf16 bits
 *   w   [B, Lq, H]     float          out [n_rows, Lk] double
 * out[r][s] = sum_j w[b,i,j] * max(0, sum_c qI[b,i,j,c] * kI[b,s,c]) for
 * s <= t, and -INFINITY for t < s < Lk (positions the query cannot see).
 */
int or_indexer_scores(const uint16_t *qI, const uint16_t *kI, const float *w,
                      int B, int Lq, int Lk, int H, int dI, int q_offset,
                      const int64_t *rows, int64_t n_rows, double *out)
{
    if (B < 0 || Lq < 0 || Lk < 0 || H <= 0 || dI <= 0 || q_offset < 0)
        return -1;
    if ((int64_t)q_offset + Lq > Lk) return -1;   /* a query past the last key */
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t rid = row_id(rows, r);
        if (rid < 0 || rid >= (int64_t)B * Lq) { bad = 1; continue; }
        int64_t b = rid / Lq, i = rid % Lq;
        int64_t t = (int64_t)q_offset + i;
        const uint16_t *q = qI + ((b * Lq + i) * (int64_t)H) * dI;
        const float *wr = w + (b * Lq + i) * (int64_t)H;
        const uint16_t *kb = kI + b * (int64_t)Lk * dI;
        double *o = out + r * (int64_t)Lk;
        for (int64_t s = 0; s < Lk; ++s) {
            if (s > t) { o[s] = -INFINITY; continue; }
            double acc = 0.0;
            for (int j = 0; j < H; ++j) {
                double dot = 0.0;
                for (int c = 0; c < dI; ++c)
                    dot += bf16_val(q[(int64_t)j * dI + c]) * bf16_val(kb[s * dI + c]);
                double relu = dot > 0.0 ? dot : 0.0;
                acc += (double)wr[j] * relu;
            }
            o[s] = acc;
        }
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* Per-row top-k.  A row at position t sees n = min(t+1, Lk)           */
/* positions.  The selected set is the min(k, n) positions that come    */
/* first in the order (score descending, position ascending); it is     */
/* written in ascending position order and padded with -1.              */
/* Scores are compared as IEEE floats, so -0 and +0 are equal.          */
/* ------------------------------------------------------------------ */

typedef struct { float v; int32_t s; } or_pair;

static int pair_cmp(const void *a, const void *b)
{
    const or_pair *x = (const or_pair *)a, *y = (const or_pair *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s < y->s) ? -1 : (x->s > y->s);
}

static int int_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Sort-based top-k.  scores [n_rows, Lk] float, tpos[r] = position t of row r. */
int or_topk_sort(const float *scores, const int64_t *tpos, int64_t n_rows, int Lk, int k,
                 int32_t *idx)
{
    if (Lk < 0 || k <= 0) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t t = tpos[r];
        int32_t *o = idx + r * (int64_t)k;
        if (t < 0) { bad = 1; continue; }
        int64_t n = t + 1 < Lk ? t + 1 : Lk;
        or_pair *p = (or_pair *)malloc(sizeof(or_pair) * (size_t)(n > 0 ? n : 1));
        for (int64_t s = 0; s < n; ++s) { p[s].v = scores[r * (int64_t)Lk + s]; p[s].s = (int32_t)s; }
        qsort(p, (size_t)n, sizeof(or_pair), pair_cmp);
        int64_t m = n < k ? n : k;
        for (int64_t j = 0; j < m; ++j) o[j] = p[j].s;
        qsort(o, (size_t)m, sizeof(int32_t), int_cmp);
        for (int64_t j = m; j < k; ++j) o[j] = -1;
        free(p);
    }
    return bad ? -1 : 0;
}

/*
 * Brute-force count form of the same definition (for tiny rows; O(n^2)):
 * position s is selected iff fewer than k visible positions s' beat it,
 * where s' beats s when S[s'] > S[s], or S[s'] == S[s] and s' < s.
 */
int or_topk_count(const float *scores, const int64_t *tpos, int64_t n_rows, int Lk, int k,
                  int32_t *idx)
{
    if (Lk < 0 || k <= 0) return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t t = tpos[r];
        const float *S = scores + r * (int64_t)Lk;
        int32_t *o = idx + r * (int64_t)k;
        if (t < 0) return -1;
        int64_t n = t + 1 < Lk ? t + 1 : Lk;
        int64_t m = 0;
        for (int64_t s = 0; s < n; ++s) {
            int64_t beat = 0;
            for (int64_t s2 = 0; s2 < n; ++s2)
                if (S[s2] > S[s] || (S[s2] == S[s] && s2 < s)) ++beat;
            if (beat < k) o[m++] = (int32_t)s;
        }
        for (; m < k; ++m) o[m] = -1;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Sparse attention over the cached positions (IndexCache              */
/* digest, Abstract: core attention over k selected tokens; knowledge   */
/* note, How It Works: every later layer attends sparsely over the     */
/* stored set).  MQA: every query head reads the one K/V head.          */
/*   q [B,Lq,Hq,d]  K,V [B,Lk,d]  idx [n_rows,k], one row per requested  */
/*   query row (-1 = empty slot)                                        */
/* For row r and head h over the valid slots:                           */
/*   z_i = scale * q[r,h] . K[idx_i];  m = max z;                       */
/*   out = sum_i e^(z_i-m) V[idx_i] / sum_i e^(z_i-m)                   */
/*   lse = m + log(sum_i e^(z_i-m))                                     */
/* A row with no valid slot gives out = 0 and lse = -INFINITY.          */
/* ------------------------------------------------------------------ */

static int attend_row(const uint16_t *qrow, const uint16_t *Kb, const uint16_t *Vb,
                      const int32_t *sel, int64_t nsel, int Hq, int d, double scale,
                      int64_t t, double *o, double *lse)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)(nsel > 0 ? nsel : 1));
    int rc = 0;
    for (int h = 0; h < Hq; ++h) {
        const uint16_t *qh = qrow + (int64_t)h * d;
        double *oh = o + (int64_t)h * d;
        double m = -INFINITY;
        int64_t nvalid = 0;
        for (int64_t i = 0; i < nsel; ++i) {
            int64_t s = sel[i];
            if (s == -1) { z[i] = -INFINITY; continue; }
            if (s < 0 || s > t) { rc = -2; z[i] = -INFINITY; continue; }
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += bf16_val(qh[c]) * bf16_val(Kb[s * d + c]);
            z[i] = scale * dot;
            if (z[i] > m) m = z[i];
            ++nvalid;
        }
        for (int c = 0; c < d; ++c) oh[c] = 0.0;
        if (nvalid == 0) { if (lse) lse[h] = -INFINITY; continue; }
        double den = 0.0;
        for (int64_t i = 0; i < nsel; ++i) {
            int64_t s = sel[i];
            if (s < 0 || s > t) continue;
            double e = exp(z[i] - m);
            den += e;
            for (int c = 0; c < d; ++c) oh[c] += e * bf16_val(Vb[s * d + c]);
        }
        for (int c = 0; c < d; ++c) oh[c] /= den;
        if (lse) lse[h] = m + log(den);
    }
    free(z);
    return rc;
}

int or_sparse_attn(const uint16_t *q, const uint16_t *K, const uint16_t *V, const int32_t *idx,
                   int B, int Lq, int Lk, int Hq, int d, int k, int q_offset, double scale,
                   const int64_t *rows, int64_t n_rows, double *out, double *lse)
{
    if (B < 0 || Lq < 0 || Lk < 0 || Hq <= 0 || d <= 0 || k <= 0 || q_offset < 0) return -1;
    if ((int64_t)q_offset + Lq > Lk) return -1;   /* a query past the last key */
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t rid = row_id(rows, r);
        if (rid < 0 || rid >= (int64_t)B * Lq) { rc = rc < -1 ? rc : -1; continue; }
        int64_t b = rid / Lq, i = rid % Lq;
        int64_t t = (int64_t)q_offset + i;
        int e = attend_row(q + rid * (int64_t)Hq * d, K + b * (int64_t)Lk * d,
                           V + b * (int64_t)Lk * d, idx + r * (int64_t)k, k, Hq, d, scale, t,
                           out + r * (int64_t)Hq * d, lse ? lse + r * (int64_t)Hq : NULL);
        if (e < rc) rc = e;
    }
    return rc;
}

/* Dense causal attention: the same softmax over every visible s <= t. */
int or_dense_attn(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                  int B, int Lq, int Lk, int Hq, int d, int q_offset, double scale,
                  const int64_t *rows, int64_t n_rows, double *out, double *lse)
{
    if (B < 0 || Lq < 0 || Lk <= 0 || Hq <= 0 || d <= 0 || q_offset < 0) return -1;
    if ((int64_t)q_offset + Lq > Lk) return -1;   /* a query past the last key */
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t rid = row_id(rows, r);
        if (rid < 0 || rid >= (int64_t)B * Lq) { rc = rc < -1 ? rc : -1; continue; }
        int64_t b = rid / Lq, i = rid % Lq;
        int64_t t = (int64_t)q_offset + i;
        int32_t *all = (int32_t *)malloc(sizeof(int32_t) * (size_t)(t + 1));
        for (int64_t s = 0; s <= t; ++s) all[s] = (int32_t)s;
        int e = attend_row(q + rid * (int64_t)Hq * d, K + b * (int64_t)Lk * d,
                           V + b * (int64_t)Lk * d, all, t + 1, Hq, d, scale, t,
                           out + r * (int64_t)Hq * d, lse ? lse + r * (int64_t)Hq : NULL);
        if (e < rc) rc = e;
        free(all);
    }
    return rc;
}

/*
 * Cross-layer index overlap ("IndexCache ... Cross-Layer Index Reuse", skill
 * page, Step 1 "Analyze Index Correlation Across Layers": the top-k sets of
 * consecutive layers are compared per query position as sets; kualia.ai
 * review, "The Redundancy That Was Sitting There": in adjacent layers 70-100%
 * of the k picks coincide).
 * Row r of a and of b holds k slots; -1 is an empty slot and every other
 * value must lie in [0, Lk).  A row is read as the SET of its valid entries
 * (a repeated position counts once).  out3[3r+0] = |A & B|, out3[3r+1] = |A|,
 * out3[3r+2] = |B|.  Returns -1 on a size error, -2 on an entry outside
 * [-1, Lk) (the row's counts then ignore that entry).
 */
int or_index_overlap(const int32_t *a, const int32_t *b, int64_t n_rows, int k, int Lk,
                     int32_t *out3)
{
    if (n_rows < 0 || k < 1 || Lk < 1) return -1;
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(min : rc)
    for (int64_t r = 0; r < n_rows; ++r) {
        unsigned char *in_a = (unsigned char *)calloc((size_t)Lk, 1);
        unsigned char *in_b = (unsigned char *)calloc((size_t)Lk, 1);
        for (int s = 0; s < k; ++s) {
            int32_t x = a[r * (int64_t)k + s], y = b[r * (int64_t)k + s];
            if (x >= 0 && x < Lk) in_a[x] = 1;
            else if (x != -1) rc = rc < -2 ? rc : -2;
            if (y >= 0 && y < Lk) in_b[y] = 1;
            else if (y != -1) rc = rc < -2 ? rc : -2;
        }
        int32_t both = 0, na = 0, nb = 0;
        for (int s = 0; s < Lk; ++s) {
            na += in_a[s];
            nb += in_b[s];
            both += in_a[s] & in_b[s];
        }
        out3[3 * r] = both;
        out3[3 * r + 1] = na;
        out3[3 * r + 2] = nb;
        free(in_a);
        free(in_b);
    }
    return rc;
}
