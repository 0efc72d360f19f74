/*
 * pisa_oracle.c -- the oracle: a plain, slow, fp64 CPU restatement of PISA
 * pyramid Top-K block selection and block-sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header, table or helper with the CUDA library.
 *
 * Source of every definition: the page "论文精读 · Block Sparse Attention with
 * Log-Linear Complexity (PISA)" (qqtang-code.github.io, Paper-Reading-Collection),
 * cited below as "close reading", by section and equation number.
 *
 *   Eq.(1)  flat block score  s_{t,i} = q_t . kbar_i / sqrt(d)        (§02)
 *   Eq.(2)  attention over the union T_t of the selected blocks       (§02)
 *   Eq.(3)  M_{l+1} = ceil(M_l / g_l), g_0 = C, g_l = g for l >= 1    (§04 4.1)
 *   Eq.(4)  kbar^{(l+1)}_i = mean of the child summaries kbar^{(l)}    (§04 4.1)
 *   Eq.(5)  A^{(L)} = {root}; I = SelectK(A, s); A^{(l-1)} = U Ch(I)  (§04 4.2)
 *   Eq.(6)  |I| <= K, |A| <= g K                                      (§04 4.2)
 *   Eq.(7)  s^{(l)}_{t,i} = log sum_{r in Ch(i)} exp(q . kbar^{(l-1)}_r / sqrt d)
 *           (at l = 1 the children are the raw keys)                  (§04 4.3)
 *   Eq.(8)-(9) the Taylor view of Eq.(7) and its ablations: PISA-1 scores a
 *           node by the mean of its children's logits, PISA-2 by that mean
 *           plus half their variance                                  (§04 4.3)
 *   Eq.(11) GQA: the node score is the SUM over the group's query heads
 *           of each head's Eq.(7) score; the group shares the choice  (§04 4.4)
 *   §5.3    forced blocks: the first, previous and current leaf and their
 *           ancestor paths are always kept; nodes on the current path may
 *           hold future keys, so they are kept but never ranked; attention
 *           masks future tokens inside a block.
 *   §04 ("close reading" 03, last paragraph): a level whose candidate count
 *           is already <= K keeps every candidate without scoring.
 *
 * Readings taken where the page is silent (each also listed in the design notes):
 *   - indices are 0-based: node i at level l covers tokens
 *     [i*C*g^(l-1), min((i+1)*C*g^(l-1), N)); level 1 = leaves, level L = root;
 *   - a node/leaf with fewer children than g (ragged tail) averages and scores
 *     over the children that exist;
 *   - causal: a node is a candidate only if its first token is <= t; the nodes
 *     that contain t (the current path) are always kept unranked when causal,
 *     because their summaries include future keys;
 *   - forced_mask: bit0 first leaf, bit1 previous leaf, bit2 current leaf;
 *     forced nodes consume the K budget (|I| <= K);
 *   - the "<= K keep all" test counts candidates after causal exclusion;
 *   - ranking key: score descending, then node index ascending (ties go to
 *     the lower index);
 *   - the output row is the selected leaves sorted ascending, padded with -1;
 *   - natural log, 1/sqrt(d) inside the exponent.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_MAX_LEVELS 64

/* ---- geometry: Eq.(3) ------------------------------------------------------ */

/* Fills M[1..L] (nodes per level) and off[1..L] (row offset of each level in
 * the concatenated pyramid); returns L (0 when N <= 0). */
int oracle_geometry(int64_t N, int C, int g, int64_t *M, int64_t *off)
{
    if (N <= 0 || C <= 0 || g < 2) return 0;
    int L = 1;
    M[1] = (N + C - 1) / C;
    off[1] = 0;
    while (M[L] > 1) {
        if (L + 1 >= OR_MAX_LEVELS) return -1;
        M[L + 1] = (M[L] + g - 1) / g;
        off[L + 1] = off[L] + M[L];
        ++L;
    }
    return L;
}

int64_t oracle_total_nodes(int64_t N, int C, int g)
{
    int64_t M[OR_MAX_LEVELS + 1], off[OR_MAX_LEVELS + 1];
    int L = oracle_geometry(N, C, g, M, off);
    if (L <= 0) return 0;
    return off[L] + M[L];
}

/* tokens covered by one node at level l: C * g^(l-1) */
static int64_t span_of(int l, int C, int g)
{
    int64_t s = C;
    for (int k = 1; k < l; ++k) s *= g;
    return s;
}

/* ---- pyramid: Eq.(3)-(4) --------------------------------------------------- */

/* K: [BH, k_rows, d], the first N rows of each head are the keys.
 * P: [BH, total_nodes(N_layout), d]; levels are laid out for N_layout >= N,
 * and only nodes that hold at least one of the first N tokens are written. */
void oracle_build_pyramid(int BH, int64_t N, int64_t N_layout, int64_t k_rows,
                          int d, int C, int g, const double *K, double *P)
{
    int64_t M[OR_MAX_LEVELS + 1], off[OR_MAX_LEVELS + 1];
    int L = oracle_geometry(N_layout, C, g, M, off);
    if (L <= 0 || N <= 0) return;
    int64_t total = off[L] + M[L];
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const double *Kh = K + (int64_t)bh * k_rows * d;
        double *Ph = P + (int64_t)bh * total * d;
        /* level 1: mean of the raw keys of each leaf (Eq.4 with l = 0) */
        int64_t M1 = (N + C - 1) / C;
        for (int64_t i = 0; i < M1; ++i) {
            int64_t lo = i * C, hi = lo + C < N ? lo + C : N;
            double *dst = Ph + (off[1] + i) * d;
            for (int e = 0; e < d; ++e) dst[e] = 0.0;
            for (int64_t j = lo; j < hi; ++j)
                for (int e = 0; e < d; ++e) dst[e] += Kh[j * d + e];
            for (int e = 0; e < d; ++e) dst[e] /= (double)(hi - lo);
        }
        /* level l+1: mean of the existing children summaries (Eq.4, l >= 1) */
        int64_t Ml = M1;
        for (int l = 1; l < L; ++l) {
            int64_t Mn = (Ml + g - 1) / g;
            for (int64_t j = 0; j < Mn; ++j) {
                int64_t r0 = j * g, r1 = r0 + g < Ml ? r0 + g : Ml;
                double *dst = Ph + (off[l + 1] + j) * d;
                for (int e = 0; e < d; ++e) dst[e] = 0.0;
                for (int64_t r = r0; r < r1; ++r)
                    for (int e = 0; e < d; ++e) dst[e] += Ph[(off[l] + r) * d + e];
                for (int e = 0; e < d; ++e) dst[e] /= (double)(r1 - r0);
            }
            Ml = Mn;
        }
    }
}

/* Decode upkeep (close reading §5.3, "decode cache"): after key row n has been
 * written, refresh the leaf holding n and every ancestor, each as the mean of
 * what exists at length n+1. P is laid out for N_layout. */
void oracle_pyramid_append(int64_t n, int64_t N_layout, int d, int C, int g,
                           const double *Kh, double *P)
{
    int64_t M[OR_MAX_LEVELS + 1], off[OR_MAX_LEVELS + 1];
    int L = oracle_geometry(N_layout, C, g, M, off);
    if (L <= 0 || n < 0 || n >= N_layout) return;
    int64_t len = n + 1;
    int64_t leaf = n / C;
    {
        int64_t lo = leaf * C, hi = len;
        double *dst = P + (off[1] + leaf) * d;
        for (int e = 0; e < d; ++e) dst[e] = 0.0;
        for (int64_t j = lo; j < hi; ++j)
            for (int e = 0; e < d; ++e) dst[e] += Kh[j * d + e];
        for (int e = 0; e < d; ++e) dst[e] /= (double)(hi - lo);
    }
    int64_t node = leaf;
    for (int l = 1; l < L; ++l) {
        int64_t parent = node / g;
        int64_t exist_l = (len + span_of(l, C, g) - 1) / span_of(l, C, g); /* nodes of level l holding data */
        int64_t r0 = parent * g, r1 = r0 + g < exist_l ? r0 + g : exist_l;
        double *dst = P + (off[l + 1] + parent) * d;
        for (int e = 0; e < d; ++e) dst[e] = 0.0;
        for (int64_t r = r0; r < r1; ++r)
            for (int e = 0; e < d; ++e) dst[e] += P[(off[l] + r) * d + e];
        for (int e = 0; e < d; ++e) dst[e] /= (double)(r1 - r0);
        node = parent;
    }
}

/* ---- scores: Eq.(7) and Eq.(11) ------------------------------------------- */

static double dot(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int e = 0; e < d; ++e) s += a[e] * b[e];
    return s;
}

/* log sum_r exp(z_r), max-subtracted */
static double lse(const double *z, int n)
{
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) if (z[i] > m) m = z[i];
    if (m == -INFINITY) return -INFINITY;
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += exp(z[i] - m);
    return m + log(s);
}

/* Score of a node from its children's logits z[0..n) (n >= 1):
 *   variant 0: Eq.(7), log sum_r exp(z_r);
 *   variant 1 (PISA-1, Eq.8 truncated): the mean logit;
 *   variant 2 (PISA-2, Eq.9): the mean logit plus half the population variance
 *   of the logits (the second cumulant; divide by n). */
static double child_score(const double *z, int n, int variant)
{
    if (variant == 0) return lse(z, n);
    double m = 0.0;
    for (int i = 0; i < n; ++i) m += z[i];
    m /= (double)n;
    if (variant == 1) return m;
    double v = 0.0;
    for (int i = 0; i < n; ++i) v += (z[i] - m) * (z[i] - m);
    return m + 0.5 * v / (double)n;
}

typedef struct {
    int G, d, C, g;
    int64_t N;              /* keys that exist */
    const int64_t *M, *off; /* layout geometry */
    const double *Kh, *P;   /* raw keys [>=N, d]; pyramid */
    int variant;            /* node score: 0 Eq.(7) LSE, 1 PISA-1, 2 PISA-2 */
} ctx_t;

/* Eq.(7) (or its PISA-1 / PISA-2 ablation) for one query head, summed over
 * the G heads of the group (Eq.11).
 * Level l >= 2: over the existing child summaries at level l-1.
 * Level 1: over the raw keys of the leaf (the exact leaf LSE for Eq.7). */
static double node_score(const ctx_t *c, const double *qg, int l, int64_t i)
{
    double inv = 1.0 / sqrt((double)c->d);
    double total = 0.0;
    if (l == 1) {
        int64_t lo = i * c->C, hi = lo + c->C < c->N ? lo + c->C : c->N;
        int n = (int)(hi - lo);
        double *z = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
        for (int h = 0; h < c->G; ++h) {
            for (int64_t j = lo; j < hi; ++j)
                z[j - lo] = dot(qg + (int64_t)h * c->d, c->Kh + j * c->d, c->d) * inv;
            total += n > 0 ? child_score(z, n, c->variant) : -INFINITY;
        }
        free(z);
    } else {
        int64_t span_child = span_of(l - 1, c->C, c->g);
        int64_t exist_child = (c->N + span_child - 1) / span_child;
        int64_t r0 = i * c->g, r1 = r0 + c->g < exist_child ? r0 + c->g : exist_child;
        double z[64];
        for (int h = 0; h < c->G; ++h) {
            int n = 0;
            for (int64_t r = r0; r < r1; ++r)
                z[n++] = dot(qg + (int64_t)h * c->d, c->P + (c->off[l - 1] + r) * c->d, c->d) * inv;
            total += n > 0 ? child_score(z, n, c->variant) : -INFINITY;
        }
    }
    return total;
}

double oracle_node_score(int G, int64_t N, int64_t N_layout, int d, int C, int g,
                         const double *Kh, const double *P, const double *qg,
                         int level, int64_t node, int variant)
{
    int64_t M[OR_MAX_LEVELS + 1], off[OR_MAX_LEVELS + 1];
    int L = oracle_geometry(N_layout, C, g, M, off);
    if (L <= 0 || level < 1 || level > L) return NAN;
    ctx_t c = {G, d, C, g, N, M, off, Kh, P, variant};
    return node_score(&c, qg, level, node);
}

/* ---- Top-K with the forced / causal rules ---------------------------------- */

typedef struct { double s; int64_t i; } ranked_t;

/* score descending, then index ascending */
static int cmp_ranked(const void *a, const void *b)
{
    const ranked_t *x = (const ranked_t *)a, *y = (const ranked_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int cmp_i64(const void *a, const void *b)
{
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x < y) ? -1 : (x > y);
}

/* forced leaves of query t (close reading §5.3): first, previous, current;
 * under causal masking the current leaf is always kept (it holds t). */
static int forced_leaves(int64_t t, int C, int causal, int mask, int64_t *f)
{
    int64_t c = t / C;
    int n = 0;
    if (mask & 1) f[n++] = 0;
    if ((mask & 2) && c >= 1) f[n++] = c - 1;
    if ((mask & 4) || causal) f[n++] = c;
    return n;
}

static int is_forced_node(int64_t node, int l, int g, const int64_t *f, int nf)
{
    for (int k = 0; k < nf; ++k) {
        int64_t a = f[k];
        for (int s = 1; s < l; ++s) a /= g;
        if (a == node) return 1;
    }
    return 0;
}

/* Keep forced candidates, then fill the remaining budget with the best-ranked
 * other candidates. Returns |I|; *gap gets the margin between the last kept
 * and first dropped ranked score (INFINITY when no ranked decision was made). */
static int select_k(const int64_t *cand, int ncand, const double *score,
                    const int *forced, int K, int64_t *I, double *gap, int *nscored)
{
    *gap = INFINITY;
    *nscored = 0;
    if (ncand <= K) {
        for (int k = 0; k < ncand; ++k) I[k] = cand[k];
        return ncand;
    }
    int nI = 0, nr = 0;
    ranked_t *rest = (ranked_t *)malloc(sizeof(ranked_t) * ncand);
    for (int k = 0; k < ncand; ++k) {
        if (forced[k]) I[nI++] = cand[k];
        else { rest[nr].s = score[k]; rest[nr].i = cand[k]; ++nr; }
    }
    int r = K - nI;
    if (r > 0) {
        qsort(rest, nr, sizeof(ranked_t), cmp_ranked);
        for (int k = 0; k < r && k < nr; ++k) I[nI++] = rest[k].i;
        if (r < nr) *gap = rest[r - 1].s - rest[r].s;
        *nscored = nr;
    }
    free(rest);
    return nI;
}

/* ---- the pyramid walk: Eq.(5)-(7), (11), forced/causal rules ---------------- */

/* One selection for query position t of one KV head.
 * qg: [G, d] the group's query rows at t. idx: [K] sorted ascending, -1 padded.
 * counts (optional): [OR_MAX_LEVELS][2] = (|candidates|, |scored|) at level l
 * stored at row l-1. */
static void walk_one(const ctx_t *c, int L, int K, int causal, int mask,
                     int64_t t, const double *qg, int32_t *idx, double *gap_out,
                     int32_t *counts)
{
    int64_t f[3];
    int nf = forced_leaves(t, c->C, causal, mask, f);
    int cap = c->g * K + 1;
    if (cap < 2) cap = 2;
    int64_t *A = (int64_t *)malloc(sizeof(int64_t) * cap);
    int64_t *cand = (int64_t *)malloc(sizeof(int64_t) * cap);
    int64_t *I = (int64_t *)malloc(sizeof(int64_t) * cap);
    double *score = (double *)malloc(sizeof(double) * cap);
    int *forced = (int *)malloc(sizeof(int) * cap);
    int nA = 1, nI = 0;
    A[0] = 0;
    double gmin = INFINITY;
    for (int l = L; l >= 1; --l) {
        int64_t span = span_of(l, c->C, c->g);
        int ncand = 0;
        for (int k = 0; k < nA; ++k) {
            int64_t i = A[k];
            if (i * span >= c->N) continue;            /* node holds no key */
            if (causal && i * span > t) continue;      /* wholly in the future */
            cand[ncand++] = i;
        }
        for (int k = 0; k < ncand; ++k) {
            forced[k] = is_forced_node(cand[k], l, c->g, f, nf);
            score[k] = 0.0;
        }
        if (ncand > K) {
            int nforced = 0;
            for (int k = 0; k < ncand; ++k) nforced += forced[k];
            if (K - nforced > 0)
                for (int k = 0; k < ncand; ++k)
                    if (!forced[k]) score[k] = node_score(c, qg, l, cand[k]);
        }
        double gap;
        int nscored;
        nI = select_k(cand, ncand, score, forced, K, I, &gap, &nscored);
        if (gap < gmin) gmin = gap;
        if (counts) { counts[(l - 1) * 2] = ncand; counts[(l - 1) * 2 + 1] = nscored; }
        if (l > 1) {
            nA = 0;
            int64_t span_child = span_of(l - 1, c->C, c->g);
            for (int k = 0; k < nI; ++k)
                for (int r = 0; r < c->g; ++r) {
                    int64_t ch = I[k] * c->g + r;
                    if (ch < c->M[l - 1] && ch * span_child < c->N) A[nA++] = ch;
                }
            qsort(A, nA, sizeof(int64_t), cmp_i64);
        }
    }
    qsort(I, nI, sizeof(int64_t), cmp_i64);
    for (int k = 0; k < K; ++k) idx[k] = k < nI ? (int32_t)I[k] : -1;
    if (gap_out) *gap_out = gmin;
    free(A); free(cand); free(I); free(score); free(forced);
}

/* Selection for n_units query rows of one KV head.
 * N: keys that exist; N_layout: length the pyramid P was laid out for.
 * Kh: [>=N, d]; P: [total_nodes(N_layout), d]; t: [n]; Qrows: [n, G, d].
 * idx: [n, K]; gap: [n] or NULL; counts: [n, OR_MAX_LEVELS, 2] or NULL. */
void oracle_select_rows(int G, int64_t N, int64_t N_layout, int d, int C, int K, int g,
                        int causal, int forced_mask, const double *Kh, const double *P,
                        int64_t n, const int64_t *t, const double *Qrows,
                        int32_t *idx, double *gap, int32_t *counts, int variant)
{
    int64_t M[OR_MAX_LEVELS + 1], off[OR_MAX_LEVELS + 1];
    int L = oracle_geometry(N_layout, C, g, M, off);
    if (L <= 0) return;
    ctx_t c = {G, d, C, g, N, M, off, Kh, P, variant};
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t u = 0; u < n; ++u)
        walk_one(&c, L, K, causal, forced_mask, t[u], Qrows + u * G * d, idx + u * K,
                 gap ? gap + u : NULL,
                 counts ? counts + u * OR_MAX_LEVELS * 2 : NULL);
}

/* ---- flat selections over every leaf (comparisons / recall reference) ------ */

/* kind 0: Eq.(1) mean-summary dot (BSA); kind 1: exact LSE over the leaf's raw
 * keys, scored for every eligible leaf (exhaustive reference). Same forced and
 * causal rules and the same ranking key as the walk. */
static void flat_one(const ctx_t *c, int kind, int K, int causal, int mask, int64_t t,
                     const double *qg, int32_t *idx, double *gap_out)
{
    int64_t f[3];
    int nf = forced_leaves(t, c->C, causal, mask, f);
    int64_t M1 = (c->N + c->C - 1) / c->C;
    int64_t *cand = (int64_t *)malloc(sizeof(int64_t) * (M1 + 1));
    double *score = (double *)malloc(sizeof(double) * (M1 + 1));
    int *forced = (int *)malloc(sizeof(int) * (M1 + 1));
    int64_t *I = (int64_t *)malloc(sizeof(int64_t) * (K + 1));
    int ncand = 0;
    for (int64_t i = 0; i < M1; ++i) {
        if (causal && i * c->C > t) break;
        cand[ncand++] = i;
    }
    double inv = 1.0 / sqrt((double)c->d);
    for (int k = 0; k < ncand; ++k) {
        forced[k] = is_forced_node(cand[k], 1, c->g, f, nf);
        score[k] = 0.0;
        if (ncand > K && !forced[k]) {
            if (kind == 0) {
                for (int h = 0; h < c->G; ++h)
                    score[k] += dot(qg + (int64_t)h * c->d, c->P + (c->off[1] + cand[k]) * c->d, c->d) * inv;
            } else {
                score[k] = node_score(c, qg, 1, cand[k]);
            }
        }
    }
    double gap;
    int nscored;
    int nI = select_k(cand, ncand, score, forced, K, I, &gap, &nscored);
    qsort(I, nI, sizeof(int64_t), cmp_i64);
    for (int k = 0; k < K; ++k) idx[k] = k < nI ? (int32_t)I[k] : -1;
    if (gap_out) *gap_out = gap;
    free(cand); free(score); free(forced); free(I);
}

void oracle_flat_rows(int kind, int G, int64_t N, int64_t N_layout, int d, int C, int K, int g,
                      int causal, int forced_mask, const double *Kh, const double *P,
                      int64_t n, const int64_t *t, const double *Qrows,
                      int32_t *idx, double *gap)
{
    int64_t M[OR_MAX_LEVELS + 1], off[OR_MAX_LEVELS + 1];
    int L = oracle_geometry(N_layout, C, g, M, off);
    if (L <= 0) return;
    ctx_t c = {G, d, C, g, N, M, off, Kh, P, 0};
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t u = 0; u < n; ++u)
        flat_one(&c, kind, K, causal, forced_mask, t[u], Qrows + u * G * d, idx + u * K,
                 gap ? gap + u : NULL);
}

/* ---- attention over the selected blocks: Eq.(2) with the causal mask ------- */

/* For each of n query rows: o = sum_{j in T, j<=t if causal} softmax_j(q.k_j/sqrt d) v_j,
 * T = union of the leaves listed in idx[u, :] (entries < 0 ignored).
 * Kh, Vh: [>=N, d]; Qrows: [n, d]; O: [n, d] (zeros when no key is visible).
 * lse_out (optional, [n]): log sum_j exp(q.k_j/sqrt d) over the visible keys. */
void oracle_attn_rows(int64_t N, int d, int C, int K, int causal,
                      const double *Kh, const double *Vh, int64_t n, const int64_t *t,
                      const double *Qrows, const int32_t *idx, double *O, double *lse_out)
{
    double inv = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t u = 0; u < n; ++u) {
        const double *q = Qrows + u * d;
        double *o = O + u * d;
        int64_t tt = t[u];
        double m = -INFINITY;
        for (int k = 0; k < K; ++k) {
            int32_t b = idx[u * K + k];
            if (b < 0) continue;
            for (int64_t j = (int64_t)b * C; j < (int64_t)(b + 1) * C && j < N; ++j) {
                if (causal && j > tt) break;
                double z = dot(q, Kh + j * d, d) * inv;
                if (z > m) m = z;
            }
        }
        for (int e = 0; e < d; ++e) o[e] = 0.0;
        if (m == -INFINITY) { if (lse_out) lse_out[u] = -INFINITY; continue; }
        double den = 0.0;
        for (int k = 0; k < K; ++k) {
            int32_t b = idx[u * K + k];
            if (b < 0) continue;
            for (int64_t j = (int64_t)b * C; j < (int64_t)(b + 1) * C && j < N; ++j) {
                if (causal && j > tt) break;
                double w = exp(dot(q, Kh + j * d, d) * inv - m);
                den += w;
                for (int e = 0; e < d; ++e) o[e] += w * Vh[j * d + e];
            }
        }
        for (int e = 0; e < d; ++e) o[e] /= den;
        if (lse_out) lse_out[u] = m + log(den);
    }
}
