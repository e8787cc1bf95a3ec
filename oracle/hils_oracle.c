/*
 * hils_oracle.c -- plain, slow, fp64 CPU oracle of HiLS attention forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it. It shares no code, header, table or helper
 * with the CUDA library; its only input is plain host arrays.
 *
 * Source: "Hierarchical Sparse Attention Done Right: Toward Infinite Context
 * Modeling" (Hu et al.), cited below by section and display:
 *   [2.1]   Sec. 2.1 Naive Block Sparse Attention: chunk partition
 *           c(j) = floor(j/S), aligned left boundary
 *           l(i) = floor((i-W+1)/S) * S, candidate set C_i = {0..l(i)/S-1},
 *           token logit s_ij = q_i.k_j / sqrt(d), and the display defining
 *           the window mass Z_swa = sum_{j=l(i)..i} exp s_ij and the chunk
 *           mass Z_ic = sum_{j in T_c} exp s_ij.
 *   [3]     Sec. 3 display after Eq. (7): surrogate score
 *           s^_ic = q_i.k'_c / sqrt(d) + b'_c, selected set I_i = the K
 *           highest s^ in C_i, Z^_ic = exp s^_ic, and the partition
 *           Z^_i = sum_{c in I_i} Z^_ic + Z_swa.
 *   [3-HS]  Sec. 3 "Answering RQ2: Hierarchical softmax" display:
 *           w_ij = [exp s_ij / Z_{i,c(j)}] * [Z^_{i,c(j)} / Z^_i], with the
 *           window's chunk-level mass taken as the exact Z_swa (stated in the
 *           text right after that display).
 *   [4.1-Q] Sec. 4.1 "Low-Rank Query Calibration": the calibrated query q^
 *           enters only the surrogate score.
 *   [4.1-G] Sec. 4.1 "HiLS-Attention in GQA": per query head, normalised
 *           chunk weights; max over the heads of a group; top-K on the group
 *           score; one selected set shared by the group.
 *
 * Readings where the pages are silent (each fixed once, here):
 *   - positions are 0-based, chunk c holds tokens [cS, cS+S);
 *   - the window starts at max(l(i), 0); C_i is empty when l(i) <= 0;
 *   - b'_c is not divided by sqrt(d);
 *   - "normalised chunk weights" = softmax of s^ over C_i for that head
 *     (the window is not part of it), so the group score is
 *     a_c = max_h (s^h_c - logsumexp_{c' in C_i} s^h_c');
 *   - ties in the top-K go to the lower chunk index; if |C_i| <= K all of
 *     C_i is selected and idx is padded with -1;
 *   - idx is reported in ascending chunk order.
 *
 * Everything is evaluated literally in the log domain in double precision:
 * log Z_c and log Z_swa by log-sum-exp, log Z^_i by log-sum-exp over
 * {s^_c : c in I_i} U {log Z_swa}, and log w_ij = s_ij - log Z_{c(j)} +
 * s^_{c(j)} - log Z^_i (window tokens: s_ij - log Z^_i).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int dtype;          /* 0: float32 storage, 1: bfloat16 storage (uint16) */
    int B, Hq, Hkv, d, S, W, K;
    int q_rows;         /* query rows per (b,h) in Q / Qs (N prefill, 1 decode) */
    int kv_rows;        /* token rows per (b,g) in K / V */
    int nC;             /* landmark rows per (b,g) in Klm / bias */
    const int32_t *head_map;    /* [Hq] query head -> kv head */
    const void *Q, *Qs, *Kc, *V, *Klm;  /* Qs may be NULL: use Q */
    const float *bias;
} oracle_problem;

/* score modes */
#define ORACLE_SCORE_LANDMARK 0   /* s^ = q^.k'/sqrt(d) + b'          [3] */
#define ORACLE_SCORE_EXACT    1   /* s^ := log Z_ic (exact chunk mass) [2.1] */

static double ld(const oracle_problem *p, const void *base, int64_t e) {
    if (p->dtype == 0) return (double)((const float *)base)[e];
    uint32_t u = ((uint32_t)((const uint16_t *)base)[e]) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* floor division for possibly negative numerators */
static int64_t floordiv(int64_t a, int64_t b) {
    int64_t q = a / b;
    if ((a % b != 0) && ((a < 0) != (b < 0))) q -= 1;
    return q;
}

static double logsumexp(const double *x, int64_t n) {
    if (n <= 0) return -INFINITY;
    double m = -INFINITY;
    for (int64_t k = 0; k < n; ++k) if (x[k] > m) m = x[k];
    if (m == -INFINITY) return -INFINITY;
    double s = 0.0;
    for (int64_t k = 0; k < n; ++k) s += exp(x[k] - m);
    return m + log(s);
}

/* q_i . k_j / sqrt(d) for query row (b,h,r) and token (b,g,j)      [2.1] */
static double token_logit(const oracle_problem *p, const void *qbase, int b,
                          int h, int r, int g, int64_t j) {
    int64_t qo = (((int64_t)b * p->Hq + h) * p->q_rows + r) * p->d;
    int64_t ko = (((int64_t)b * p->Hkv + g) * p->kv_rows + j) * p->d;
    double acc = 0.0;
    for (int k = 0; k < p->d; ++k)
        acc += ld(p, qbase, qo + k) * ld(p, p->Kc, ko + k);
    return acc / sqrt((double)p->d);
}

/* s^_ic = q^_i . k'_c / sqrt(d) + b'_c                           [3][4.1-Q] */
static double surrogate_score(const oracle_problem *p, int b, int h, int r,
                              int g, int c) {
    const void *qb = p->Qs ? p->Qs : p->Q;
    int64_t qo = (((int64_t)b * p->Hq + h) * p->q_rows + r) * p->d;
    int64_t ko = (((int64_t)b * p->Hkv + g) * p->nC + c) * p->d;
    double acc = 0.0;
    for (int k = 0; k < p->d; ++k)
        acc += ld(p, qb, qo + k) * ld(p, p->Klm, ko + k);
    return acc / sqrt((double)p->d) +
           (double)p->bias[((int64_t)b * p->Hkv + g) * p->nC + c];
}

/* log Z_ic = log sum_{j in T_c} exp s_ij                           [2.1] */
static double exact_log_mass(const oracle_problem *p, int b, int h, int r,
                             int g, int c, double *tmp) {
    for (int t = 0; t < p->S; ++t)
        tmp[t] = token_logit(p, p->Q, b, h, r, g, (int64_t)c * p->S + t);
    return logsumexp(tmp, p->S);
}

typedef struct { double a; int c; } cand;

static int cand_cmp(const void *x, const void *y) {
    const cand *u = (const cand *)x, *v = (const cand *)y;
    if (u->a > v->a) return -1;   /* descending group score */
    if (u->a < v->a) return 1;
    return (u->c < v->c) ? -1 : (u->c > v->c);   /* ties: lower index first */
}

static int int_cmp(const void *x, const void *y) {
    int u = *(const int *)x, v = *(const int *)y;
    return (u > v) - (u < v);
}

/*
 * One (b, g, i) row for all G query heads of kv group g.
 *   heads[G]     query heads of the group, ascending
 *   imposed_idx  NULL, or K chunk indices (ascending, -1 padded) to use
 *                instead of the selection (scores are still computed)
 * Outputs: O[G*d], idx[K], shat_sel[G*K] (s^ of the selected chunks, in idx
 * order; NAN for padding), gap (a_(K) - a_(K+1) or +inf), akth (a_(K), the
 * lowest selected group score, -inf if none), lse[G].
 * Returns 0, or -1 on allocation failure / bad imposed index.
 */
static int oracle_one(const oracle_problem *p, int b, int g, int64_t i, int r,
                      const int *heads, int G, int score_mode,
                      const int32_t *imposed_idx, double *O, int32_t *idx,
                      double *shat_sel, double *gap, double *akth,
                      double *lse) {
    const int S = p->S, d = p->d, K = p->K;
    /* [2.1] aligned window and candidate set */
    int64_t lq = floordiv(i - p->W + 1, S);
    int64_t l = lq * S;
    int64_t w0 = l > 0 ? l : 0;
    int64_t nc = lq > 0 ? lq : 0;
    if (nc > p->nC) return -1;

    double *shat = (double *)malloc(sizeof(double) * (size_t)(G * nc + 1));
    cand *cs = (cand *)malloc(sizeof(cand) * (size_t)(nc + 1));
    double *tmp = (double *)malloc(sizeof(double) * (size_t)(S + 1));
    int ntok_max = K * S + (int)(i - w0 + 1);
    double *e = (double *)malloc(sizeof(double) * (size_t)ntok_max);
    int64_t *tj = (int64_t *)malloc(sizeof(int64_t) * (size_t)ntok_max);
    int *sel = (int *)malloc(sizeof(int) * (size_t)(K + 1));
    if (!shat || !cs || !tmp || !e || !tj || !sel) {
        free(shat); free(cs); free(tmp); free(e); free(tj); free(sel);
        return -1;
    }

    /* [3] / [2.1] chunk scores for every head of the group */
    for (int hh = 0; hh < G; ++hh)
        for (int64_t c = 0; c < nc; ++c)
            shat[hh * nc + c] =
                (score_mode == ORACLE_SCORE_EXACT)
                    ? exact_log_mass(p, b, heads[hh], r, g, (int)c, tmp)
                    : surrogate_score(p, b, heads[hh], r, g, (int)c);

    /* [4.1-G] per-head normaliser over C_i, then the group score */
    for (int hh = 0; hh < G; ++hh) lse[hh] = logsumexp(shat + hh * nc, nc);
    for (int64_t c = 0; c < nc; ++c) {
        double a = -INFINITY;
        for (int hh = 0; hh < G; ++hh) {
            double v = shat[hh * nc + c] - lse[hh];
            if (v > a) a = v;
        }
        cs[c].a = a;
        cs[c].c = (int)c;
    }

    /* [3] top-K by rank; ties to the lower chunk index */
    qsort(cs, (size_t)nc, sizeof(cand), cand_cmp);
    int nsel = (int)(nc < K ? nc : K);
    *gap = (nc > K) ? cs[K - 1].a - cs[K].a : INFINITY;
    *akth = nsel > 0 ? cs[nsel - 1].a : -INFINITY;
    if (imposed_idx) {
        nsel = 0;
        for (int k = 0; k < K; ++k) {
            int c = imposed_idx[k];
            if (c < 0) continue;
            if (c >= nc) { nsel = -1; break; }
            sel[nsel++] = c;
        }
        if (nsel < 0) {
            free(shat); free(cs); free(tmp); free(e); free(tj); free(sel);
            return -1;
        }
    } else {
        for (int k = 0; k < nsel; ++k) sel[k] = cs[k].c;
    }
    qsort(sel, (size_t)nsel, sizeof(int), int_cmp);
    for (int k = 0; k < K; ++k) idx[k] = k < nsel ? sel[k] : -1;

    /* [3-HS] hierarchical softmax per head */
    for (int hh = 0; hh < G; ++hh) {
        int h = heads[hh];
        for (int k = 0; k < K; ++k)
            shat_sel[hh * K + k] = k < nsel ? shat[hh * nc + sel[k]] : NAN;

        int nt = 0;
        /* window tokens: log w = s_ij - log Z^_i (mass Z_swa cancels) */
        int64_t nwin = i - w0 + 1;
        for (int64_t j = w0; j <= i; ++j) {
            e[nt] = token_logit(p, p->Q, b, h, r, g, j);
            tj[nt++] = j;
        }
        double log_zswa = logsumexp(e, nwin);
        /* log Z^_i = log( sum_{c in I} exp s^_c + Z_swa )              [3] */
        double *terms = (double *)malloc(sizeof(double) * (size_t)(nsel + 1));
        if (!terms) {
            free(shat); free(cs); free(tmp); free(e); free(tj); free(sel);
            return -1;
        }
        for (int k = 0; k < nsel; ++k) terms[k] = shat[hh * nc + sel[k]];
        terms[nsel] = log_zswa;
        double log_zhat = logsumexp(terms, nsel + 1);
        free(terms);
        for (int t = 0; t < nt; ++t) e[t] -= log_zhat;
        /* chunk tokens: log w = s_ij - log Z_c + s^_c - log Z^_i */
        for (int k = 0; k < nsel; ++k) {
            int c = sel[k];
            int t0 = nt;
            for (int t = 0; t < S; ++t) {
                int64_t j = (int64_t)c * S + t;
                e[nt] = token_logit(p, p->Q, b, h, r, g, j);
                tj[nt++] = j;
            }
            double log_zc = logsumexp(e + t0, S);
            for (int t = t0; t < nt; ++t)
                e[t] = e[t] - log_zc + shat[hh * nc + c] - log_zhat;
        }
        /* o_i = sum_j w_ij v_j */
        for (int k = 0; k < d; ++k) O[hh * d + k] = 0.0;
        for (int t = 0; t < nt; ++t) {
            double w = exp(e[t]);
            int64_t vo = (((int64_t)b * p->Hkv + g) * p->kv_rows + tj[t]) * d;
            for (int k = 0; k < d; ++k) O[hh * d + k] += w * ld(p, p->V, vo + k);
        }
    }
    free(shat); free(cs); free(tmp); free(e); free(tj); free(sel);
    return 0;
}

/*
 * Evaluate nrows (b, g, i, r) rows: b batch, g kv head, i query position,
 * r row of Q holding that query. Outputs are row-major per row:
 *   O [nrows, G, d]  idx [nrows, K]  shat_sel [nrows, G, K]  gap [nrows]
 *   akth [nrows]  lse [nrows, G]
 * imposed_idx: NULL or [nrows, K]. Returns 0, or the count of failed rows.
 */
int oracle_rows(const oracle_problem *p, int64_t nrows, const int32_t *rb,
                const int32_t *rg, const int64_t *ri, const int32_t *rr,
                int score_mode, const int32_t *imposed_idx, double *O,
                int32_t *idx, double *shat_sel, double *gap, double *akth,
                double *lse, int nthreads) {
    int G = p->Hq / p->Hkv;
    int fails = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : fails)
    for (int64_t n = 0; n < nrows; ++n) {
        int heads[256];
        int cnt = 0;
        for (int h = 0; h < p->Hq && cnt < 256; ++h)
            if (p->head_map[h] == rg[n]) heads[cnt++] = h;
        if (cnt != G) { fails++; continue; }
        int rc = oracle_one(p, rb[n], rg[n], ri[n], rr[n], heads, G,
                            score_mode,
                            imposed_idx ? imposed_idx + n * p->K : NULL,
                            O + n * (int64_t)G * p->d, idx + n * p->K,
                            shat_sel + n * (int64_t)G * p->K, gap + n,
                            akth + n, lse + n * G);
        if (rc) fails++;
    }
    return fails;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
