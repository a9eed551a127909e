/*
 * scope_oracle.c -- plain, slow, fp64 CPU oracle of the SCOPE per-layer hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path links, loads or
 * calls this file; only the tests, the package's smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or constant with the CUDA path.
 *
 * Source of the method: "SCOPE: Subspace Clustering with Online Per-Head Top-K
 * Estimation for Sparse Video Attention" (arXiv 2608.12780) -- its abstract, and the
 * pith.science review page, whose fields "key_machinery" (Eqs. 6 and 9),
 * "major_comments" (Eq. 3 k-means, Eq. 7 hybrid Top-p/fixed Top-k, Eq. 8 base counts,
 * Eq. 10 top-up, Eq. 27 product-code identity, Cq=300, Cm=333, alpha=0.1) and
 * "forward_implications" (attention over the original keys/values) restate the
 * equations.  Where those pages leave a step open, the reading taken is written beside
 * the code that takes it.
 *
 * Every function works on ONE (batch, head) slice; heads are independent in SCOPE.
 * All arithmetic is IEEE binary64 on the exact values of the float32 inputs (bf16 and
 * fp32 inputs are both passed as float32 holding the input's values).  Sums run in
 * the order written, one rounding per multiply and per add (build with
 * -ffp-contract=off); parallel loops only split independent outputs.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Squared Euclidean distance over dm channels, channel order, fp64. */
static double sqdist(const float *x, const double *mu, int dm)
{
    double acc = 0.0;
    for (int i = 0; i < dm; ++i) {
        double diff = (double)x[i] - mu[i];
        acc = acc + diff * diff;
    }
    return acc;
}

/*
 * k-means by Lloyd's iteration (the paper's Eq. 3: per subspace, centroids minimise
 * the Euclidean reconstruction error).  One problem = the channels [ch0, ch0+dm) of
 * the N rows of X (row stride ld floats).  Queries use all d channels; keys run this
 * once per 3D-RoPE subspace (temporal, height, width channel ranges).
 *
 * Readings (the pages are silent on these):
 *  - initial centroids are the rows init_idx[0..C) (seeded, distinct), or init_cent;
 *  - one iteration = assign every row to its nearest centroid, then move every
 *    non-empty centroid to the mean of its members; an empty centroid keeps its value;
 *  - ties in the assignment go to the lowest centroid index;
 *  - the outputs are the last iteration's assignments and the centroids of the last
 *    update, so each centroid is exactly the mean of its output members;
 *  - means are the member sums, accumulated in increasing row order, divided by the
 *    member count.
 * Optional logs: margin[j] = min over iterations of (d2 - d1)/d2 for row j (d1, d2 the
 * best and second-best squared distances); obj_assign[it] / obj_update[it] = total
 * squared error after the assignment / after the update of iteration it.
 */
int oracle_kmeans(const float *X, int64_t N, int64_t ld, int ch0, int dm, int C,
                  const int32_t *init_idx, const double *init_cent, int iters,
                  double *cent, uint16_t *assign, int32_t *sizes,
                  double *margin, double *obj_assign, double *obj_update)
{
    if (N <= 0 || dm <= 0 || C <= 0 || C > 65535 || iters < 1)
        return 1;
    if (init_cent) {
        memcpy(cent, init_cent, sizeof(double) * (size_t)C * dm);
    } else {
        for (int c = 0; c < C; ++c) {
            int64_t r = init_idx[c];
            if (r < 0 || r >= N)
                return 2;
            for (int i = 0; i < dm; ++i)
                cent[(size_t)c * dm + i] = (double)X[r * ld + ch0 + i];
        }
    }
    double *sums = (double *)malloc(sizeof(double) * (size_t)C * dm);
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)C);
    if (!sums || !cnt) {
        free(sums);
        free(cnt);
        return 3;
    }
    if (margin)
        for (int64_t j = 0; j < N; ++j)
            margin[j] = INFINITY;

    for (int it = 0; it < iters; ++it) {
        /* assignment step */
        #pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < N; ++j) {
            const float *x = X + j * ld + ch0;
            int best = 0;
            double d1 = sqdist(x, cent, dm), d2 = INFINITY;
            for (int c = 1; c < C; ++c) {
                double dd = sqdist(x, cent + (size_t)c * dm, dm);
                if (dd < d1) {
                    d2 = d1;
                    d1 = dd;
                    best = c;
                } else if (dd < d2) {
                    d2 = dd;
                }
            }
            assign[j] = (uint16_t)best;
            if (margin) {
                double m = (d2 > 0.0 && d2 < INFINITY) ? (d2 - d1) / d2 : (C == 1 ? INFINITY : 0.0);
                if (m < margin[j])
                    margin[j] = m;
            }
        }
        if (obj_assign) {
            double J = 0.0;
            for (int64_t j = 0; j < N; ++j)
                J = J + sqdist(X + j * ld + ch0, cent + (size_t)assign[j] * dm, dm);
            obj_assign[it] = J;
        }
        /* update step: member means, rows in increasing order */
        memset(sums, 0, sizeof(double) * (size_t)C * dm);
        memset(cnt, 0, sizeof(int64_t) * (size_t)C);
        for (int64_t j = 0; j < N; ++j) {
            int c = assign[j];
            const float *x = X + j * ld + ch0;
            double *s = sums + (size_t)c * dm;
            cnt[c] += 1;
            for (int i = 0; i < dm; ++i)
                s[i] = s[i] + (double)x[i];
        }
        for (int c = 0; c < C; ++c)
            if (cnt[c] > 0)
                for (int i = 0; i < dm; ++i)
                    cent[(size_t)c * dm + i] = sums[(size_t)c * dm + i] / (double)cnt[c];
        if (obj_update) {
            double J = 0.0;
            for (int64_t j = 0; j < N; ++j)
                J = J + sqdist(X + j * ld + ch0, cent + (size_t)assign[j] * dm, dm);
            obj_update[it] = J;
        }
    }
    for (int c = 0; c < C; ++c)
        sizes[c] = (int32_t)cnt[c];
    free(sums);
    free(cnt);
    return 0;
}

/*
 * Lookup tables and proxy logits (Eq. 6).  For query cluster c with centroid qc
 * (d values) and the key centroids kc ([Cm, d], subspace m's centroid z stored in m's
 * channel range of row z):
 *     P^m[c, z] = sum_{i in m} qc[i] * kc[z, i]            (channel order)
 *     s_j       = (1/sqrt(d)) * ((P^T[z^T_j] + P^H[z^H_j]) + P^W[z^W_j])
 * 1/sqrt(d) is the binary64 value 1.0/sqrt((double)d).  Writes s[0..N).
 */
static void proxy_scores(const double *qc, const double *kc, const uint16_t *codes, int64_t N,
                         int d, const int bounds[4], int Cm, double *lut, double *s)
{
    for (int m = 0; m < 3; ++m)
        for (int z = 0; z < Cm; ++z) {
            double acc = 0.0;
            for (int i = bounds[m]; i < bounds[m + 1]; ++i)
                acc = acc + qc[i] * kc[(size_t)z * d + i];
            lut[(size_t)m * Cm + z] = acc;
        }
    const double inv = 1.0 / sqrt((double)d);
    const uint16_t *zt = codes, *zh = codes + N, *zw = codes + 2 * N;
    for (int64_t j = 0; j < N; ++j)
        s[j] = inv * ((lut[zt[j]] + lut[(size_t)Cm + zh[j]]) + lut[(size_t)2 * Cm + zw[j]]);
}

/* Ranking of keys inside one query cluster: proxy logit descending, key index
 * ascending on equal logits (keys sharing a code triple have equal logits, so the
 * index tie-break is part of the definition). */
typedef struct {
    double s;
    int64_t j;
} ranked_key;

static int cmp_ranked(const void *pa, const void *pb)
{
    const ranked_key *a = (const ranked_key *)pa, *b = (const ranked_key *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static void rank_keys(const double *s, int64_t N, ranked_key *order)
{
    for (int64_t j = 0; j < N; ++j) {
        order[j].s = s[j];
        order[j].j = j;
    }
    qsort(order, (size_t)N, sizeof(ranked_key), cmp_ranked);
}

/* Fixed Top-k minimum.  Reading: alpha is a fraction of the key count N,
 * k_fix = ceil(alpha * N) in binary64, clamped to [0, N]. */
int64_t oracle_kfix(double alpha, int64_t N)
{
    double v = ceil(alpha * (double)N);
    if (v < 0.0) return 0;
    if (v > (double)N) return N;
    return (int64_t)v;
}

/*
 * Selection for one head: Eqs. (6)-(10).
 *   Eq. 7 (hybrid Top-p / fixed Top-k), reading: with w_j = exp(s_j - max_j s_j) and
 *     Z = sum_j w_j (index order), p_c is the smallest r such that the first r keys
 *     of the ranking hold mass >= rho * Z (mass accumulated in ranking order);
 *     rho = 1 means p_c = N exactly.
 *   Eq. 8: b_c = max(p_c, k_fix) -- the union of two prefixes of one ranking.
 *   Eq. 9: k_head = ceil( sum_c n_c b_c / sum_c n_c ), exact integer arithmetic.
 *   Eq. 10: r_c = max(b_c, k_head): only clusters below k_head take extra keys, the
 *     next ones in their ranking.  S_c = the first r_c keys of the ranking.
 *   khead_off != 0 (the review page's ablation, significance: the online k_head
 *     disabled): k_head is still computed and reported, r_c = b_c.
 * Outputs: p, b, r [Cq]; *khead; mask [Cq, ceil(N/32)] (bit j%32 of word j/32 set iff
 * key j is in S_c); optional scores [Cq, N]; optional topp_margin [Cq]
 * = min over r in {p_c - 1, p_c} of |mass_r - rho Z| / Z (the decision's closeness to
 * a tie; +inf when rho = 1).
 */
int oracle_select(const double *qcent, const int32_t *qsizes, const double *kcent,
                  const uint16_t *codes, int64_t N, int d, int dt, int dh, int dw, int Cq, int Cm,
                  double rho, double alpha, double *scores, int32_t *p_out, int32_t *b_out,
                  int32_t *khead_out, int32_t *r_out, uint32_t *mask, double *topp_margin,
                  int khead_off)
{
    if (dt + dh + dw != d || N <= 0 || Cq <= 0 || Cm <= 0 || !(rho > 0.0 && rho <= 1.0)
        || !(alpha >= 0.0 && alpha <= 1.0))
        return 1;
    const int bounds[4] = {0, dt, dt + dh, d};
    const int64_t kfix = oracle_kfix(alpha, N);
    const int64_t nw = (N + 31) / 32;
    int failed = 0;

    #pragma omp parallel
    {
        double *lut = (double *)malloc(sizeof(double) * 3 * (size_t)Cm);
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        ranked_key *order = (ranked_key *)malloc(sizeof(ranked_key) * (size_t)N);
        if (!lut || !s || !order) {
            #pragma omp atomic write
            failed = 1;
        }
        #pragma omp for schedule(dynamic, 1)
        for (int c = 0; c < Cq; ++c) {
            if (failed) continue;
            proxy_scores(qcent + (size_t)c * d, kcent, codes, N, d, bounds, Cm, lut, s);
            if (scores)
                memcpy(scores + (size_t)c * N, s, sizeof(double) * (size_t)N);
            rank_keys(s, N, order);
            const double smax = order[0].s;
            double Z = 0.0;
            for (int64_t j = 0; j < N; ++j)
                Z = Z + exp(s[j] - smax);
            int64_t p = N;
            double margin = INFINITY;
            if (rho < 1.0) {
                const double target = rho * Z;
                double cum = 0.0, prev = 0.0;
                for (int64_t r = 1; r <= N; ++r) {
                    prev = cum;
                    cum = cum + exp(order[r - 1].s - smax);
                    if (cum >= target) {
                        p = r;
                        break;
                    }
                }
                double m1 = fabs(cum - target) / Z, m0 = fabs(prev - target) / Z;
                margin = m1 < m0 ? m1 : m0;
            }
            p_out[c] = (int32_t)p;
            b_out[c] = (int32_t)(p > kfix ? p : kfix);
            if (topp_margin)
                topp_margin[c] = margin;
        }
        free(lut);
        free(s);
        free(order);
    }
    if (failed)
        return 3;

    /* Eq. 9 */
    int64_t num = 0, den = 0;
    for (int c = 0; c < Cq; ++c) {
        num += (int64_t)qsizes[c] * (int64_t)b_out[c];
        den += (int64_t)qsizes[c];
    }
    if (den <= 0)
        return 4;
    const int64_t khead = (num + den - 1) / den;
    *khead_out = (int32_t)khead;

    /* Eq. 10 and the selected sets */
    #pragma omp parallel
    {
        double *lut = (double *)malloc(sizeof(double) * 3 * (size_t)Cm);
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        ranked_key *order = (ranked_key *)malloc(sizeof(ranked_key) * (size_t)N);
        #pragma omp for schedule(dynamic, 1)
        for (int c = 0; c < Cq; ++c) {
            if (!lut || !s || !order) continue;
            int64_t r = (b_out[c] < khead && !khead_off) ? khead : b_out[c];
            r_out[c] = (int32_t)r;
            proxy_scores(qcent + (size_t)c * d, kcent, codes, N, d, bounds, Cm, lut, s);
            rank_keys(s, N, order);
            uint32_t *row = mask + (size_t)c * nw;
            memset(row, 0, sizeof(uint32_t) * (size_t)nw);
            for (int64_t t = 0; t < r; ++t) {
                int64_t j = order[t].j;
                row[j >> 5] |= 1u << (j & 31);
            }
        }
        free(lut);
        free(s);
        free(order);
    }
    return 0;
}

/*
 * Sparse attention over the selected ORIGINAL keys and values: for query row i in
 * cluster c = qassign[i],
 *     o_i = sum_{j in S_c} softmax_j(q_i . k_j / sqrt(d)) v_j,
 * softmax with the maximum subtracted, all in binary64.  rows lists the query rows to
 * compute (NULL = all N, in order); O is [nrows, d].
 */
int oracle_attention(const float *Q, const float *K, const float *V, int64_t N, int d,
                     const uint16_t *qassign, const uint32_t *mask, int Cq,
                     const int64_t *rows, int64_t nrows, double *O)
{
    const int64_t nw = (N + 31) / 32;
    const double inv = 1.0 / sqrt((double)d);
    int failed = 0;
    #pragma omp parallel
    {
        double *l = (double *)malloc(sizeof(double) * (size_t)N);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < nrows; ++t) {
            if (!l || !acc) {
                failed = 1;
                continue;
            }
            const int64_t i = rows ? rows[t] : t;
            const int c = qassign[i];
            if (c >= Cq) {
                failed = 2;
                continue;
            }
            const uint32_t *row = mask + (size_t)c * nw;
            const float *q = Q + i * d;
            double mx = -INFINITY;
            for (int64_t j = 0; j < N; ++j) {
                if (!((row[j >> 5] >> (j & 31)) & 1u)) continue;
                const float *k = K + j * d;
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot = dot + (double)q[e] * (double)k[e];
                l[j] = dot * inv;
                if (l[j] > mx) mx = l[j];
            }
            double den = 0.0;
            for (int e = 0; e < d; ++e) acc[e] = 0.0;
            for (int64_t j = 0; j < N; ++j) {
                if (!((row[j >> 5] >> (j & 31)) & 1u)) continue;
                const double p = exp(l[j] - mx);
                den = den + p;
                const float *v = V + j * d;
                for (int e = 0; e < d; ++e)
                    acc[e] = acc[e] + p * (double)v[e];
            }
            for (int e = 0; e < d; ++e)
                O[t * d + e] = den > 0.0 ? acc[e] / den : 0.0;
        }
        free(l);
        free(acc);
    }
    return failed;
}
