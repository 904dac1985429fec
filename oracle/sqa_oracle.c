/*
 * sqa_oracle.c -- plain, slow fp64 CPU oracle for Sparse Query Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the reference that the CUDA path is
 * checked against.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may build, load or call it.  It shares no code, header,
 * table or helper with the CUDA library, and the library never calls it.
 *
 * What it computes (Sparse Query Attention, "SQAT-m" model card, sections
 * "Architecture details" and "Model size difference"; arXiv 2510.01817
 * abstract; GQA summary, section "The idea"):
 *   H_q query heads, fewer than the H-way head split, attend over H_kv key/value
 *   heads.  The query heads are split into H_kv contiguous groups of
 *   g = H_q / H_kv heads, and every head of a group reads the same K and V head:
 *   kv(h) = floor(h / g).  With H_q = H_kv this is multi-head attention, with
 *   H_kv = 1 it is multi-query attention (GQA summary, "The notation").
 *
 * The pages print no formula, so the plain scaled dot-product softmax reading
 * is used, all in fp64, on inputs that are already fp64:
 *   s_ij  = scale * sum_d Q[b,i,h,d] K[b,j,kv(h),d]      (masked to -inf when
 *           causal and j > i; the diagonal j == i is visible)
 *   lse_i = m_i + ln sum_j exp(s_ij - m_i),  m_i = max_j s_ij    (natural log)
 *   P_ij  = exp(s_ij - lse_i)
 *   O_i   = sum_j P_ij V[b,j,kv(h),:]
 * and, for an upstream gradient dO of the loss L = sum dO * O,
 *   D_i   = sum_d dO_i,d O_i,d
 *   dP_ij = sum_d dO_i,d V_j,d
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij K_j
 *   dK_j  = scale * sum_{h in group} sum_i dS_ij Q_i
 *   dV_j  = sum_{h in group} sum_i P_ij dO_i
 *
 * Layouts: q, out, dout, dq are [B][N][H_q][dh]; k, v, dk, dv are
 * [B][N][H_kv][dh]; lse is [B][H_q][N].  Every loop follows the definition:
 * no tiling, no online softmax, no fusion.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *dout;
    int64_t B, N, Hq, Hkv, dh;
    int causal;
    double scale;
} problem;

static int64_t group_size(const problem *p) { return p->Hq / p->Hkv; }

/* Contiguous grouping: query head h reads key/value head floor(h / g). */
static int64_t kv_head(const problem *p, int64_t h) { return h / group_size(p); }

static const double *q_row(const problem *p, int64_t b, int64_t i, int64_t h) {
    return p->q + ((b * p->N + i) * p->Hq + h) * p->dh;
}
static const double *do_row(const problem *p, int64_t b, int64_t i, int64_t h) {
    return p->dout + ((b * p->N + i) * p->Hq + h) * p->dh;
}
static const double *k_row(const problem *p, int64_t b, int64_t j, int64_t kvh) {
    return p->k + ((b * p->N + j) * p->Hkv + kvh) * p->dh;
}
static const double *v_row(const problem *p, int64_t b, int64_t j, int64_t kvh) {
    return p->v + ((b * p->N + j) * p->Hkv + kvh) * p->dh;
}

static int visible(const problem *p, int64_t i, int64_t j) { return !p->causal || j <= i; }

static double dot(const double *a, const double *b, int64_t n) {
    double acc = 0.0;
    for (int64_t d = 0; d < n; ++d) acc += a[d] * b[d];
    return acc;
}

static int check(const problem *p) {
    if (p->B < 1 || p->N < 1 || p->Hq < 1 || p->Hkv < 1 || p->dh < 1) return 1;
    if (p->Hq % p->Hkv != 0) return 2;
    if (!(p->scale > 0.0) || !isfinite(p->scale)) return 3;
    return 0;
}

/* Scores of query row (b, i, h) against every key; masked keys get -inf.
 * Returns the row's log-sum-exp. */
static double score_row(const problem *p, int64_t b, int64_t h, int64_t i, double *s) {
    const double *qi = q_row(p, b, i, h);
    const int64_t kvh = kv_head(p, h);
    double m = -INFINITY;
    for (int64_t j = 0; j < p->N; ++j) {
        s[j] = visible(p, i, j) ? p->scale * dot(qi, k_row(p, b, j, kvh), p->dh) : -INFINITY;
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j < p->N; ++j)
        if (s[j] != -INFINITY) sum += exp(s[j] - m);
    return m + log(sum);
}

/* O_i (dh values) of row (b, i, h) from its scores and log-sum-exp. */
static void output_row(const problem *p, int64_t b, int64_t h, const double *s, double lse, double *o) {
    const int64_t kvh = kv_head(p, h);
    for (int64_t d = 0; d < p->dh; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < p->N; ++j) {
        if (s[j] == -INFINITY) continue;
        const double pij = exp(s[j] - lse);
        const double *vj = v_row(p, b, j, kvh);
        for (int64_t d = 0; d < p->dh; ++d) o[d] += pij * vj[d];
    }
}

/* dQ_i of row (b, i, h), given its scores, lse_i and D_i. */
static void dq_row(const problem *p, int64_t b, int64_t h, int64_t i, const double *s, double lse,
                   double Di, double *dq) {
    const int64_t kvh = kv_head(p, h);
    const double *doi = do_row(p, b, i, h);
    for (int64_t d = 0; d < p->dh; ++d) dq[d] = 0.0;
    for (int64_t j = 0; j < p->N; ++j) {
        if (s[j] == -INFINITY) continue;
        const double pij = exp(s[j] - lse);
        const double dpij = dot(doi, v_row(p, b, j, kvh), p->dh);
        const double dsij = pij * (dpij - Di);
        const double *kj = k_row(p, b, j, kvh);
        for (int64_t d = 0; d < p->dh; ++d) dq[d] += p->scale * dsij * kj[d];
    }
}

/* dK_j and dV_j of key row (b, j, kvh): sums over every query head of the
 * group and every query row that sees key j.  lse and D are [B][Hq][N]. */
static void dkdv_row(const problem *p, int64_t b, int64_t kvh, int64_t j, const double *lse,
                     const double *D, double *dk, double *dv) {
    const int64_t g = group_size(p);
    const double *kj = k_row(p, b, j, kvh);
    const double *vj = v_row(p, b, j, kvh);
    for (int64_t d = 0; d < p->dh; ++d) dk[d] = dv[d] = 0.0;
    for (int64_t h = kvh * g; h < (kvh + 1) * g; ++h) {
        for (int64_t i = 0; i < p->N; ++i) {
            if (!visible(p, i, j)) continue;
            const int64_t r = (b * p->Hq + h) * p->N + i;
            const double *qi = q_row(p, b, i, h);
            const double *doi = do_row(p, b, i, h);
            const double sij = p->scale * dot(qi, kj, p->dh);
            const double pij = exp(sij - lse[r]);
            const double dsij = pij * (dot(doi, vj, p->dh) - D[r]);
            for (int64_t d = 0; d < p->dh; ++d) {
                dk[d] += p->scale * dsij * qi[d];
                dv[d] += pij * doi[d];
            }
        }
    }
}

/* lse_i and D_i of row (b, i, h). */
static void row_stats(const problem *p, int64_t b, int64_t h, int64_t i, double *s, double *o,
                      double *lse, double *Di) {
    *lse = score_row(p, b, h, i, s);
    output_row(p, b, h, s, *lse, o);
    *Di = dot(do_row(p, b, i, h), o, p->dh);
}

/* ------------------------------------------------------------------------ */
/* Exported entry points.  Return 0 on success, nonzero on invalid arguments. */

int sqa_oracle_fwd(const double *q, const double *k, const double *v, int64_t B, int64_t N,
                   int64_t Hq, int64_t Hkv, int64_t dh, int causal, double scale, double *out,
                   double *lse) {
    problem p = {q, k, v, NULL, B, N, Hq, Hkv, dh, causal, scale};
    int rc = check(&p);
    if (rc) return rc;
    const int64_t rows = B * Hq * N;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t b = r / (Hq * N), h = (r / N) % Hq, i = r % N;
            const double l = score_row(&p, b, h, i, s);
            lse[r] = l;
            output_row(&p, b, h, s, l, out + ((b * N + i) * Hq + h) * dh);
        }
        free(s);
    }
    return 0;
}

/* Forward for selected query rows; rows holds n triples (b, i, h). */
int sqa_oracle_fwd_rows(const double *q, const double *k, const double *v, int64_t B, int64_t N,
                        int64_t Hq, int64_t Hkv, int64_t dh, int causal, double scale,
                        const int64_t *rows, int64_t n, double *out_rows, double *lse_rows) {
    problem p = {q, k, v, NULL, B, N, Hq, Hkv, dh, causal, scale};
    int rc = check(&p);
    if (rc) return rc;
    for (int64_t t = 0; t < n; ++t) {
        const int64_t b = rows[3 * t], i = rows[3 * t + 1], h = rows[3 * t + 2];
        if (b < 0 || b >= B || i < 0 || i >= N || h < 0 || h >= Hq) return 4;
    }
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n; ++t) {
            const int64_t b = rows[3 * t], i = rows[3 * t + 1], h = rows[3 * t + 2];
            const double l = score_row(&p, b, h, i, s);
            lse_rows[t] = l;
            output_row(&p, b, h, s, l, out_rows + t * dh);
        }
        free(s);
    }
    return 0;
}

int sqa_oracle_bwd(const double *q, const double *k, const double *v, const double *dout, int64_t B,
                   int64_t N, int64_t Hq, int64_t Hkv, int64_t dh, int causal, double scale,
                   double *dq, double *dk, double *dv) {
    problem p = {q, k, v, dout, B, N, Hq, Hkv, dh, causal, scale};
    int rc = check(&p);
    if (rc) return rc;
    const int64_t rows = B * Hq * N;
    double *lse = (double *)malloc(sizeof(double) * rows);
    double *D = (double *)malloc(sizeof(double) * rows);
    /* Pass 1: lse_i and D_i for every query row, then dQ_i. */
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * N);
        double *o = (double *)malloc(sizeof(double) * dh);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t b = r / (Hq * N), h = (r / N) % Hq, i = r % N;
            row_stats(&p, b, h, i, s, o, &lse[r], &D[r]);
            dq_row(&p, b, h, i, s, lse[r], D[r], dq + ((b * N + i) * Hq + h) * dh);
        }
        free(o);
        free(s);
    }
    /* Pass 2: dK_j and dV_j for every key row. */
    const int64_t krows = B * Hkv * N;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < krows; ++r) {
        const int64_t b = r / (Hkv * N), kvh = (r / N) % Hkv, j = r % N;
        const int64_t off = ((b * N + j) * Hkv + kvh) * dh;
        dkdv_row(&p, b, kvh, j, lse, D, dk + off, dv + off);
    }
    free(D);
    free(lse);
    return 0;
}

/* Backward for selected rows: dQ for n_q query rows (triples b, i, h) and
 * dK, dV for n_k key rows (triples b, j, kvh). */
int sqa_oracle_bwd_rows(const double *q, const double *k, const double *v, const double *dout,
                        int64_t B, int64_t N, int64_t Hq, int64_t Hkv, int64_t dh, int causal,
                        double scale, const int64_t *qrows, int64_t n_q, double *dq_rows,
                        const int64_t *krows, int64_t n_k, double *dk_rows, double *dv_rows) {
    problem p = {q, k, v, dout, B, N, Hq, Hkv, dh, causal, scale};
    int rc = check(&p);
    if (rc) return rc;
    for (int64_t t = 0; t < n_q; ++t)
        if (qrows[3 * t] < 0 || qrows[3 * t] >= B || qrows[3 * t + 1] < 0 || qrows[3 * t + 1] >= N ||
            qrows[3 * t + 2] < 0 || qrows[3 * t + 2] >= Hq)
            return 4;
    for (int64_t t = 0; t < n_k; ++t)
        if (krows[3 * t] < 0 || krows[3 * t] >= B || krows[3 * t + 1] < 0 || krows[3 * t + 1] >= N ||
            krows[3 * t + 2] < 0 || krows[3 * t + 2] >= Hkv)
            return 4;

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * N);
        double *o = (double *)malloc(sizeof(double) * dh);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n_q; ++t) {
            const int64_t b = qrows[3 * t], i = qrows[3 * t + 1], h = qrows[3 * t + 2];
            double l, Di;
            row_stats(&p, b, h, i, s, o, &l, &Di);
            dq_row(&p, b, h, i, s, l, Di, dq_rows + t * dh);
        }
        free(o);
        free(s);
    }
    if (n_k == 0) return 0;

    /* lse and D are needed for every query row that sees one of the key rows. */
    const int64_t rows = B * Hq * N;
    const int64_t g = Hq / Hkv;
    char *need = (char *)calloc(rows, 1);
    double *lse = (double *)calloc(rows, sizeof(double));
    double *D = (double *)calloc(rows, sizeof(double));
    for (int64_t t = 0; t < n_k; ++t) {
        const int64_t b = krows[3 * t], j = krows[3 * t + 1], kvh = krows[3 * t + 2];
        for (int64_t h = kvh * g; h < (kvh + 1) * g; ++h)
            for (int64_t i = 0; i < N; ++i)
                if (visible(&p, i, j)) need[(b * Hq + h) * N + i] = 1;
    }
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * N);
        double *o = (double *)malloc(sizeof(double) * dh);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < rows; ++r) {
            if (!need[r]) continue;
            const int64_t b = r / (Hq * N), h = (r / N) % Hq, i = r % N;
            row_stats(&p, b, h, i, s, o, &lse[r], &D[r]);
        }
        free(o);
        free(s);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n_k; ++t) {
        const int64_t b = krows[3 * t], j = krows[3 * t + 1], kvh = krows[3 * t + 2];
        dkdv_row(&p, b, kvh, j, lse, D, dk_rows + t * dh, dv_rows + t * dh);
    }
    free(D);
    free(lse);
    free(need);
    return 0;
}

/* Decoding step (one new token per sequence attending to its key/value cache;
 * the step where SQA's query-head reduction saves nothing, since the cost is
 * reading the cache: arXiv 2510.01817 abstract).  For every batch entry b and
 * query head h, the single query q[b][h] attends to the first lens[b] entries
 * of the cache with no further mask:
 *   s_j   = scale * sum_d q[b,h,d] K[b,j,kv(h),d],   j < lens[b]
 *   lse   = m + ln sum_j exp(s_j - m),  m = max_j s_j
 *   out   = sum_j exp(s_j - lse) V[b,j,kv(h),:]
 * Layouts: q, out [B][H_q][dh]; k, v [B][N][H_kv][dh] (N = cache capacity);
 * lse [B][H_q].  lens[b] must lie in [1, N]. */
int sqa_oracle_decode(const double *q, const double *k, const double *v, const int64_t *lens, int64_t B,
                      int64_t N, int64_t Hq, int64_t Hkv, int64_t dh, double scale, double *out,
                      double *lse) {
    problem p = {q, k, v, NULL, B, N, Hq, Hkv, dh, 0, scale};
    int rc = check(&p);
    if (rc) return rc;
    for (int64_t b = 0; b < B; ++b)
        if (lens[b] < 1 || lens[b] > N) return 4;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < B * Hq; ++r) {
            const int64_t b = r / Hq, h = r % Hq, kvh = kv_head(&p, h), len = lens[b];
            const double *qh = q + (b * Hq + h) * dh;
            double m = -INFINITY;
            for (int64_t j = 0; j < len; ++j) {
                s[j] = scale * dot(qh, k_row(&p, b, j, kvh), dh);
                if (s[j] > m) m = s[j];
            }
            double sum = 0.0;
            for (int64_t j = 0; j < len; ++j) sum += exp(s[j] - m);
            const double l = m + log(sum);
            lse[r] = l;
            double *o = out + r * dh;
            for (int64_t d = 0; d < dh; ++d) o[d] = 0.0;
            for (int64_t j = 0; j < len; ++j) {
                const double pj = exp(s[j] - l);
                const double *vj = v_row(&p, b, j, kvh);
                for (int64_t d = 0; d < dh; ++d) o[d] += pj * vj[d];
            }
        }
        free(s);
    }
    return 0;
}
