/*
 * attention_oracle.c -- plain fp64 CPU oracle for (causal) scaled dot-product
 * attention and its gradients.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * path.
 *
 * What it computes is the plain definition, not the tiled algorithm:
 *
 *   forward  (CS336 A2 Systems handout, section 4.1.1 Eq. 1 and section 4.2.2
 *             Eqs. 4-6 and 12):
 *       S_ij = scale * q_i . k_j                   (Eq. 4 with a general scale)
 *       causal: key j is visible to query i iff j <= i
 *               (handout, Problem flash_forward (c): index comparison of the
 *               query and key positions; masked scores take no part in the
 *               softmax)
 *       L_i  = log sum_j exp(S_ij)                 (Eq. 12, natural log)
 *       P_ij = exp(S_ij - L_i)                     (= softmax_j, Eq. 5)
 *       O_i  = sum_j P_ij v_j                      (Eq. 6)
 *
 *   backward (same section, standard backward Eqs. 7-11, i.e. through the
 *             softmax Jacobian, NOT through the D = rowsum(O o dO) shortcut):
 *       dV_j  = sum_i P_ij dO_i                    (Eq. 7)
 *       dP_ij = dO_i . v_j                         (Eq. 8)
 *       dS_i  = (diag(P_i) - P_i P_i^T) dP_i       (Eq. 9)
 *             -> dS_ij = P_ij dP_ij - P_ij * sum_k P_ik dP_ik
 *       dQ_i  = scale * sum_j dS_ij k_j            (Eq. 10)
 *       dK_j  = scale * sum_i dS_ij q_i            (Eq. 11)
 *
 * Layout: every tensor is a dense row-major array of `heads` independent
 * problems; q and dout are [heads][nq][d], k and v are [heads][nk][d], o is
 * [heads][nq][d], lse is [heads][nq].  Everything is double.
 *
 * Parallelism: OpenMP over (head, row) and (head, key) only; the arithmetic of
 * each output element is a plain loop in the order the definition gives.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEMORY 2

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double dot(const double* a, const double* b, long d) {
    double s = 0.0;
    for (long t = 0; t < d; ++t) s += a[t] * b[t];
    return s;
}

/* Number of keys query row i may see: all nk, or keys 0..i under the causal
 * rule (at least one key when nk >= 1). */
static long visible_keys(long i, long nk, int causal) {
    if (!causal) return nk;
    long n = i + 1;
    return n < nk ? n : nk;
}

/* Scores of row i into s[0..nvis): S_ij = scale * q_i . k_j. */
static void row_scores(const double* qi, const double* kh, long d, long nvis,
                       double scale, double* s) {
    for (long j = 0; j < nvis; ++j) s[j] = scale * dot(qi, kh + j * d, d);
}

/* L_i = log sum_j exp(S_ij), evaluated with the usual max shift so that the
 * exponentials cannot overflow: L = m + log sum_j exp(S_ij - m). */
static double row_logsumexp(const double* s, long nvis) {
    double m = -INFINITY;
    for (long j = 0; j < nvis; ++j) if (s[j] > m) m = s[j];
    double z = 0.0;
    for (long j = 0; j < nvis; ++j) z += exp(s[j] - m);
    return m + log(z);
}

static int check_dims(long heads, long nq, long nk, long d) {
    return heads >= 1 && nq >= 1 && nk >= 1 && d >= 1;
}

/*
 * Forward: O and L for every head and query row.
 */
int oracle_forward(const double* q, const double* k, const double* v,
                   double* o, double* lse,
                   long heads, long nq, long nk, long d, int causal, double scale) {
    if (!q || !k || !v || !o || !lse || !check_dims(heads, nq, nk, d)) return ORACLE_BAD_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)nk);
        if (!s) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (long h = 0; h < heads; ++h) {
            for (long i = 0; i < nq; ++i) {
                if (!s) continue;
                const double* qi = q + (h * nq + i) * d;
                const double* kh = k + h * nk * d;
                const double* vh = v + h * nk * d;
                long nvis = visible_keys(i, nk, causal);
                row_scores(qi, kh, d, nvis, scale, s);
                double L = row_logsumexp(s, nvis);
                double* oi = o + (h * nq + i) * d;
                for (long t = 0; t < d; ++t) oi[t] = 0.0;
                for (long j = 0; j < nvis; ++j) {
                    double p = exp(s[j] - L);
                    const double* vj = vh + j * d;
                    for (long t = 0; t < d; ++t) oi[t] += p * vj[t];
                }
                lse[h * nq + i] = L;
            }
        }
        free(s);
    }
    return err;
}

/*
 * Per-row statistics the gradient needs for one head:
 *   L_i  (the normaliser, Eq. 12) and
 *   c_i  = P_i^T dP_i = sum_k P_ik dP_ik  (the scalar in the Jacobian
 *          product of Eq. 9).
 * Optionally the row's dQ_i (Eq. 10), which only needs row i.
 */
static void row_grad_stats(const double* qh, const double* kh, const double* vh,
                           const double* doh, long i, long nk, long d, int causal,
                           double scale, double* s, double* dp,
                           double* L_out, double* c_out, double* dq_out) {
    const double* qi = qh + i * d;
    const double* doi = doh + i * d;
    long nvis = visible_keys(i, nk, causal);
    row_scores(qi, kh, d, nvis, scale, s);
    double L = row_logsumexp(s, nvis);
    double c = 0.0;
    for (long j = 0; j < nvis; ++j) {
        s[j] = exp(s[j] - L);                 /* s now holds P_ij */
        dp[j] = dot(doi, vh + j * d, d);      /* dP_ij = dO_i . v_j (Eq. 8) */
        c += s[j] * dp[j];
    }
    *L_out = L;
    *c_out = c;
    if (dq_out) {
        for (long t = 0; t < d; ++t) dq_out[t] = 0.0;
        for (long j = 0; j < nvis; ++j) {
            double ds = s[j] * dp[j] - s[j] * c;   /* (diag(P_i) - P_i P_i^T) dP_i */
            const double* kj = kh + j * d;
            for (long t = 0; t < d; ++t) dq_out[t] += ds * kj[t];
        }
        for (long t = 0; t < d; ++t) dq_out[t] *= scale;
    }
}

/* dK_j and dV_j for key row j of one head, given every row's L_i and c_i:
 * dV_j = sum_i P_ij dO_i, dK_j = scale * sum_i dS_ij q_i over the query rows
 * that see key j. */
static void key_grads(const double* qh, const double* kh, const double* vh,
                      const double* doh, const double* L, const double* c,
                      long j, long nq, long d, int causal, double scale,
                      double* dk_out, double* dv_out) {
    const double* kj = kh + j * d;
    const double* vj = vh + j * d;
    for (long t = 0; t < d; ++t) { dk_out[t] = 0.0; dv_out[t] = 0.0; }
    long i0 = causal ? j : 0;
    for (long i = i0; i < nq; ++i) {
        const double* qi = qh + i * d;
        const double* doi = doh + i * d;
        double p = exp(scale * dot(qi, kj, d) - L[i]);
        double dp = dot(doi, vj, d);
        double ds = p * dp - p * c[i];
        for (long t = 0; t < d; ++t) {
            dv_out[t] += p * doi[t];
            dk_out[t] += ds * qi[t];
        }
    }
    for (long t = 0; t < d; ++t) dk_out[t] *= scale;
}

/*
 * Backward: dQ, dK, dV for every head.  `stats` (optional, [heads][nq][2])
 * receives (L_i, c_i) per row so that callers can inspect the Jacobian
 * scalar; pass NULL to skip.
 */
int oracle_backward(const double* q, const double* k, const double* v, const double* dout,
                    double* dq, double* dk, double* dv, double* stats,
                    long heads, long nq, long nk, long d, int causal, double scale) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !check_dims(heads, nq, nk, d))
        return ORACLE_BAD_ARG;
    double* L = (double*)malloc(sizeof(double) * (size_t)(heads * nq));
    double* c = (double*)malloc(sizeof(double) * (size_t)(heads * nq));
    if (!L || !c) { free(L); free(c); return ORACLE_NO_MEMORY; }
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)nk);
        double* dp = (double*)malloc(sizeof(double) * (size_t)nk);
        if (!s || !dp) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (long h = 0; h < heads; ++h) {
            for (long i = 0; i < nq; ++i) {
                if (!s || !dp) continue;
                row_grad_stats(q + h * nq * d, k + h * nk * d, v + h * nk * d,
                               dout + h * nq * d, i, nk, d, causal, scale, s, dp,
                               &L[h * nq + i], &c[h * nq + i], dq + (h * nq + i) * d);
            }
        }
        free(s);
        free(dp);
    }
    if (err == ORACLE_OK) {
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
        for (long h = 0; h < heads; ++h) {
            for (long j = 0; j < nk; ++j) {
                key_grads(q + h * nq * d, k + h * nk * d, v + h * nk * d, dout + h * nq * d,
                          L + h * nq, c + h * nq, j, nq, d, causal, scale,
                          dk + (h * nk + j) * d, dv + (h * nk + j) * d);
            }
        }
        if (stats) {
            for (long r = 0; r < heads * nq; ++r) {
                stats[2 * r] = L[r];
                stats[2 * r + 1] = c[r];
            }
        }
    }
    free(L);
    free(c);
    return err;
}

/*
 * Block-sparse attention ("Notes on flashattention" post, section
 * "Block-sparse Flashattention", with its Proposition 4): a block mask M over
 * (query block, key block) pairs of bq x bk rows; key j is visible to query i
 * iff M[i / bq][j / bk] != 0 and, with causal, j <= i.  Masked scores take no
 * part in the softmax: the page's algorithm skips the zero blocks entirely,
 * which is what excluding them computes (the page's "(S o 1_M)_kl = 0 where
 * M_kl = 0" is read as "excluded from the softmax", the only reading under
 * which skipping those blocks gives the same P).  A query row that sees no key
 * has O_i = 0 and L_i = -inf, dQ_i = 0, and adds nothing to dK or dV.
 * mask is [ceil(nq / bq)][ceil(nk / bk)] bytes, row-major.
 */
static int visible_bs(long i, long j, int causal, const unsigned char* mask, long nbk,
                      long bq, long bk) {
    if (causal && j > i) return 0;
    return mask[(i / bq) * nbk + (j / bk)] != 0;
}

static int check_mask(const unsigned char* mask, long bq, long bk) {
    return mask != NULL && bq >= 1 && bk >= 1;
}

/* Scores of row i over its visible keys: idx[0..n) the key indices in
 * increasing order, s[0..n) the scores; returns n. */
static long row_scores_bs(const double* qi, const double* kh, long i, long nk, long d,
                          int causal, double scale, const unsigned char* mask, long nbk,
                          long bq, long bk, long* idx, double* s) {
    long n = 0;
    for (long j = 0; j < nk; ++j) {
        if (!visible_bs(i, j, causal, mask, nbk, bq, bk)) continue;
        idx[n] = j;
        s[n] = scale * dot(qi, kh + j * d, d);
        ++n;
    }
    return n;
}

int oracle_forward_bs(const double* q, const double* k, const double* v,
                      double* o, double* lse,
                      long heads, long nq, long nk, long d, int causal, double scale,
                      const unsigned char* mask, long bq, long bk) {
    if (!q || !k || !v || !o || !lse || !check_dims(heads, nq, nk, d) || !check_mask(mask, bq, bk))
        return ORACLE_BAD_ARG;
    const long nbk = (nk + bk - 1) / bk;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)nk);
        long* idx = (long*)malloc(sizeof(long) * (size_t)nk);
        if (!s || !idx) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (long h = 0; h < heads; ++h) {
            for (long i = 0; i < nq; ++i) {
                if (!s || !idx) continue;
                const double* vh = v + h * nk * d;
                long n = row_scores_bs(q + (h * nq + i) * d, k + h * nk * d, i, nk, d, causal,
                                       scale, mask, nbk, bq, bk, idx, s);
                double* oi = o + (h * nq + i) * d;
                for (long t = 0; t < d; ++t) oi[t] = 0.0;
                if (n == 0) {
                    lse[h * nq + i] = -INFINITY;
                    continue;
                }
                double L = row_logsumexp(s, n);
                for (long r = 0; r < n; ++r) {
                    double p = exp(s[r] - L);
                    const double* vj = vh + idx[r] * d;
                    for (long t = 0; t < d; ++t) oi[t] += p * vj[t];
                }
                lse[h * nq + i] = L;
            }
        }
        free(s);
        free(idx);
    }
    return err;
}

int oracle_backward_bs(const double* q, const double* k, const double* v, const double* dout,
                       double* dq, double* dk, double* dv,
                       long heads, long nq, long nk, long d, int causal, double scale,
                       const unsigned char* mask, long bq, long bk) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !check_dims(heads, nq, nk, d) ||
        !check_mask(mask, bq, bk))
        return ORACLE_BAD_ARG;
    const long nbk = (nk + bk - 1) / bk;
    double* L = (double*)malloc(sizeof(double) * (size_t)(heads * nq));
    double* c = (double*)malloc(sizeof(double) * (size_t)(heads * nq));
    if (!L || !c) { free(L); free(c); return ORACLE_NO_MEMORY; }
    int err = ORACLE_OK;
    /* Per row: L_i, c_i = sum_j P_ij dP_ij (Eq. 9's scalar) and dQ_i (Eq. 10). */
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)nk);
        double* dp = (double*)malloc(sizeof(double) * (size_t)nk);
        long* idx = (long*)malloc(sizeof(long) * (size_t)nk);
        if (!s || !dp || !idx) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (long h = 0; h < heads; ++h) {
            for (long i = 0; i < nq; ++i) {
                if (!s || !dp || !idx) continue;
                const double* kh = k + h * nk * d;
                const double* vh = v + h * nk * d;
                const double* doi = dout + (h * nq + i) * d;
                double* dqi = dq + (h * nq + i) * d;
                for (long t = 0; t < d; ++t) dqi[t] = 0.0;
                long n = row_scores_bs(q + (h * nq + i) * d, kh, i, nk, d, causal, scale,
                                       mask, nbk, bq, bk, idx, s);
                if (n == 0) {
                    L[h * nq + i] = -INFINITY;
                    c[h * nq + i] = 0.0;
                    continue;
                }
                double Li = row_logsumexp(s, n);
                double ci = 0.0;
                for (long r = 0; r < n; ++r) {
                    s[r] = exp(s[r] - Li);                       /* P_ij */
                    dp[r] = dot(doi, vh + idx[r] * d, d);        /* dP_ij (Eq. 8) */
                    ci += s[r] * dp[r];
                }
                for (long r = 0; r < n; ++r) {
                    double ds = s[r] * dp[r] - s[r] * ci;
                    const double* kj = kh + idx[r] * d;
                    for (long t = 0; t < d; ++t) dqi[t] += ds * kj[t];
                }
                for (long t = 0; t < d; ++t) dqi[t] *= scale;
                L[h * nq + i] = Li;
                c[h * nq + i] = ci;
            }
        }
        free(s);
        free(dp);
        free(idx);
    }
    /* Per key: dV_j = sum_i P_ij dO_i (Eq. 7), dK_j = scale sum_i dS_ij q_i (Eq. 11)
     * over the query rows that see key j. */
    if (err == ORACLE_OK) {
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
        for (long h = 0; h < heads; ++h) {
            for (long j = 0; j < nk; ++j) {
                const double* qh = q + h * nq * d;
                const double* doh = dout + h * nq * d;
                const double* kj = k + (h * nk + j) * d;
                const double* vj = v + (h * nk + j) * d;
                double* dkj = dk + (h * nk + j) * d;
                double* dvj = dv + (h * nk + j) * d;
                for (long t = 0; t < d; ++t) { dkj[t] = 0.0; dvj[t] = 0.0; }
                for (long i = 0; i < nq; ++i) {
                    if (!visible_bs(i, j, causal, mask, nbk, bq, bk)) continue;
                    const double* qi = qh + i * d;
                    const double* doi = doh + i * d;
                    double p = exp(scale * dot(qi, kj, d) - L[h * nq + i]);
                    double dpv = dot(doi, vj, d);
                    double ds = p * dpv - p * c[h * nq + i];
                    for (long t = 0; t < d; ++t) {
                        dvj[t] += p * doi[t];
                        dkj[t] += ds * qi[t];
                    }
                }
                for (long t = 0; t < d; ++t) dkj[t] *= scale;
            }
        }
    }
    free(L);
    free(c);
    return err;
}

/*
 * Sampled outputs of ONE head (q, dout: [nq][d]; k, v: [nk][d]) for checking
 * sizes where the full outputs would take too long to compare:
 *   o_rows/lse_rows/dq_rows for the query rows listed in qrows,
 *   dk_rows/dv_rows for the key rows listed in krows.
 * dK/dV of one key need L_i and c_i of every query row, so those are computed
 * for all rows first (a full pass over the head).  Any output pointer may be
 * NULL to skip it; dout may be NULL when no gradient is asked for.
 */
int oracle_head_sampled(const double* q, const double* k, const double* v, const double* dout,
                        long nq, long nk, long d, int causal, double scale,
                        const long* qrows, long n_qrows, const long* krows, long n_krows,
                        double* o_rows, double* lse_rows, double* dq_rows,
                        double* dk_rows, double* dv_rows) {
    if (!q || !k || !v || !check_dims(1, nq, nk, d)) return ORACLE_BAD_ARG;
    if ((n_qrows > 0 && !qrows) || (n_krows > 0 && !krows)) return ORACLE_BAD_ARG;
    int want_grad = (dq_rows && n_qrows > 0) || ((dk_rows || dv_rows) && n_krows > 0);
    if (want_grad && !dout) return ORACLE_BAD_ARG;
    for (long r = 0; r < n_qrows; ++r) if (qrows[r] < 0 || qrows[r] >= nq) return ORACLE_BAD_ARG;
    for (long r = 0; r < n_krows; ++r) if (krows[r] < 0 || krows[r] >= nk) return ORACLE_BAD_ARG;

    /* Forward rows: reuse the full forward on the selected rows of a 1-row
     * view each (row i of the head with its own causal horizon). */
    int err = ORACLE_OK;
    if (o_rows || lse_rows) {
#pragma omp parallel
        {
            double* s = (double*)malloc(sizeof(double) * (size_t)nk);
            if (!s) {
#pragma omp atomic write
                err = ORACLE_NO_MEMORY;
            }
#pragma omp for schedule(dynamic, 4)
            for (long r = 0; r < n_qrows; ++r) {
                if (!s) continue;
                long i = qrows[r];
                long nvis = visible_keys(i, nk, causal);
                row_scores(q + i * d, k, d, nvis, scale, s);
                double L = row_logsumexp(s, nvis);
                if (lse_rows) lse_rows[r] = L;
                if (o_rows) {
                    double* orow = o_rows + r * d;
                    for (long t = 0; t < d; ++t) orow[t] = 0.0;
                    for (long j = 0; j < nvis; ++j) {
                        double p = exp(s[j] - L);
                        for (long t = 0; t < d; ++t) orow[t] += p * v[j * d + t];
                    }
                }
            }
            free(s);
        }
        if (err != ORACLE_OK) return err;
    }
    if (!want_grad) return ORACLE_OK;

    int need_all_rows = (dk_rows || dv_rows) && n_krows > 0;
    double* L = (double*)malloc(sizeof(double) * (size_t)nq);
    double* c = (double*)malloc(sizeof(double) * (size_t)nq);
    if (!L || !c) { free(L); free(c); return ORACLE_NO_MEMORY; }
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)nk);
        double* dp = (double*)malloc(sizeof(double) * (size_t)nk);
        if (!s || !dp) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
        if (need_all_rows) {
#pragma omp for schedule(dynamic, 16)
            for (long i = 0; i < nq; ++i) {
                if (!s || !dp) continue;
                row_grad_stats(q, k, v, dout, i, nk, d, causal, scale, s, dp, &L[i], &c[i], NULL);
            }
        }
        if (dq_rows) {
#pragma omp for schedule(dynamic, 4)
            for (long r = 0; r < n_qrows; ++r) {
                if (!s || !dp) continue;
                double Lr, cr;
                row_grad_stats(q, k, v, dout, qrows[r], nk, d, causal, scale, s, dp, &Lr, &cr,
                               dq_rows + r * d);
            }
        }
        free(s);
        free(dp);
    }
    if (err == ORACLE_OK && need_all_rows) {
        double* tmp_dk = NULL;
        double* tmp_dv = NULL;
        if (!dk_rows) tmp_dk = (double*)malloc(sizeof(double) * (size_t)(n_krows * d));
        if (!dv_rows) tmp_dv = (double*)malloc(sizeof(double) * (size_t)(n_krows * d));
        double* dkp = dk_rows ? dk_rows : tmp_dk;
        double* dvp = dv_rows ? dv_rows : tmp_dv;
        if (!dkp || !dvp) {
            err = ORACLE_NO_MEMORY;
        } else {
#pragma omp parallel for schedule(dynamic, 4)
            for (long r = 0; r < n_krows; ++r) {
                key_grads(q, k, v, dout, L, c, krows[r], nq, d, causal, scale,
                          dkp + r * d, dvp + r * d);
            }
        }
        free(tmp_dk);
        free(tmp_dv);
    }
    free(L);
    free(c);
    return err;
}
