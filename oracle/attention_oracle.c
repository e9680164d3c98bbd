/*
 * attention_oracle.c -- plain, slow, fp64 CPU oracle for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or call this file: only the tests, the package smoke check and the
 * CPU-baseline leg of the benchmark use it.  It shares no code, header,
 * table or helper with the CUDA path.
 *
 * What it computes is the plain definition of attention that the method
 * claims to reproduce exactly ("Flash Attention Explained", institutepm.com,
 * section "How Flash Attention Fixes It": the result is identical, only the
 * memory access pattern changes; "What Is Flash Attention?", bestllmfor.com,
 * table "Standard attention vs Flash Attention": exact up to floating-point
 * rounding).  So the oracle does NOT follow the tiled algorithm: for every
 * checked query row it materialises the whole score row
 *
 *     S_ij = scale * sum_k q_ik k_jk                     (j visible to i)
 *
 * then a two-pass softmax (row max, then sum of exp(S - max)), then the
 * weighted sum of value rows -- standard attention, "softmax(QK^T)V"
 * (holysheep.ai review, section "What Is Flash Attention and Why Does It
 * Matter?"; the scale defaults to 1/sqrt(head_dim) per the same page,
 * section "Implementing Flash Attention in Your Architecture").
 *
 * Causal masking follows the autoregressive reading (avichala.com,
 * "Flash Attention vs Standard Attention", section "Engineering
 * Perspective"): key j is visible to query i iff j <= i.  Sequence lengths of
 * queries and keys are equal, so top-left and bottom-right alignment agree.
 * A sliding window ("Flash Attention Explained", institutepm.com, "Sliding Window
 * Attention": each token only attends to nearby tokens) further limits causal
 * attention to the last `window` + 1 keys: j visible to i iff i - window <= j <= i.
 * window < 0 means no window.
 *
 * LSE_i = ln sum_j exp(S_ij) over visible j (natural log), the per-row
 * statistic the backward pass recomputes from.
 *
 * Backward: the pages only say that the backward pass recomputes the
 * attention matrix instead of storing it ("Flash Attention Explained",
 * "Recompute during backward pass").  The gradients themselves are the
 * textbook derivatives of L = sum(O * dO), written in Jacobian form:
 *
 *     P_ij  = exp(S_ij - LSE_i)
 *     dP_ij = sum_k dO_ik v_jk
 *     c_i   = sum_t P_it dP_it                 (Jacobian row constant)
 *     dS_ij = P_ij (dP_ij - c_i)
 *     dQ_i  = scale * sum_j dS_ij k_j
 *     dK_j  = scale * sum_i dS_ij q_i
 *     dV_j  = sum_i P_ij dO_i
 *
 * c_i is formed from P and dP directly, deliberately NOT from the shortcut
 * rowsum(dO * O), so that the GPU path's use of that shortcut is checked
 * against an independent computation.
 *
 * Data: every function works on ONE head at a time.  q, k, v, dO are
 * row-major [N][d] fp64 arrays (the caller widens bf16 exactly to fp64).
 * Outputs are fp64.  OpenMP parallelises over independent rows only; each
 * row's sums run in plain index order.
 *
 * Return value: 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Visible keys of query i: [lo, hi). */
static void visible_range(int64_t i, int64_t N, int causal, int64_t window, int64_t* lo, int64_t* hi) {
    *hi = causal ? (i + 1) : N;
    *lo = (window >= 0 && i - window > 0) ? (i - window) : 0;
}

static double dot(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int x = 0; x < d; ++x) s += a[x] * b[x];
    return s;
}

/* Scores of row i against every visible key, into srow[0..nv) for keys lo..lo+nv-1.
 * Returns nv and stores lo. */
static int score_row(const double* q, const double* k, int64_t N, int d, double scale, int causal,
                     int64_t window, int64_t i, double* srow, int64_t* lo_out) {
    int64_t lo, hi;
    visible_range(i, N, causal, window, &lo, &hi);
    const double* qi = q + i * d;
    for (int64_t j = lo; j < hi; ++j) srow[j - lo] = scale * dot(qi, k + j * d, d);
    *lo_out = lo;
    return (int)(hi - lo);
}

/* Two-pass log-sum-exp of srow[0..nv): max first, then sum of exp(s - max). */
static double lse_two_pass(const double* srow, int nv) {
    double m = -INFINITY;
    for (int j = 0; j < nv; ++j) if (srow[j] > m) m = srow[j];
    double l = 0.0;
    for (int j = 0; j < nv; ++j) l += exp(srow[j] - m);
    return m + log(l);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Forward for selected query rows of one head.
 * rows[r] in [0, N); o_out is [n_rows][d]; lse_out is [n_rows].
 */
int oracle_fwd_rows(const double* q, const double* k, const double* v,
                    int64_t N, int d, double scale, int causal, int64_t window,
                    const int64_t* rows, int64_t n_rows,
                    double* o_out, double* lse_out) {
    if (!q || !k || !v || !rows || !o_out || !lse_out || N < 1 || d < 1) return -1;
    if (window >= 0 && !causal) return -1;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return -1;
    int err = 0;
#pragma omp parallel
    {
        double* srow = (double*)malloc(sizeof(double) * (size_t)N);
        if (!srow) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < n_rows; ++r) {
                int64_t i = rows[r], lo;
                int nv = score_row(q, k, N, d, scale, causal, window, i, srow, &lo);
                double lse = lse_two_pass(srow, nv);
                double* o = o_out + r * d;
                for (int x = 0; x < d; ++x) o[x] = 0.0;
                for (int j = 0; j < nv; ++j) {
                    double p = exp(srow[j] - lse);
                    const double* vj = v + (lo + j) * d;
                    for (int x = 0; x < d; ++x) o[x] += p * vj[x];
                }
                lse_out[r] = lse;
            }
            free(srow);
        }
    }
    return err;
}

/*
 * Normalised probabilities of one query row: p_out[j] = P_ij for j < nv,
 * zero for masked keys.  p_out has N entries.  Used by the tests to check
 * the softmax itself (rows sum to one, agreement with a library softmax).
 */
int oracle_prob_row(const double* q, const double* k, int64_t N, int d,
                    double scale, int causal, int64_t window, int64_t i, double* p_out) {
    if (!q || !k || !p_out || N < 1 || d < 1 || i < 0 || i >= N) return -1;
    if (window >= 0 && !causal) return -1;
    double* srow = (double*)malloc(sizeof(double) * (size_t)N);
    if (!srow) return -2;
    int64_t lo;
    int nv = score_row(q, k, N, d, scale, causal, window, i, srow, &lo);
    double lse = lse_two_pass(srow, nv);
    for (int64_t j = 0; j < N; ++j) p_out[j] = (j >= lo && j < lo + nv) ? exp(srow[j - lo] - lse) : 0.0;
    free(srow);
    return 0;
}

/*
 * Backward for one head.
 *   Pass 1 (all query rows): LSE_i and the Jacobian row constant c_i.
 *   dQ at the requested query rows  qrows[0..nq)  -> dq_out [nq][d],
 *       and c at those rows -> c_out [nq] (may be NULL).
 *   dK, dV at the requested key rows krows[0..nk) -> dk_out, dv_out [nk][d].
 * Every dS_ij is recomputed from scratch where it is needed; nothing is
 * blocked or reordered beyond the definitions in the file header.
 */
int oracle_bwd_rows(const double* q, const double* k, const double* v,
                    const double* dO, int64_t N, int d, double scale, int causal, int64_t window,
                    const int64_t* qrows, int64_t nq, double* dq_out, double* c_out,
                    const int64_t* krows, int64_t nk, double* dk_out, double* dv_out) {
    if (!q || !k || !v || !dO || N < 1 || d < 1) return -1;
    if (window >= 0 && !causal) return -1;
    if (nq > 0 && (!qrows || !dq_out)) return -1;
    if (nk > 0 && (!krows || !dk_out || !dv_out)) return -1;
    for (int64_t r = 0; r < nq; ++r) if (qrows[r] < 0 || qrows[r] >= N) return -1;
    for (int64_t r = 0; r < nk; ++r) if (krows[r] < 0 || krows[r] >= N) return -1;

    double* lse = (double*)malloc(sizeof(double) * (size_t)N);
    double* crow = (double*)malloc(sizeof(double) * (size_t)N);
    if (!lse || !crow) { free(lse); free(crow); return -2; }
    int err = 0;

    /* Pass 1: per query row, LSE_i and c_i = sum_t P_it dP_it. */
#pragma omp parallel
    {
        double* srow = (double*)malloc(sizeof(double) * (size_t)N);
        if (!srow) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = 0; i < N; ++i) {
                int64_t lo;
                int nv = score_row(q, k, N, d, scale, causal, window, i, srow, &lo);
                double l = lse_two_pass(srow, nv);
                double c = 0.0;
                const double* doi = dO + i * d;
                for (int j = 0; j < nv; ++j) {
                    double p = exp(srow[j] - l);
                    double dp = dot(doi, v + (lo + j) * d, d);
                    c += p * dp;
                }
                lse[i] = l;
                crow[i] = c;
            }
            free(srow);
        }
    }
    if (err) { free(lse); free(crow); return err; }

    /* dQ_i = scale * sum_j dS_ij k_j at the requested query rows. */
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nq; ++r) {
        int64_t i = qrows[r], lo, hi;
        visible_range(i, N, causal, window, &lo, &hi);
        const double* qi = q + i * d;
        const double* doi = dO + i * d;
        double* dq = dq_out + r * d;
        for (int x = 0; x < d; ++x) dq[x] = 0.0;
        for (int64_t j = lo; j < hi; ++j) {
            const double* kj = k + j * d;
            double p = exp(scale * dot(qi, kj, d) - lse[i]);
            double ds = p * (dot(doi, v + j * d, d) - crow[i]);
            for (int x = 0; x < d; ++x) dq[x] += ds * kj[x];
        }
        for (int x = 0; x < d; ++x) dq[x] *= scale;
        if (c_out) c_out[r] = crow[i];
    }

    /* dK_j = scale * sum_i dS_ij q_i and dV_j = sum_i P_ij dO_i at the requested key rows. */
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nk; ++r) {
        int64_t j = krows[r];
        const double* kj = k + j * d;
        const double* vj = v + j * d;
        double* dk = dk_out + r * d;
        double* dv = dv_out + r * d;
        for (int x = 0; x < d; ++x) { dk[x] = 0.0; dv[x] = 0.0; }
        /* queries that see key j: i >= j when causal, and i <= j + window with a window */
        int64_t i0 = causal ? j : 0;
        int64_t i1 = (window >= 0 && j + window + 1 < N) ? (j + window + 1) : N;
        for (int64_t i = i0; i < i1; ++i) {
            const double* qi = q + i * d;
            const double* doi = dO + i * d;
            double p = exp(scale * dot(qi, kj, d) - lse[i]);
            double ds = p * (dot(doi, vj, d) - crow[i]);
            for (int x = 0; x < d; ++x) {
                dk[x] += ds * qi[x];
                dv[x] += p * doi[x];
            }
        }
        for (int x = 0; x < d; ++x) dk[x] *= scale;
    }

    free(lse);
    free(crow);
    return 0;
}
