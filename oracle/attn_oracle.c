/*
 * fp64 CPU oracle for exact scaled-dot-product attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or call
 * this file: only the test suite, the package smoke check and the CPU-baseline leg
 * of the benchmark use it. It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes is the plain three-step definition of attention, written out
 * without tiling, fusion or reordering:
 *
 *   s_ij = scale * (q_i . k_j)            the score matrix, one full row at a time
 *                                         (josueisai.com "flash-attention",
 *                                          section "La matriz que nunca deberias
 *                                          guardar": S = Q K^T, step 1)
 *   P_ij = exp(s_ij - m_i) / l_i          row softmax with max subtraction,
 *          m_i = max_j s_ij,              (same section, step 2; the max is
 *          l_i = sum_j exp(s_ij - m_i)     subtracted "por estabilidad numerica" as
 *                                          section "El truco" states)
 *   O_i  = sum_j P_ij v_j                 (same section, step 3)
 *   L_i  = m_i + ln l_i                   the per-row log-sum-exp statistic that the
 *                                         backward keeps (kerneldigest.dev
 *                                         "FlashAttention", first paragraph:
 *                                         online log-sum-exp scaling; josueisai.com
 *                                         section "Recomputar sale mas barato que
 *                                         recordar": only per-row statistics survive)
 *
 * Causal masking (a reading, not on the pages): key j is visible to query i iff
 * j <= i + (N_k - N_q), i.e. the last query sees every key ("bottom-right"
 * alignment; with N_q = N_k this is j <= i). Masked scores do not enter the max or
 * the sum, so P_ij = 0 there. With N_q > N_k the first N_q - N_k queries see no key
 * at all; their rows are defined as O_i = 0, L_i = -inf, dQ_i = 0, D_i = 0 (the
 * empty sum), and they add nothing to dK or dV.
 *
 * Backward, given dO (standard calculus of the three steps above; the pages say only
 * that the gradient needs P and that P is recomputed from Q, K, V):
 *
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = dO_i . v_j
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)            (the softmax Jacobian applied to dP)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 *
 * Inputs are double arrays, q and dO [BH][N_q][d], k and v [BH][N_k][d] (the
 * square entry points take N_q = N_k = N); for parity checks they hold the exact 16-bit
 * values used on the GPU (widening is exact). Every product and sum is taken in
 * double, and outputs are double.
 *
 * Return codes: 0 on success, -1 for invalid arguments, -2 when scratch memory
 * cannot be allocated.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_ENOMEM (-2)

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Number of keys that query row i sees: a prefix of the Nk keys. */
static long visible_keys(long i, long Nq, long Nk, int causal) {
    if (!causal) return Nk;
    const long n = i + 1 + (Nk - Nq);
    return n < 0 ? 0 : (n > Nk ? Nk : n);
}

/* s[j] = scale * (q_i . k_j) for the first nvis keys of one head. */
static void score_row(const double *qi, const double *kh, long nvis, long d, double scale,
                      double *s) {
    for (long j = 0; j < nvis; ++j) {
        const double *kj = kh + j * d;
        double acc = 0.0;
        for (long t = 0; t < d; ++t) acc += qi[t] * kj[t];
        s[j] = scale * acc;
    }
}

/* Two-pass row softmax: in place, scores -> probabilities. Returns m and l. */
static void softmax_row(double *s, long nvis, double *m_out, double *l_out) {
    double m = -INFINITY;
    for (long j = 0; j < nvis; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (long j = 0; j < nvis; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    if (nvis > 0)
        for (long j = 0; j < nvis; ++j) s[j] /= l;
    *m_out = m;  /* -inf and 0 for a row that sees no key */
    *l_out = l;
}

/* out[t] = sum_j w[j] * x_j[t] over the first nvis rows of x (one head, row stride d). */
static void weighted_rows(const double *w, const double *xh, long nvis, long d, double *out) {
    for (long t = 0; t < d; ++t) out[t] = 0.0;
    for (long j = 0; j < nvis; ++j) {
        const double *xj = xh + j * d;
        const double wj = w[j];
        for (long t = 0; t < d; ++t) out[t] += wj * xj[t];
    }
}

/*
 * Everything that depends on one query row only: P_i (left in p), O_i, m_i, l_i,
 * and, when doi != NULL, dP_i (left in dp), D_i and dQ_i.
 */
static void query_row(const double *qh, const double *kh, const double *vh, const double *doh,
                      long Nq, long Nk, long d, int causal, double scale, long i, double *p,
                      double *dp, double *o_i, double *m_i, double *l_i, double *D_i,
                      double *dq_i) {
    const long nvis = visible_keys(i, Nq, Nk, causal);
    const double *qi = qh + i * d;
    score_row(qi, kh, nvis, d, scale, p);
    softmax_row(p, nvis, m_i, l_i);
    if (o_i) weighted_rows(p, vh, nvis, d, o_i);
    if (!doh) return;
    const double *doi = doh + i * d;
    double D = 0.0;
    for (long j = 0; j < nvis; ++j) {
        const double *vj = vh + j * d;
        double acc = 0.0;
        for (long t = 0; t < d; ++t) acc += doi[t] * vj[t];
        dp[j] = acc;
        D += p[j] * acc;
    }
    *D_i = D;
    if (dq_i) {
        /* dS_ij = P_ij (dP_ij - D_i), reusing dp as storage for dS */
        for (long j = 0; j < nvis; ++j) dp[j] = p[j] * (dp[j] - D);
        weighted_rows(dp, kh, nvis, d, dq_i);
        for (long t = 0; t < d; ++t) dq_i[t] *= scale;
    }
}

static int check_args(const void *q, const void *k, const void *v, long BH, long Nq, long Nk,
                      long d) {
    if (!q || !k || !v) return ORC_EINVAL;
    if (BH < 0 || Nq < 0 || Nk < 0 || d <= 0) return ORC_EINVAL;
    return ORC_OK;
}

/* Forward: o [BH][Nq][d] and L [BH][Nq] (either may be NULL). */
int oracle_attn_fwd_qk(const double *q, const double *k, const double *v, long BH, long Nq,
                       long Nk, long d, int causal, double scale, double *o, double *L) {
    if (check_args(q, k, v, BH, Nq, Nk, d)) return ORC_EINVAL;
    int err = ORC_OK;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        if (!p) {
#pragma omp atomic write
            err = ORC_ENOMEM;
        }
#pragma omp for schedule(dynamic, 16) collapse(2)
        for (long bh = 0; bh < BH; ++bh)
            for (long i = 0; i < Nq; ++i) {
                if (!p) continue;
                const size_t hq = (size_t)bh * Nq * d, hk = (size_t)bh * Nk * d;
                double m, l;
                query_row(q + hq, k + hk, v + hk, NULL, Nq, Nk, d, causal, scale, i, p, NULL,
                          o ? o + hq + (size_t)i * d : NULL, &m, &l, NULL, NULL);
                if (L) L[(size_t)bh * Nq + i] = m + log(l);
            }
        free(p);
    }
    return err;
}

int oracle_attn_fwd(const double *q, const double *k, const double *v, long BH, long N, long d,
                    int causal, double scale, double *o, double *L) {
    return oracle_attn_fwd_qk(q, k, v, BH, N, N, d, causal, scale, o, L);
}

/*
 * Per-row statistics of every row of one head that can see a key >= j_min:
 * m, l, D (arrays of N doubles, rows below the first such row left untouched).
 */
static int head_row_stats(const double *qh, const double *kh, const double *vh, const double *doh,
                          long N, long d, int causal, double scale, long j_min, double *m,
                          double *l, double *D) {
    const long i0 = causal ? j_min : 0;
    int err = ORC_OK;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *dp = (double *)malloc(sizeof(double) * (size_t)N);
        if (!p || !dp) {
#pragma omp atomic write
            err = ORC_ENOMEM;
        }
#pragma omp for schedule(dynamic, 16)
        for (long i = i0; i < N; ++i) {
            if (!p || !dp) continue;
            query_row(qh, kh, vh, doh, N, N, d, causal, scale, i, p, dp, NULL, &m[i], &l[i],
                      &D[i], NULL);
        }
        free(p);
        free(dp);
    }
    return err;
}

/*
 * dK_j and dV_j of one key of one head, from the row statistics m, l, D:
 * P_ij = exp(s_ij - m_i) / l_i for every row i that sees key j.
 */
static void key_grads(const double *qh, const double *kh, const double *vh, const double *doh,
                      long Nq, long Nk, long d, int causal, double scale, long j, const double *m,
                      const double *l, const double *D, double *dk_j, double *dv_j) {
    const double *kj = kh + j * d;
    const double *vj = vh + j * d;
    for (long t = 0; t < d; ++t) dk_j[t] = dv_j[t] = 0.0;
    /* rows that see key j: i + (Nk - Nq) >= j */
    long i0 = causal ? j - (Nk - Nq) : 0;
    if (i0 < 0) i0 = 0;
    for (long i = i0; i < Nq; ++i) {
        const double *qi = qh + i * d;
        const double *doi = doh + i * d;
        double s = 0.0, dp = 0.0;
        for (long t = 0; t < d; ++t) {
            s += qi[t] * kj[t];
            dp += doi[t] * vj[t];
        }
        s *= scale;
        const double P = exp(s - m[i]) / l[i];
        const double dS = P * (dp - D[i]);
        for (long t = 0; t < d; ++t) {
            dv_j[t] += P * doi[t];
            dk_j[t] += scale * dS * qi[t];
        }
    }
}

/*
 * Forward and backward for every head. o, L, dq, dk, dv, D may each be NULL.
 * Row-wise quantities first, then key-wise ones (dK, dV) from the stored m, l, D.
 */
int oracle_attn_bwd_qk(const double *q, const double *k, const double *v, const double *dO,
                       long BH, long Nq, long Nk, long d, int causal, double scale, double *o,
                       double *L, double *dq, double *dk, double *dv, double *D_out) {
    if (check_args(q, k, v, BH, Nq, Nk, d) || !dO) return ORC_EINVAL;
    if (Nq == 0 || Nk == 0 || BH == 0) return ORC_OK;
    double *m = (double *)malloc(sizeof(double) * (size_t)Nq);
    double *l = (double *)malloc(sizeof(double) * (size_t)Nq);
    double *D = (double *)malloc(sizeof(double) * (size_t)Nq);
    if (!m || !l || !D) {
        free(m); free(l); free(D);
        return ORC_ENOMEM;
    }
    int err = ORC_OK;
    for (long bh = 0; bh < BH && err == ORC_OK; ++bh) {
        const size_t hq = (size_t)bh * Nq * d, hk = (size_t)bh * Nk * d;
        const double *qh = q + hq, *kh = k + hk, *vh = v + hk, *doh = dO + hq;
#pragma omp parallel
        {
            double *p = (double *)malloc(sizeof(double) * (size_t)Nk);
            double *dp = (double *)malloc(sizeof(double) * (size_t)Nk);
            if (!p || !dp) {
#pragma omp atomic write
                err = ORC_ENOMEM;
            }
#pragma omp for schedule(dynamic, 8)
            for (long i = 0; i < Nq; ++i) {
                if (!p || !dp) continue;
                query_row(qh, kh, vh, doh, Nq, Nk, d, causal, scale, i, p, dp,
                          o ? o + hq + (size_t)i * d : NULL, &m[i], &l[i], &D[i],
                          dq ? dq + hq + (size_t)i * d : NULL);
            }
            free(p);
            free(dp);
        }
        if (err != ORC_OK) break;
        for (long i = 0; i < Nq; ++i) {
            if (L) L[(size_t)bh * Nq + i] = m[i] + log(l[i]);
            if (D_out) D_out[(size_t)bh * Nq + i] = D[i];
        }
        if (dk || dv) {
#pragma omp parallel
            {
                double *gk = (double *)malloc(sizeof(double) * (size_t)d);
                double *gv = (double *)malloc(sizeof(double) * (size_t)d);
                if (!gk || !gv) {
#pragma omp atomic write
                    err = ORC_ENOMEM;
                }
#pragma omp for schedule(dynamic, 8)
                for (long j = 0; j < Nk; ++j) {
                    if (!gk || !gv) continue;
                    key_grads(qh, kh, vh, doh, Nq, Nk, d, causal, scale, j, m, l, D, gk, gv);
                    if (dk) memcpy(dk + hk + (size_t)j * d, gk, sizeof(double) * (size_t)d);
                    if (dv) memcpy(dv + hk + (size_t)j * d, gv, sizeof(double) * (size_t)d);
                }
                free(gk);
                free(gv);
            }
        }
    }
    free(m); free(l); free(D);
    return err;
}

int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dO, long BH,
                    long N, long d, int causal, double scale, double *o, double *L, double *dq,
                    double *dk, double *dv, double *D_out) {
    return oracle_attn_bwd_qk(q, k, v, dO, BH, N, N, d, causal, scale, o, L, dq, dk, dv, D_out);
}

/*
 * Selected query rows only, each in O(N d): for n pairs (bh_sel[r], row_sel[r])
 * write o[r][d], L[r], and when dO != NULL also dq[r][d] and D[r].
 */
int oracle_attn_rows(const double *q, const double *k, const double *v, const double *dO, long BH,
                     long N, long d, int causal, double scale, long n, const long *bh_sel,
                     const long *row_sel, double *o, double *L, double *dq, double *D) {
    if (check_args(q, k, v, BH, N, N, d) || n < 0 || (n > 0 && (!bh_sel || !row_sel)))
        return ORC_EINVAL;
    for (long r = 0; r < n; ++r)
        if (bh_sel[r] < 0 || bh_sel[r] >= BH || row_sel[r] < 0 || row_sel[r] >= N)
            return ORC_EINVAL;
    int err = ORC_OK;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        double *dp = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!p || !dp) {
#pragma omp atomic write
            err = ORC_ENOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n; ++r) {
            if (!p || !dp) continue;
            const size_t h = (size_t)bh_sel[r] * N * d;
            double m, l, Dr = 0.0;
            query_row(q + h, k + h, v + h, dO ? dO + h : NULL, N, N, d, causal, scale, row_sel[r],
                      p, dp, o ? o + (size_t)r * d : NULL, &m, &l, &Dr,
                      (dO && dq) ? dq + (size_t)r * d : NULL);
            if (L) L[r] = m + log(l);
            if (D) D[r] = Dr;
        }
        free(p);
        free(dp);
    }
    return err;
}

/*
 * Selected keys only: for n pairs (bh_sel[r], key_sel[r]) write dk[r][d] and dv[r][d].
 * The row statistics of every row that sees one of the selected keys are computed
 * first, once per distinct head (in causal mode only rows i >= the smallest selected
 * key, which makes keys near the end of a long sequence cheap).
 */
int oracle_attn_keys(const double *q, const double *k, const double *v, const double *dO, long BH,
                     long N, long d, int causal, double scale, long n, const long *bh_sel,
                     const long *key_sel, double *dk, double *dv) {
    if (check_args(q, k, v, BH, N, N, d) || !dO || n < 0 || (n > 0 && (!bh_sel || !key_sel)))
        return ORC_EINVAL;
    for (long r = 0; r < n; ++r)
        if (bh_sel[r] < 0 || bh_sel[r] >= BH || key_sel[r] < 0 || key_sel[r] >= N)
            return ORC_EINVAL;
    if (n == 0) return ORC_OK;
    double *m = (double *)malloc(sizeof(double) * (size_t)N);
    double *l = (double *)malloc(sizeof(double) * (size_t)N);
    double *D = (double *)malloc(sizeof(double) * (size_t)N);
    char *done = (char *)calloc((size_t)n, 1);
    if (!m || !l || !D || !done) {
        free(m); free(l); free(D); free(done);
        return ORC_ENOMEM;
    }
    int err = ORC_OK;
    for (long r0 = 0; r0 < n && err == ORC_OK; ++r0) {
        if (done[r0]) continue;
        const long bh = bh_sel[r0];
        long j_min = N;
        for (long r = r0; r < n; ++r)
            if (bh_sel[r] == bh && key_sel[r] < j_min) j_min = key_sel[r];
        const size_t h = (size_t)bh * N * d;
        err = head_row_stats(q + h, k + h, v + h, dO + h, N, d, causal, scale, j_min, m, l, D);
        if (err != ORC_OK) break;
#pragma omp parallel for schedule(dynamic, 1)
        for (long r = r0; r < n; ++r) {
            if (bh_sel[r] != bh) continue;
            key_grads(q + h, k + h, v + h, dO + h, N, N, d, causal, scale, key_sel[r], m, l, D,
                      dk + (size_t)r * d, dv + (size_t)r * d);
            done[r] = 1;
        }
    }
    free(m); free(l); free(D); free(done);
    return err;
}

/*
 * ----------------------------------------------------------------- windowed masks
 * Local ("sliding window") attention: query i sees the keys j with
 *     i + off - wl <= j <= i + off + wr,      off = Nk - Nq,
 * clipped to [0, Nk), where a negative wl or wr leaves that side unbounded. So
 * (wl, wr) = (-1, -1) is unmasked attention and (-1, 0) the bottom-right causal mask
 * above. A row whose range is empty has O = 0, L = -inf, dQ = 0, D = 0. (A reading:
 * josueisai.com "flash-attention", section "Que ganas y que no", names window
 * attention as what to combine the method with for very long sequences but does not
 * define it; this is the usual left/right window.) These functions are separate from
 * the ones above so that those stay as they are; they follow the same three steps over
 * the row's key range [lo, hi).
 */
static void window_range(long i, long Nq, long Nk, long wl, long wr, long *lo, long *hi) {
    const long c = i + (Nk - Nq);
    long a = wl < 0 ? 0 : c - wl;
    long b = wr < 0 ? Nk : c + wr + 1;
    if (a < 0) a = 0;
    if (b > Nk) b = Nk;
    if (b < a) b = a;
    *lo = a;
    *hi = b;
}

/* One query row over keys [lo, hi): P_i (in p, indexed from lo), O_i, m_i, l_i and,
 * with doi, D_i and dQ_i. */
static void window_row(const double *qi, const double *kh, const double *vh, const double *doi,
                       long lo, long hi, long d, double scale, double *p, double *dp,
                       double *o_i, double *m_i, double *l_i, double *D_i, double *dq_i) {
    const long n = hi - lo;
    score_row(qi, kh + lo * d, n, d, scale, p);
    softmax_row(p, n, m_i, l_i);
    if (o_i) weighted_rows(p, vh + lo * d, n, d, o_i);
    if (!doi) return;
    double D = 0.0;
    for (long j = 0; j < n; ++j) {
        const double *vj = vh + (lo + j) * d;
        double acc = 0.0;
        for (long t = 0; t < d; ++t) acc += doi[t] * vj[t];
        dp[j] = acc;
        D += p[j] * acc;
    }
    *D_i = D;
    if (dq_i) {
        for (long j = 0; j < n; ++j) dp[j] = p[j] * (dp[j] - D);
        weighted_rows(dp, kh + lo * d, n, d, dq_i);
        for (long t = 0; t < d; ++t) dq_i[t] *= scale;
    }
}

/* Forward and backward with a window (o, L, dq, dk, dv, D may each be NULL; dO may be
 * NULL for the forward alone). Shapes as oracle_attn_bwd_qk. */
int oracle_attn_window(const double *q, const double *k, const double *v, const double *dO,
                       long BH, long Nq, long Nk, long d, long wl, long wr, double scale,
                       double *o, double *L, double *dq, double *dk, double *dv, double *D_out) {
    if (check_args(q, k, v, BH, Nq, Nk, d)) return ORC_EINVAL;
    if ((dq || dk || dv || D_out) && !dO) return ORC_EINVAL;
    if (Nq == 0 || Nk == 0 || BH == 0) return ORC_OK;
    double *m = (double *)malloc(sizeof(double) * (size_t)Nq);
    double *l = (double *)malloc(sizeof(double) * (size_t)Nq);
    double *D = (double *)malloc(sizeof(double) * (size_t)Nq);
    double *p = (double *)malloc(sizeof(double) * (size_t)Nk);
    double *dp = (double *)malloc(sizeof(double) * (size_t)Nk);
    if (!m || !l || !D || !p || !dp) {
        free(m); free(l); free(D); free(p); free(dp);
        return ORC_ENOMEM;
    }
    for (long bh = 0; bh < BH; ++bh) {
        const size_t hq = (size_t)bh * Nq * d, hk = (size_t)bh * Nk * d;
        const double *qh = q + hq, *kh = k + hk, *vh = v + hk;
        const double *doh = dO ? dO + hq : NULL;
        for (long i = 0; i < Nq; ++i) {
            long lo, hi;
            window_range(i, Nq, Nk, wl, wr, &lo, &hi);
            D[i] = 0.0;
            window_row(qh + i * d, kh, vh, doh ? doh + i * d : NULL, lo, hi, d, scale, p, dp,
                       o ? o + hq + (size_t)i * d : NULL, &m[i], &l[i], &D[i],
                       dq ? dq + hq + (size_t)i * d : NULL);
            if (L) L[(size_t)bh * Nq + i] = m[i] + log(l[i]);
            if (D_out) D_out[(size_t)bh * Nq + i] = D[i];
        }
        if (!dk && !dv) continue;
        /* dK_j, dV_j: the rows whose range holds key j */
        for (long j = 0; j < Nk; ++j) {
            double *gk = dk ? dk + hk + (size_t)j * d : NULL;
            double *gv = dv ? dv + hk + (size_t)j * d : NULL;
            for (long t = 0; t < d; ++t) {
                if (gk) gk[t] = 0.0;
                if (gv) gv[t] = 0.0;
            }
            const double *kj = kh + j * d, *vj = vh + j * d;
            for (long i = 0; i < Nq; ++i) {
                long lo, hi;
                window_range(i, Nq, Nk, wl, wr, &lo, &hi);
                if (j < lo || j >= hi) continue;
                const double *qi = qh + i * d, *doi = doh + i * d;
                double s = 0.0, dpv = 0.0;
                for (long t = 0; t < d; ++t) {
                    s += qi[t] * kj[t];
                    dpv += doi[t] * vj[t];
                }
                s *= scale;
                const double P = exp(s - m[i]) / l[i];
                const double dS = P * (dpv - D[i]);
                for (long t = 0; t < d; ++t) {
                    if (gv) gv[t] += P * doi[t];
                    if (gk) gk[t] += scale * dS * qi[t];
                }
            }
        }
    }
    free(m); free(l); free(D); free(p); free(dp);
    return ORC_OK;
}
