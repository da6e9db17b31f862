/*
 * Exact scaled dot-product attention, forward and backward passes: the fp64
 * CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the checker of the CUDA path, not
 * part of it. Only the test suite, the smoke check and the benchmark's CPU
 * baseline may load it. It shares no code, header, table or helper with the
 * CUDA library, and the CUDA library never calls it.
 *
 * What it computes is the plain definition, written out:
 *
 *   Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V
 *     ("week17 efficiency attention", recall of scaled dot-product attention;
 *      "Quadratic cost and efficient attention", section "Where the n^2 hides")
 *
 * with the row softmax taken only over the keys a mask allows. For query row
 * i the allowed key set A(i) is
 *   none   : every key j < n
 *   causal : j <= i  (the triu(..., 1) mask of naive_attention in
 *            "Efficient Transformers ...", section "Family 3")
 *   window : max(0, i - w) <= j <= i  (the causal sliding-window mask code on
 *            "week17 efficiency attention", section on local attention)
 *   symmetric window (causal = 0, w >= 0) :
 *            max(0, i - w) <= j <= min(n - 1, i + w)  (the same page's local
 *            attention: each token attends to its w nearest neighbours on
 *            either side)
 *   block-local (block b > 0, no window) : floor(j/b) is floor(i/b) or
 *            floor(i/b) - 1, and j <= i as well when causal (the block-sparse
 *            pattern of "Sparse & sub-quadratic attention", section "Escape 1":
 *            a token sees the keys of its own block and of the block before)
 * Then, all in fp64 over the bf16-decoded inputs,
 *   s_ij  = scale * sum_c q_ic k_jc          for j in A(i)
 *   M_i   = max_{j in A(i)} s_ij
 *   Z_i   = sum_{j in A(i)} exp(s_ij - M_i)
 *   O_i   = sum_{j in A(i)} exp(s_ij - M_i) v_j / Z_i
 *   LSE_i = M_i + ln Z_i        (natural-log units)
 *
 * It is a two-pass softmax over an explicit per-row mask vector; it never
 * forms the n x n matrix, so a single row of any size can be checked.
 * There is no tiling, no online rescaling and no reordering beyond the
 * definition. OpenMP spreads independent rows over host cores.
 *
 * Grouped-query attention ("week17 efficiency attention", MQA / GQA
 * section): K and V have H_kv heads, H_kv divides H, and query head h reads
 * key/value head h / (H / H_kv); H_kv = 1 is multi-query attention and
 * H_kv = H is ordinary multi-head attention.
 *
 * The "identity" kernel (ORACLE_KERNEL_IDENTITY) replaces the softmax weight
 * exp(s_ij - M_i)/Z_i by the raw score s_ij and uses no mask: it yields the
 * unnormalised product (Q K^T) V * scale, which the associativity identity
 * (Q K^T) V = Q (K^T V) on "Sparse & sub-quadratic attention" (section
 * "Escape 2 - change the operator") pins from outside.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_KERNEL_SOFTMAX 0
#define ORACLE_KERNEL_IDENTITY 1

/* bf16 is the upper half of an IEEE binary32: widen exactly, then to fp64. */
static double bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* sum_c a[c*sa] * b[c*sb], c = 0 .. len-1, in order. */
double oracle_dot_f64(const double *a, int64_t sa, const double *b, int64_t sb, int64_t len)
{
    double acc = 0.0;
    for (int64_t c = 0; c < len; ++c)
        acc += a[c * sa] * b[c * sb];
    return acc;
}

/*
 * C[m x n] = op(A) op(B), row-major, op(X) = X or X^T.
 * A is stored m x k (ta = 0) or k x m (ta = 1); B is stored k x n (tb = 0)
 * or n x k (tb = 1). Built from oracle_dot_f64 so that the contraction used
 * by the attention rows is the one the associativity test exercises.
 */
int oracle_matmul_f64(int64_t m, int64_t n, int64_t k, const double *A, int ta,
                      const double *B, int tb, double *C)
{
    if (m < 0 || n < 0 || k < 0 || (!A && m * k != 0) || (!B && k * n != 0) || (!C && m * n != 0))
        return 1;
    for (int64_t i = 0; i < m; ++i) {
        const double *arow = ta ? A + i : A + i * k;
        int64_t sa = ta ? m : 1;
        for (int64_t j = 0; j < n; ++j) {
            const double *bcol = tb ? B + j * k : B + j;
            int64_t sb = tb ? 1 : n;
            C[i * n + j] = oracle_dot_f64(arow, sa, bcol, sb, k);
        }
    }
    return 0;
}

/* Is key j in A(i)? The one definition of the masks (see the top of the file). */
static int allowed_pair(int64_t i, int64_t j, int causal, int64_t window, int64_t block)
{
    if (causal && j > i)
        return 0;
    if (block > 0) {
        const int64_t bi = i / block, bj = j / block;
        return bj == bi || bj == bi - 1;
    }
    if (window >= 0 && j < i - window)
        return 0;
    if (!causal && window >= 0 && j > i + window)
        return 0;
    return 1;
}

/* Explicit mask row: allowed[j] = 1 iff key j is in A(i). */
int oracle_mask_row(int64_t n, int64_t i, int causal, int64_t window, int64_t block, unsigned char *allowed)
{
    if (n < 0 || i < 0 || i >= n || !allowed || (block > 0 && window >= 0))
        return 1;
    for (int64_t j = 0; j < n; ++j)
        allowed[j] = (unsigned char)allowed_pair(i, j, causal, window, block);
    return 0;
}

/*
 * Attention for a list of rows, grouped-query form.
 *   q       : bf16 bit patterns, contiguous [B, H, n, d]
 *   k, v    : bf16 bit patterns, contiguous [B, Hkv, n, d]; Hkv divides H
 *   rows    : flat row ids r = (b*H + h)*n + i, nrows of them
 *   o       : nrows x d   fp64 output (row-major, in the order of rows)
 *   lse     : nrows       fp64 output (may be NULL)
 *   weights : nrows x n   fp64 normalised weights, 0 where masked (may be NULL)
 *   kernel  : ORACLE_KERNEL_SOFTMAX or ORACLE_KERNEL_IDENTITY
 * Returns 0 on success, nonzero on bad input.
 */
int oracle_attn_rows_gqa_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             int64_t B, int64_t H, int64_t Hkv, int64_t n, int64_t d,
                             double scale, int causal, int64_t window, int64_t block, int kernel,
                             const int64_t *rows, int64_t nrows,
                             double *o, double *lse, double *weights)
{
    if (block > 0 && window >= 0)
        return 1;
    if (!q || !k || !v || !o || (!rows && nrows) || B <= 0 || H <= 0 || n <= 0 || d <= 0)
        return 1;
    if (Hkv <= 0 || H % Hkv != 0)
        return 1;
    if (kernel != ORACLE_KERNEL_SOFTMAX && kernel != ORACLE_KERNEL_IDENTITY)
        return 1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= B * H * n)
            return 1;

    int bad = 0;
#pragma omp parallel
    {
        double *qi = (double *)malloc(sizeof(double) * (size_t)d);
        double *kj = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        unsigned char *allowed = (unsigned char *)malloc((size_t)n);
        if (!qi || !kj || !s || !acc || !allowed) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t bh = rows[r] / n;
                int64_t i = rows[r] % n;
                /* key/value head of query head h = bh % H in batch b = bh / H */
                int64_t bkv = (bh / H) * Hkv + (bh % H) / (H / Hkv);
                const uint16_t *Kh = k + bkv * n * d;
                const uint16_t *Vh = v + bkv * n * d;
                for (int64_t c = 0; c < d; ++c)
                    qi[c] = bf16_to_f64(q[(bh * n + i) * d + c]);

                if (kernel == ORACLE_KERNEL_IDENTITY) {
                    for (int64_t j = 0; j < n; ++j)
                        allowed[j] = 1;
                } else {
                    oracle_mask_row(n, i, causal, window, block, allowed);
                }

                /* pass 1: scores of allowed keys and their maximum */
                double M = -INFINITY;
                for (int64_t j = 0; j < n; ++j) {
                    if (!allowed[j]) {
                        s[j] = -INFINITY;
                        continue;
                    }
                    for (int64_t c = 0; c < d; ++c)
                        kj[c] = bf16_to_f64(Kh[j * d + c]);
                    s[j] = scale * oracle_dot_f64(qi, 1, kj, 1, d);
                    if (s[j] > M)
                        M = s[j];
                }

                /* pass 2: weights, normaliser and weighted sum of values */
                for (int64_t c = 0; c < d; ++c)
                    acc[c] = 0.0;
                double Z = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    if (!allowed[j])
                        continue;
                    double w = (kernel == ORACLE_KERNEL_IDENTITY) ? s[j] : exp(s[j] - M);
                    Z += w;
                    for (int64_t c = 0; c < d; ++c)
                        acc[c] += w * bf16_to_f64(Vh[j * d + c]);
                }

                if (kernel == ORACLE_KERNEL_IDENTITY) {
                    for (int64_t c = 0; c < d; ++c)
                        o[r * d + c] = acc[c];
                    if (lse)
                        lse[r] = NAN;
                    if (weights)
                        for (int64_t j = 0; j < n; ++j)
                            weights[r * n + j] = s[j];
                } else {
                    for (int64_t c = 0; c < d; ++c)
                        o[r * d + c] = acc[c] / Z;
                    if (lse)
                        lse[r] = M + log(Z);
                    if (weights)
                        for (int64_t j = 0; j < n; ++j)
                            weights[r * n + j] = allowed[j] ? exp(s[j] - M) / Z : 0.0;
                }
            }
        }
        free(qi);
        free(kj);
        free(s);
        free(acc);
        free(allowed);
    }
    return bad ? 2 : 0;
}

/* Multi-head attention (Hkv = H) for a list of rows; arguments as above. */
int oracle_attn_rows_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         int64_t B, int64_t H, int64_t n, int64_t d, double scale,
                         int causal, int64_t window, int64_t block, int kernel,
                         const int64_t *rows, int64_t nrows,
                         double *o, double *lse, double *weights)
{
    return oracle_attn_rows_gqa_f64(q, k, v, B, H, H, n, d, scale, causal, window, block, kernel,
                                    rows, nrows, o, lse, weights);
}

/* Every row of every head: o is [B, H, n, d] fp64, lse is [B, H, n] fp64. */
int oracle_attn_fwd_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        int64_t B, int64_t H, int64_t n, int64_t d, double scale,
                        int causal, int64_t window, int64_t block, double *o, double *lse)
{
    if (B <= 0 || H <= 0 || n <= 0)
        return 1;
    int64_t total = B * H * n;
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)total);
    if (!rows)
        return 2;
    for (int64_t r = 0; r < total; ++r)
        rows[r] = r;
    int rc = oracle_attn_rows_f64(q, k, v, B, H, n, d, scale, causal, window, block,
                                  ORACLE_KERNEL_SOFTMAX, rows, total, o, lse, NULL);
    free(rows);
    return rc;
}

/* Threads an OpenMP parallel region of this library uses. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ========================================================================
 * Backward pass: gradients of the attention output with respect to Q, K, V.
 *
 * The pages note that FlashAttention recomputes in the backward pass what it
 * needs instead of storing the score matrix ("Efficient Transformers ...",
 * section "Family 3"). What the backward pass computes is fixed by the
 * forward definition above and the chain rule alone: for an upstream
 * gradient dO = dL/dO, with P_ij = exp(s_ij - LSE_i) for j in A(i) (0
 * elsewhere) and s_ij = scale * q_i . k_j,
 *
 *   dV_j  = sum_i P_ij dO_i                          (O_i = sum_j P_ij v_j)
 *   dP_ij = dO_i . v_j
 *   dS_ij = P_ij (dP_ij - sum_t P_it dP_it)          (Jacobian of a row softmax)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 *
 * The row term sum_t P_it dP_it is computed as written, from the row's own
 * weights (not from O). Every sum runs over the allowed (i, j) pairs only.
 * Rows are independent for dQ; a key row j needs, for every query i that
 * attends to it, that query's LSE_i and row term, so those are computed for
 * all rows of each head that a requested key row belongs to.
 *
 * Inputs are Q, K, V, dO as [B, H, n, d], either bf16 bit patterns
 * (ORACLE_IN_BF16) or fp64 values (ORACLE_IN_F64); all arithmetic is fp64.
 * ======================================================================== */

#define ORACLE_IN_BF16 0
#define ORACLE_IN_F64 1

static double in_at(const void *p, int type, int64_t idx)
{
    return type == ORACLE_IN_F64 ? ((const double *)p)[idx] : bf16_to_f64(((const uint16_t *)p)[idx]);
}

/* One query row's softmax statistics and, if dq != NULL, its gradient.
 * qbase = (b*H + h)*n*d is the query head's offset (q, dout), kbase that of
 * its key/value head (k, v); s and dp are n-long scratch. */
static void bwd_row(const void *q, const void *k, const void *v, const void *dout, int type,
                    int64_t qbase, int64_t kbase, int64_t n, int64_t d, double scale, int causal,
                    int64_t window, int64_t block, int64_t i, unsigned char *allowed, double *s,
                    double *dp, double *lse_out, double *rowterm_out, double *dq)
{
    oracle_mask_row(n, i, causal, window, block, allowed);
    double M = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        if (!allowed[j])
            continue;
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c)
            acc += in_at(q, type, qbase + i * d + c) * in_at(k, type, kbase + j * d + c);
        s[j] = scale * acc;
        if (s[j] > M)
            M = s[j];
    }
    double Z = 0.0;
    for (int64_t j = 0; j < n; ++j)
        if (allowed[j])
            Z += exp(s[j] - M);
    const double lse = M + log(Z);
    /* dP_ij and the row term sum_j P_ij dP_ij */
    double rowterm = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        if (!allowed[j])
            continue;
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c)
            acc += in_at(dout, type, qbase + i * d + c) * in_at(v, type, kbase + j * d + c);
        dp[j] = acc;
        rowterm += exp(s[j] - lse) * acc;
    }
    if (lse_out)
        *lse_out = lse;
    if (rowterm_out)
        *rowterm_out = rowterm;
    if (dq) {
        for (int64_t c = 0; c < d; ++c)
            dq[c] = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            if (!allowed[j])
                continue;
            const double ds = exp(s[j] - lse) * (dp[j] - rowterm);
            for (int64_t c = 0; c < d; ++c)
                dq[c] += ds * in_at(k, type, kbase + j * d + c);
        }
        for (int64_t c = 0; c < d; ++c)
            dq[c] *= scale;
    }
}

/*
 * Gradients for selected rows, grouped-query form.
 *   q, dout       : [B, H, n, d];  k, v : [B, Hkv, n, d], Hkv divides H; query
 *                   head h of batch b reads key/value head b*Hkv + h/(H/Hkv)
 *                   (element type `type`)
 *   qrows (nq)    : flat query rows (b*H + h)*n + i whose dQ is wanted -> dq (nq x d)
 *   krows (nk)    : flat key rows (b*Hkv + g)*n + j whose dK, dV are wanted
 *                   -> dk, dv (nk x d each). A key/value head's gradient sums
 *                   the contributions of every query head that reads it.
 * Returns 0 on success, nonzero on bad input.
 */
int oracle_attn_bwd_rows_gqa_f64(const void *q, const void *k, const void *v, const void *dout, int type,
                                 int64_t B, int64_t H, int64_t Hkv, int64_t n, int64_t d, double scale,
                                 int causal, int64_t window, int64_t block, const int64_t *qrows,
                                 int64_t nq, const int64_t *krows, int64_t nk, double *dq, double *dk,
                                 double *dv)
{
    if (block > 0 && window >= 0)
        return 1;
    if (!q || !k || !v || !dout || B <= 0 || H <= 0 || Hkv <= 0 || n <= 0 || d <= 0)
        return 1;
    if (H % Hkv != 0)
        return 1;
    if (type != ORACLE_IN_BF16 && type != ORACLE_IN_F64)
        return 1;
    if ((nq && (!qrows || !dq)) || (nk && (!krows || !dk || !dv)) || nq < 0 || nk < 0)
        return 1;
    const int64_t G = H / Hkv;
    for (int64_t r = 0; r < nq; ++r)
        if (qrows[r] < 0 || qrows[r] >= B * H * n)
            return 1;
    for (int64_t r = 0; r < nk; ++r)
        if (krows[r] < 0 || krows[r] >= B * Hkv * n)
            return 1;

    /* query heads of the key/value heads with requested key rows, and their
     * per-row statistics */
    const int64_t nheads = B * H;
    int64_t *slot = (int64_t *)malloc(sizeof(int64_t) * (size_t)nheads);
    if (!slot)
        return 2;
    for (int64_t h = 0; h < nheads; ++h)
        slot[h] = -1;
    int64_t nstat = 0;
    for (int64_t r = 0; r < nk; ++r) {
        const int64_t kvh = krows[r] / n;             /* b*Hkv + g */
        const int64_t qh0 = (kvh / Hkv) * H + (kvh % Hkv) * G;
        for (int64_t u = 0; u < G; ++u)
            if (slot[qh0 + u] < 0)
                slot[qh0 + u] = nstat++;
    }
    int64_t *stat_head = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nstat + 1));
    double *lse = (double *)malloc(sizeof(double) * (size_t)(nstat * n + 1));
    double *rowterm = (double *)malloc(sizeof(double) * (size_t)(nstat * n + 1));
    if (!stat_head || !lse || !rowterm) {
        free(slot);
        free(stat_head);
        free(lse);
        free(rowterm);
        return 2;
    }
    for (int64_t h = 0; h < nheads; ++h)
        if (slot[h] >= 0)
            stat_head[slot[h]] = h;

    int bad = 0;
#pragma omp parallel
    {
        unsigned char *allowed = (unsigned char *)malloc((size_t)n);
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
        double *dp = (double *)malloc(sizeof(double) * (size_t)n);
        if (!allowed || !s || !dp) {
#pragma omp atomic write
            bad = 1;
        } else {
            /* 1. statistics of every row of the query heads involved */
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < nstat * n; ++t) {
                const int64_t h = stat_head[t / n], i = t % n;
                const int64_t kvh = (h / H) * Hkv + (h % H) / G;
                bwd_row(q, k, v, dout, type, h * n * d, kvh * n * d, n, d, scale, causal, window, block,
                        i, allowed, s, dp, &lse[t], &rowterm[t], NULL);
            }
            /* 2. dQ of the requested query rows */
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nq; ++r) {
                const int64_t h = qrows[r] / n, i = qrows[r] % n;
                const int64_t kvh = (h / H) * Hkv + (h % H) / G;
                bwd_row(q, k, v, dout, type, h * n * d, kvh * n * d, n, d, scale, causal, window, block,
                        i, allowed, s, dp, NULL, NULL, dq + r * d);
            }
            /* 3. dK, dV of the requested key rows: sums over the query heads
             * of the group and the queries that attend to key j, with each
             * query's own LSE and row term */
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nk; ++r) {
                const int64_t kvh = krows[r] / n, j = krows[r] % n;
                const int64_t kbase = kvh * n * d;
                const int64_t qh0 = (kvh / Hkv) * H + (kvh % Hkv) * G;
                double *gk = dk + r * d, *gv = dv + r * d;
                for (int64_t c = 0; c < d; ++c)
                    gk[c] = gv[c] = 0.0;
                for (int64_t u = 0; u < G; ++u) {
                    const int64_t h = qh0 + u;
                    const int64_t qbase = h * n * d;
                    const double *L = lse + slot[h] * n;
                    const double *R = rowterm + slot[h] * n;
                    for (int64_t i = 0; i < n; ++i) {
                        if (!allowed_pair(i, j, causal, window, block))
                            continue;
                        double sij = 0.0, dpij = 0.0;
                        for (int64_t c = 0; c < d; ++c) {
                            sij += in_at(q, type, qbase + i * d + c) * in_at(k, type, kbase + j * d + c);
                            dpij += in_at(dout, type, qbase + i * d + c) * in_at(v, type, kbase + j * d + c);
                        }
                        const double pij = exp(scale * sij - L[i]);
                        const double dsij = pij * (dpij - R[i]);
                        for (int64_t c = 0; c < d; ++c) {
                            gv[c] += pij * in_at(dout, type, qbase + i * d + c);
                            gk[c] += dsij * in_at(q, type, qbase + i * d + c);
                        }
                    }
                }
                for (int64_t c = 0; c < d; ++c)
                    gk[c] *= scale;
            }
        }
        free(allowed);
        free(s);
        free(dp);
    }
    free(slot);
    free(stat_head);
    free(lse);
    free(rowterm);
    return bad ? 2 : 0;
}

/* Multi-head form (Hkv = H); arguments as above. */
int oracle_attn_bwd_rows_f64(const void *q, const void *k, const void *v, const void *dout, int type,
                             int64_t B, int64_t H, int64_t n, int64_t d, double scale, int causal,
                             int64_t window, int64_t block, const int64_t *qrows, int64_t nq,
                             const int64_t *krows, int64_t nk, double *dq, double *dk, double *dv)
{
    return oracle_attn_bwd_rows_gqa_f64(q, k, v, dout, type, B, H, H, n, d, scale, causal, window, block,
                                        qrows, nq, krows, nk, dq, dk, dv);
}

/* ========================================================================
 * Decode against a rolling key/value cache.
 *
 * One query token per sequence attends to the keys a sliding window keeps.
 * The cache is the rolling buffer of "Beyond attention" (section "For
 * engineers -- Show the maths", worked example: a 4,096-position cache
 * serving n = 32,768, after Mistral): W slots per key/value head, position p stored
 * at slot p mod W, so after writing position t the cache holds positions
 * max(0, t - W + 1) .. t. For sequence b with query position t = pos[b] and
 * query head h (key/value head h / (H / Hkv), as for grouped-query
 * attention) the output is the plain definition over those positions:
 *   s_p  = scale * q . k(slot p mod W),  M = max_p s_p,
 *   O    = sum_p exp(s_p - M) v(slot p mod W) / sum_p exp(s_p - M),
 *   LSE  = M + ln sum_p exp(s_p - M).
 *   q      : bf16 [B, H, d];  k, v : bf16 [B, Hkv, W, d];  pos : int64 [B], >= 0
 *   o      : fp64 [B, H, d];  lse : fp64 [B, H]
 * ======================================================================== */
int oracle_attn_decode_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int64_t *pos,
                           int64_t B, int64_t H, int64_t Hkv, int64_t W, int64_t d, double scale,
                           double *o, double *lse)
{
    if (!q || !k || !v || !pos || !o || !lse || B <= 0 || H <= 0 || Hkv <= 0 || W <= 0 || d <= 0)
        return 1;
    if (H % Hkv != 0)
        return 1;
    for (int64_t b = 0; b < B; ++b)
        if (pos[b] < 0)
            return 1;
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)W);
        if (!s) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bh = 0; bh < B * H; ++bh) {
                const int64_t b = bh / H, h = bh % H;
                const int64_t kvh = b * Hkv + h / (H / Hkv);
                const int64_t t = pos[b];
                const int64_t first = (t - W + 1 > 0) ? t - W + 1 : 0;
                const int64_t count = t - first + 1;
                const uint16_t *qh = q + bh * d;
                /* pass 1: scores of the cached positions and their maximum */
                double M = -INFINITY;
                for (int64_t u = 0; u < count; ++u) {
                    const int64_t slot = (first + u) % W;
                    const uint16_t *kr = k + (kvh * W + slot) * d;
                    double acc = 0.0;
                    for (int64_t c = 0; c < d; ++c)
                        acc += bf16_to_f64(qh[c]) * bf16_to_f64(kr[c]);
                    s[u] = scale * acc;
                    if (s[u] > M)
                        M = s[u];
                }
                /* pass 2: normaliser and weighted sum of values */
                double Z = 0.0;
                for (int64_t c = 0; c < d; ++c)
                    o[bh * d + c] = 0.0;
                for (int64_t u = 0; u < count; ++u) {
                    const int64_t slot = (first + u) % W;
                    const uint16_t *vr = v + (kvh * W + slot) * d;
                    const double w = exp(s[u] - M);
                    Z += w;
                    for (int64_t c = 0; c < d; ++c)
                        o[bh * d + c] += w * bf16_to_f64(vr[c]);
                }
                for (int64_t c = 0; c < d; ++c)
                    o[bh * d + c] /= Z;
                lse[bh] = M + log(Z);
            }
        }
        free(s);
    }
    return bad ? 2 : 0;
}

/* ========================================================================
 * Decode of a few new tokens per sequence against a rolling cache.
 *
 * The same rolling buffer as above (position p in slot p mod W), now with T
 * new query tokens per sequence, at positions t_u = pos[b] - T + 1 + u for
 * u = 0 .. T-1 (pos[b] is the last of them; all T have been written to the
 * cache before the step). Token u attends causally within the new tokens and
 * to the sliding window of w earlier positions (the causal window-w mask of
 * "week17 efficiency attention", local attention section):
 *   A(u) = { p : max(0, t_u - w) <= p <= t_u },
 * so the T outputs are rows t_0 .. t_{T-1} of the causal window-w forward
 * pass over the sequence that filled the cache. Every p in A(u) is still in
 * the cache only if w + T <= W (the oldest needed position, t_0 - w, is then
 * at least pos - W + 1); the oracle rejects other arguments. T = 1 and
 * w = W - 1 is the single-token decode above.
 *   s_p  = scale * q_u . k(slot p mod W),  M = max_{p in A(u)} s_p,
 *   O    = sum_{p in A(u)} exp(s_p - M) v(slot p mod W) / sum exp(s_p - M),
 *   LSE  = M + ln sum_{p in A(u)} exp(s_p - M).
 *   q : bf16 [B, H, T, d];  k, v : bf16 [B, Hkv, W, d];  pos : int64 [B], >= T - 1
 *   o : fp64 [B, H, T, d];  lse : fp64 [B, H, T]
 * ======================================================================== */
int oracle_attn_decode_multi_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int64_t *pos,
                                 int64_t B, int64_t H, int64_t Hkv, int64_t T, int64_t W, int64_t d,
                                 int64_t window, double scale, double *o, double *lse)
{
    if (!q || !k || !v || !pos || !o || !lse || B <= 0 || H <= 0 || Hkv <= 0 || T <= 0 || W <= 0 || d <= 0)
        return 1;
    if (H % Hkv != 0 || window < 0 || window + T > W)
        return 1;
    for (int64_t b = 0; b < B; ++b)
        if (pos[b] < T - 1)
            return 1;
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(window + 1));
        if (!s) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t row = 0; row < B * H * T; ++row) {
                const int64_t bh = row / T, u = row % T;
                const int64_t b = bh / H, h = bh % H;
                const int64_t kvh = b * Hkv + h / (H / Hkv);
                const int64_t t = pos[b] - T + 1 + u;           /* this token's position */
                const int64_t first = (t - window > 0) ? t - window : 0;
                const int64_t count = t - first + 1;
                const uint16_t *qr = q + row * d;
                double M = -INFINITY;
                for (int64_t i = 0; i < count; ++i) {
                    const uint16_t *kr = k + (kvh * W + (first + i) % W) * d;
                    double acc = 0.0;
                    for (int64_t c = 0; c < d; ++c)
                        acc += bf16_to_f64(qr[c]) * bf16_to_f64(kr[c]);
                    s[i] = scale * acc;
                    if (s[i] > M)
                        M = s[i];
                }
                double Z = 0.0;
                for (int64_t c = 0; c < d; ++c)
                    o[row * d + c] = 0.0;
                for (int64_t i = 0; i < count; ++i) {
                    const uint16_t *vr = v + (kvh * W + (first + i) % W) * d;
                    const double w = exp(s[i] - M);
                    Z += w;
                    for (int64_t c = 0; c < d; ++c)
                        o[row * d + c] += w * bf16_to_f64(vr[c]);
                }
                for (int64_t c = 0; c < d; ++c)
                    o[row * d + c] /= Z;
                lse[row] = M + log(Z);
            }
        }
        free(s);
    }
    return bad ? 2 : 0;
}
