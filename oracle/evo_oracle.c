/*
 * Float64 CPU oracle for the biased-attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the GPU path computes.  It shares no code, header, table
 * or helper with the CUDA library; only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg call it.
 *
 * What it computes (DeepSpeed DS4Sci_EvoformerAttention guide, hmyw.cn:
 * section 4, the unit test's attention_reference, softmax(Q K^T * scale +
 * sum of biases) V; section 5.2, the bias shapes [B, N, 1, 1, S] and
 * [B, 1, H, S, S]; section 5.4, the per-row log-sum-exp that the forward
 * kernel also returns).  For one (b, n, h) slice and one query row i:
 *
 *     t_j    = (sum_d q[i,d] * k[j,d]) / sqrt(D) + mask[j] + pair[i,j]
 *     m      = max_j t_j
 *     w_j    = exp(t_j - m)
 *     l      = sum_j w_j
 *     o[i,:] = sum_j (w_j / l) * v[j,:]
 *     lse[i] = m + log(l)
 *
 * Readings where the guide is silent: the scale is 1/sqrt(D) and applies to
 * Q K^T only; the biases are added; the pair bias is indexed [query i, key j];
 * when every t_j of a row is -inf the row has no defined softmax and the
 * oracle returns o = 0, lse = -inf.  Every sum runs in index order in double;
 * build with -ffp-contract=off so no fused multiply-add changes the rounding.
 *
 * Parity pins (tests/test_oracle.py): a brute-force pure-Python softmax
 * without max subtraction, hand-derived closed forms (tests/golden/), shift,
 * permutation and affine invariants, and float64 scaled_dot_product_attention
 * with an additive float mask.
 *
 * Backward pass.  The guide (section 1 and the "FlashAttention-style
 * backward" part of section 5.4) states that the backward kernel returns the
 * gradients of Q, K, V and of whichever biases the caller needs, recomputing
 * the attention weights instead of storing them, with the per-row quantity
 * delta as an intermediate.  It prints no formula; the oracle is the chain
 * rule of the forward formula above, for an upstream gradient dO of O, per
 * (b, n, h) slice:
 *
 *     p_ij    = exp(t_ij - lse_i)                (the softmax weights)
 *     dp_ij   = sum_d dO[i,d] * v[j,d]
 *     delta_i = sum_j p_ij * dp_ij               (equals sum_d dO[i,d] o[i,d])
 *     dt_ij   = p_ij * (dp_ij - delta_i)         (gradient of the logit t_ij)
 *     dq[i,:] = sum_j dt_ij * k[j,:] / sqrt(D)
 *     dk[j,:] = sum_i dt_ij * q[i,:] / sqrt(D)
 *     dv[j,:] = sum_i p_ij * dO[i,:]
 *
 * and, because the mask is broadcast over heads and query rows and the pair
 * bias over n, dmask[b,n,j] = sum_h sum_i dt_ij and dpair[b,h,i,j] =
 * sum_n dt_ij.  The C side returns, per slice, dq, dk, dv and the column
 * sums sum_i dt_ij, and accumulates dt into one [S, S] matrix per pair-bias
 * matrix; the Python side adds the column sums over heads.  A row with no
 * finite logit has p = 0 and so contributes nothing.  Backward pins
 * (tests/test_oracle_bwd.py): central finite differences of the forward
 * oracle, float64 autograd of scaled_dot_product_attention, closed forms and
 * invariants.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* One query row of one slice.  t is caller scratch of length S. */
static void oracle_row(int64_t i, int64_t S, int64_t D,
                       const double* q, const double* k, const double* v,
                       const double* mask, const double* pair,
                       double* t, double* o_row, double* lse_row)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    double m = -INFINITY;
    for (int64_t j = 0; j < S; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d)
            dot += q[i * D + d] * k[j * D + d];
        double tj = dot * inv_sqrt_d;
        if (mask) tj += mask[j];
        if (pair) tj += pair[i * S + j];
        t[j] = tj;
        if (tj > m) m = tj;
    }
    if (m == -INFINITY) {            /* no finite logit: empty softmax */
        for (int64_t d = 0; d < D; ++d) o_row[d] = 0.0;
        *lse_row = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int64_t j = 0; j < S; ++j) {
        t[j] = exp(t[j] - m);        /* t now holds w_j */
        l += t[j];
    }
    for (int64_t d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int64_t j = 0; j < S; ++j)
            acc += (t[j] / l) * v[j * D + d];
        o_row[d] = acc;
    }
    *lse_row = m + log(l);
}

/*
 * Batched entry: ns independent slices, each with contiguous [S, D] q, k, v
 * and outputs o [S, D], lse [S].  mask is an array of [S] rows selected per
 * slice by mask_row[s] (NULL mask = no mask bias); pair is an array of [S, S]
 * matrices selected per slice by pair_mat[s] (NULL pair = no pair bias).
 * nthreads <= 0 uses the OpenMP default.  Returns 0, or -1 on a bad argument
 * or allocation failure.
 */
int evo_oracle_slices(int64_t ns, int64_t S, int64_t D,
                      const double* q, const double* k, const double* v,
                      const double* mask, const int64_t* mask_row,
                      const double* pair, const int64_t* pair_mat,
                      double* o, double* lse, int nthreads)
{
    if (ns < 0 || S < 0 || D <= 0) return -1;
    if (!q || !k || !v || !o || !lse) return -1;
    if ((mask && !mask_row) || (pair && !pair_mat)) return -1;
    if (ns == 0 || S == 0) return 0;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
    #pragma omp parallel num_threads(nthreads) reduction(|:failed)
#endif
    {
        double* t = (double*)malloc((size_t)S * sizeof(double));
        if (!t) {
            failed = 1;
        } else {
#ifdef _OPENMP
            #pragma omp for schedule(dynamic)
#endif
            for (int64_t s = 0; s < ns; ++s) {
                const double* qs = q + s * S * D;
                const double* ks = k + s * S * D;
                const double* vs = v + s * S * D;
                const double* ms = mask ? mask + mask_row[s] * S : NULL;
                const double* ps = pair ? pair + pair_mat[s] * S * S : NULL;
                for (int64_t i = 0; i < S; ++i)
                    oracle_row(i, S, D, qs, ks, vs, ms, ps, t,
                               o + (s * S + i) * D, lse + s * S + i);
            }
            free(t);
        }
    }
    return failed ? -1 : 0;
}

/* Threads the batched entry would use by default (for reporting). */
int evo_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Backward, one slice.  p and dt are caller scratch of S * S doubles each;
 * lse is scratch of S doubles.  Writes dq, dk, dv ([S, D]) and colsum ([S]);
 * adds dt into dpair ([S, S]) when dpair is not NULL.
 */
static void oracle_bwd_slice(int64_t S, int64_t D,
                             const double* q, const double* k, const double* v,
                             const double* mask, const double* pair, const double* dO,
                             double* p, double* dt, double* lse,
                             double* dq, double* dk, double* dv, double* colsum,
                             double* dpair)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    /* the logits and each row's log-sum-exp */
    for (int64_t i = 0; i < S; ++i) {
        double m = -INFINITY;
        for (int64_t j = 0; j < S; ++j) {
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d)
                dot += q[i * D + d] * k[j * D + d];
            double tij = dot * inv_sqrt_d;
            if (mask) tij += mask[j];
            if (pair) tij += pair[i * S + j];
            p[i * S + j] = tij;
            if (tij > m) m = tij;
        }
        if (m == -INFINITY) {
            lse[i] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int64_t j = 0; j < S; ++j)
            l += exp(p[i * S + j] - m);
        lse[i] = m + log(l);
    }
    /* weights, dp, delta and the logit gradient, row by row */
    for (int64_t i = 0; i < S; ++i) {
        if (lse[i] == -INFINITY) {
            for (int64_t j = 0; j < S; ++j) {
                p[i * S + j] = 0.0;
                dt[i * S + j] = 0.0;
            }
            continue;
        }
        double delta = 0.0;
        for (int64_t j = 0; j < S; ++j) {
            double pij = exp(p[i * S + j] - lse[i]);
            double dp = 0.0;
            for (int64_t d = 0; d < D; ++d)
                dp += dO[i * D + d] * v[j * D + d];
            p[i * S + j] = pij;
            dt[i * S + j] = dp;          /* holds dp until delta is known */
            delta += pij * dp;
        }
        for (int64_t j = 0; j < S; ++j)
            dt[i * S + j] = p[i * S + j] * (dt[i * S + j] - delta);
    }
    for (int64_t i = 0; i < S; ++i)
        for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t j = 0; j < S; ++j)
                acc += dt[i * S + j] * k[j * D + d];
            dq[i * D + d] = acc * inv_sqrt_d;
        }
    for (int64_t j = 0; j < S; ++j) {
        for (int64_t d = 0; d < D; ++d) {
            double acck = 0.0, accv = 0.0;
            for (int64_t i = 0; i < S; ++i) {
                acck += dt[i * S + j] * q[i * D + d];
                accv += p[i * S + j] * dO[i * D + d];
            }
            dk[j * D + d] = acck * inv_sqrt_d;
            dv[j * D + d] = accv;
        }
        double cs = 0.0;
        for (int64_t i = 0; i < S; ++i)
            cs += dt[i * S + j];
        colsum[j] = cs;
    }
    if (dpair)
        for (int64_t e = 0; e < S * S; ++e)
            dpair[e] += dt[e];
}

/*
 * Batched backward over ns slices laid out as in evo_oracle_slices, with the
 * upstream gradient dO ([S, D] per slice).  Outputs dq, dk, dv ([S, D] per
 * slice) and colsum ([S] per slice: sum over query rows of the logit
 * gradient).  dpair, when not NULL, is an array of npair [S, S] matrices set
 * to the sum of the logit gradients of the slices that read pair matrix
 * pair_mat[s] (it requires pair); the slices of one matrix are added in
 * index order, so the result does not depend on the thread count.  Returns
 * 0, or -1 on a bad argument or allocation failure.
 */
int evo_oracle_bwd_slices(int64_t ns, int64_t S, int64_t D,
                          const double* q, const double* k, const double* v,
                          const double* mask, const int64_t* mask_row,
                          const double* pair, const int64_t* pair_mat, int64_t npair,
                          const double* dO,
                          double* dq, double* dk, double* dv, double* colsum,
                          double* dpair, int nthreads)
{
    if (ns < 0 || S < 0 || D <= 0 || npair < 0) return -1;
    if (!q || !k || !v || !dO || !dq || !dk || !dv || !colsum) return -1;
    if ((mask && !mask_row) || (pair && !pair_mat) || (dpair && !pair)) return -1;
    if (dpair)
        for (int64_t e = 0; e < npair * S * S; ++e) dpair[e] = 0.0;
    if (ns == 0 || S == 0) return 0;
    /* with dpair: one task per pair matrix (its slices in order); else one per slice */
    const int64_t tasks = dpair ? npair : ns;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
    #pragma omp parallel num_threads(nthreads) reduction(|:failed)
#endif
    {
        double* p = (double*)malloc((size_t)(2 * S * S + S) * sizeof(double));
        if (!p) {
            failed = 1;
        } else {
            double* dt = p + S * S;
            double* lse = dt + S * S;
#ifdef _OPENMP
            #pragma omp for schedule(dynamic)
#endif
            for (int64_t task = 0; task < tasks; ++task) {
                for (int64_t s = dpair ? 0 : task; s < (dpair ? ns : task + 1); ++s) {
                    if (dpair && pair_mat[s] != task) continue;
                    oracle_bwd_slice(S, D, q + s * S * D, k + s * S * D, v + s * S * D,
                                     mask ? mask + mask_row[s] * S : NULL,
                                     pair ? pair + pair_mat[s] * S * S : NULL,
                                     dO + s * S * D, p, dt, lse,
                                     dq + s * S * D, dk + s * S * D, dv + s * S * D,
                                     colsum + s * S,
                                     dpair ? dpair + task * S * S : NULL);
                }
            }
            free(p);
        }
    }
    return failed ? -1 : 0;
}

/*
 * The logit gradient of selected query rows: for each of nr (slice, row)
 * pairs, dt[r, :] = p_i. * (dp_i. - delta_i) of query row_i[r] of slice
 * row_slice[r], slices laid out as in evo_oracle_bwd_slices.  Used to check
 * single rows of the pair-bias gradient (a sum over every n) at sizes where
 * whole slices are too slow.  Returns 0 or -1.
 */
int evo_oracle_bwd_rows(int64_t ns, int64_t S, int64_t D,
                        const double* q, const double* k, const double* v,
                        const double* mask, const int64_t* mask_row,
                        const double* pair, const int64_t* pair_mat,
                        const double* dO, int64_t nr, const int64_t* row_slice,
                        const int64_t* row_i, double* dt, int nthreads)
{
    if (ns < 0 || S < 0 || D <= 0 || nr < 0) return -1;
    if (!q || !k || !v || !dO || !dt || (nr && (!row_slice || !row_i))) return -1;
    if ((mask && !mask_row) || (pair && !pair_mat)) return -1;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
    #pragma omp parallel for num_threads(nthreads) schedule(dynamic) reduction(|:failed)
#endif
    for (int64_t r = 0; r < nr; ++r) {
        const int64_t s = row_slice[r], i = row_i[r];
        if (s < 0 || s >= ns || i < 0 || i >= S) { failed = 1; continue; }
        const double* qs = q + s * S * D;
        const double* ks = k + s * S * D;
        const double* vs = v + s * S * D;
        const double* ms = mask ? mask + mask_row[s] * S : NULL;
        const double* ps = pair ? pair + pair_mat[s] * S * S + i * S : NULL;
        const double* go = dO + s * S * D + i * D;
        double* out = dt + r * S;
        double m = -INFINITY;
        for (int64_t j = 0; j < S; ++j) {
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d)
                dot += qs[i * D + d] * ks[j * D + d];
            double tij = dot * inv_sqrt_d;
            if (ms) tij += ms[j];
            if (ps) tij += ps[j];
            out[j] = tij;
            if (tij > m) m = tij;
        }
        if (m == -INFINITY) {
            for (int64_t j = 0; j < S; ++j) out[j] = 0.0;
            continue;
        }
        double l = 0.0;
        for (int64_t j = 0; j < S; ++j)
            l += exp(out[j] - m);
        const double lse = m + log(l);
        double delta = 0.0;
        double* dp = (double*)malloc((size_t)S * sizeof(double));
        if (!dp) { failed = 1; continue; }
        for (int64_t j = 0; j < S; ++j) {
            double acc = 0.0;
            for (int64_t d = 0; d < D; ++d)
                acc += go[d] * vs[j * D + d];
            dp[j] = acc;
            out[j] = exp(out[j] - lse);
            delta += out[j] * acc;
        }
        for (int64_t j = 0; j < S; ++j)
            out[j] = out[j] * (dp[j] - delta);
        free(dp);
    }
    return failed ? -1 : 0;
}
