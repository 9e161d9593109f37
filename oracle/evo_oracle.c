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
