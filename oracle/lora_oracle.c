/*
 * fp64 CPU oracle of the heterogeneous-batch LoRA adapter branch, in plain C.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, by the smoke check and by the
 * CPU-baseline / reference legs of the benchmark.  The product library never
 * links, loads or calls it, and it shares no source with the CUDA path.
 *
 * What it computes (page "Multi-LoRA Serving in Production", llms.blog,
 * section "The Mathematical Anatomy of Heterogeneous Batches", equation
 * Y = X W0 + (alpha/r)(X A) B, with sequence i of the batch using its own
 * A_i [d_in x r_i] and B_i [r_i x d_out]; section "Segmented Gather
 * Matrix-Vector Multiplication (SGMV)" names the two steps shrink v = x A and
 * expand y += (alpha/r) v B):
 *
 *   for every token t with i = ids[t] >= 0:
 *     v[k]    = sum_j X[t][j] * A_i[j][k]              k < r_i
 *     Y[t][c] = Y_base[t][c] + s_i * sum_k v[k] * B_i[k][c]
 *
 * in double precision, on the same bf16-valued inputs as the GPU.  A token
 * with id = -1 keeps Y_base (a base-model request); an id outside [-1, S) or
 * naming an empty slot keeps Y_base and sets an error bit.  Tokens are
 * independent, so the loop over tokens is split across OpenMP threads.
 */
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_ERR_BAD_ID 1
#define ORACLE_ERR_EMPTY_SLOT 2
/* bit 4: host allocation failure inside the oracle itself */

/* A_all / B_all hold every slot's logical matrices back to back:
 * slot i's A starts at A_all + a_off[i] ([d_in][r_i] row-major) and its B at
 * B_all + b_off[i] ([r_i][d_out] row-major).  Y_out is [T][d_out] doubles.
 * Returns the OR of the error bits.  nthreads <= 0 lets OpenMP choose. */
int oracle_lora_apply(const float *X, int T, int d_in, int d_out,
                      const float *Y_base, const int32_t *ids, int S,
                      const int32_t *ranks, const float *scales,
                      const float *A_all, const int64_t *a_off,
                      const float *B_all, const int64_t *b_off,
                      double *Y_out, int nthreads)
{
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int t = 0; t < T; ++t) {
        const float *yb = Y_base + (int64_t)t * d_out;
        double *y = Y_out + (int64_t)t * d_out;
        for (int c = 0; c < d_out; ++c) y[c] = (double)yb[c];
        int i = ids[t];
        if (i == -1) continue;
        if (i < -1 || i >= S) { err |= ORACLE_ERR_BAD_ID; continue; }
        int r = ranks[i];
        if (r <= 0) { err |= ORACLE_ERR_EMPTY_SLOT; continue; }
        const float *x = X + (int64_t)t * d_in;
        const float *A = A_all + a_off[i];
        const float *B = B_all + b_off[i];
        double *v = (double *)calloc((size_t)r, sizeof(double));
        if (!v) { err |= 4; continue; }
        /* shrink: v = x A_i */
        for (int j = 0; j < d_in; ++j) {
            double xj = (double)x[j];
            for (int k = 0; k < r; ++k) v[k] += xj * (double)A[(int64_t)j * r + k];
        }
        /* expand-add: y += s_i * (v B_i); acc[c] sums over k in ascending order */
        double s = (double)scales[i];
        double *acc = (double *)calloc((size_t)d_out, sizeof(double));
        if (!acc) { free(v); err |= 4; continue; }
        for (int k = 0; k < r; ++k) {
            const float *Bk = B + (int64_t)k * d_out;
            for (int c = 0; c < d_out; ++c) acc[c] += v[k] * (double)Bk[c];
        }
        for (int c = 0; c < d_out; ++c) y[c] += s * acc[c];
        free(acc);
        free(v);
    }
    return err;
}

/* Number of threads OpenMP would use for the loop above. */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
