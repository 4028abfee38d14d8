/*
 * tp_mlp_oracle.c -- the oracle: a plain, slow CPU implementation of the
 * tensor-parallel two-projection MLP with every arithmetic step in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and
 * the benchmark's CPU-baseline leg load this library.  The product (the CUDA
 * library under tensor_sharded_mlp_b200/) shares no code with it and never
 * calls it.
 *
 * What it computes, and where the pages say so:
 *
 *  - "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 2) 张量并行（TP）, the worked
 *    NumPy function tensor_parallel_output: for every rank i (pairs of shards
 *    taken together; unequal counts are an error), hidden_i = act(x @ A_i),
 *    partial_i = hidden_i @ B_i, and the result is the sum of the partials over
 *    the ranks.  The default activation there is tanh.
 *  - "大模型推理系统揭秘（07）：Multi-GPU：一张卡不够时如何扩展？", §1.2.2: a
 *    column-parallel linear gives each rank Y_i = X W_i for its column block
 *    W[:, cols_i]; a row-parallel linear gives Z_i = Y_i W_i for its row block,
 *    a partial sum.  §1.2.3 (boxed equations): Z = [Y_0|..|Y_3][W_20;..;W_23]
 *    = sum_i Y_i W_2i.
 *  - same page, §1.4.3: the SwiGLU FFN W_2[SiLU(W_1 x) ⊙ (W_3 x)] (row-vector
 *    form: (SiLU(X W_1) ⊙ (X W_3)) W_2); §1.2.4: gate and up projections are
 *    column-parallel, the activation is rank-local, down is row-parallel.
 *
 * Readings taken where the pages are silent:
 *  - no bias terms (none appear in the code or the equations);
 *  - SiLU(g) = g * sigma(g) = g / (1 + exp(-g)), the textbook definition;
 *  - for SwiGLU the rank's first-projection shard A_i is the column block
 *    [gate_i | up_i] (d_in x 2*f_s), gate_i and up_i covering the same
 *    intermediate features;
 *  - the partials are summed in rank order 0..P-1;
 *  - the output width d_out may differ from d_in (the §1.2.3 example maps
 *    8 -> 8 -> 4).
 *
 * Inputs are fp32 arrays holding exact values (an fp32 or bf16 number is
 * exactly representable in fp32); every product and sum is done in double.
 * Plain loops, row-major arrays, OpenMP over tokens only.  Each entry point
 * returns the number of multiply-adds it executed (counted as the loops run),
 * or -1 on an argument error.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_ACT_TANH = 0, ORACLE_ACT_SWIGLU = 1, ORACLE_ACT_IDENTITY = 2 };

/* SiLU(g) = g * sigma(g), sigma(g) = 1 / (1 + e^{-g}). */
static double silu(double g) { return g / (1.0 + exp(-g)); }

/*
 * One rank's partial (or the whole unsharded MLP when f_s = d_ff):
 *   first projection  u[t][n] = sum_j x[t][j] * a_g[j][n]       (column block)
 *                     v[t][n] = sum_j x[t][j] * a_u[j][n]       (SwiGLU only)
 *   activation        h[t][n] = tanh(u) | SiLU(u) * v | u
 *   second projection z[t][c] = sum_n h[t][n] * b[n][c]          (row block)
 * a_g / a_u point at the first column of the gate (or only) and up blocks;
 * lda is the row stride of the first-projection matrix, in elements.
 */
static long long mlp_block(const float *x, int T, int d_in, int f_s, int d_out,
                           int act, const float *a_g, const float *a_u,
                           long lda, const float *b, double *z)
{
    long long macs = 0;
#pragma omp parallel for schedule(static) reduction(+ : macs)
    for (int t = 0; t < T; ++t) {
        double *u = (double *)calloc((size_t)f_s, sizeof(double));
        double *v = (double *)calloc((size_t)f_s, sizeof(double));
        const float *xt = x + (size_t)t * d_in;
        for (int j = 0; j < d_in; ++j) {
            const double xj = (double)xt[j];
            const float *rg = a_g + (size_t)j * lda;
            for (int n = 0; n < f_s; ++n) u[n] += xj * (double)rg[n];
            macs += f_s;
            if (act == ORACLE_ACT_SWIGLU) {
                const float *ru = a_u + (size_t)j * lda;
                for (int n = 0; n < f_s; ++n) v[n] += xj * (double)ru[n];
                macs += f_s;
            }
        }
        for (int n = 0; n < f_s; ++n) {
            if (act == ORACLE_ACT_TANH) u[n] = tanh(u[n]);
            else if (act == ORACLE_ACT_SWIGLU) u[n] = silu(u[n]) * v[n];
            /* identity: h = u */
        }
        double *zt = z + (size_t)t * d_out;
        for (int c = 0; c < d_out; ++c) zt[c] = 0.0;
        for (int n = 0; n < f_s; ++n) {
            const double hn = u[n];
            const float *rb = b + (size_t)n * d_out;
            for (int c = 0; c < d_out; ++c) zt[c] += hn * (double)rb[c];
            macs += d_out;
        }
        free(u);
        free(v);
    }
    return macs;
}

static int args_ok(int T, int d_in, int d_ff, int d_out, int act)
{
    if (T < 0 || d_in < 1 || d_ff < 1 || d_out < 1) return 0;
    if (act != ORACLE_ACT_TANH && act != ORACLE_ACT_SWIGLU &&
        act != ORACLE_ACT_IDENTITY) return 0;
    return 1;
}

/*
 * Sharded form, the pages' tensor_parallel_output: n_a first-projection
 * shards and n_b second-projection shards (they must be equal: P ranks).
 *   tanh / identity: a_shards[i] is d_in x f_s, b_shards[i] is f_s x d_out;
 *   SwiGLU:          a_shards[i] is d_in x 2 f_s laid out [gate_i | up_i].
 * z (T x d_out) receives sum_i Z_i, summed in rank order.  If partials is not
 * NULL it receives every Z_i (P x T x d_out) before the sum.
 */
long long oracle_tp_mlp_sharded(const float *x, int T, int d_in, int d_ff,
                                int d_out, int act, int n_a,
                                const float *const *a_shards, int n_b,
                                const float *const *b_shards, double *z,
                                double *partials)
{
    if (!args_ok(T, d_in, d_ff, d_out, act)) return -1;
    if (n_a != n_b || n_a < 1) return -1;          /* zip(..., strict=True) */
    const int P = n_a;
    if (d_ff % P != 0) return -1;
    const int f_s = d_ff / P;
    const long lda = (act == ORACLE_ACT_SWIGLU) ? 2L * f_s : (long)f_s;
    const size_t zn = (size_t)T * d_out;
    double *zi = (double *)malloc((zn ? zn : 1) * sizeof(double));
    long long macs = 0;
    for (size_t e = 0; e < zn; ++e) z[e] = 0.0;
    for (int i = 0; i < P; ++i) {
        const float *a_i = a_shards[i];
        const float *a_up = (act == ORACLE_ACT_SWIGLU) ? a_i + f_s : NULL;
        macs += mlp_block(x, T, d_in, f_s, d_out, act, a_i, a_up, lda,
                          b_shards[i], zi);
        if (partials) memcpy(partials + (size_t)i * zn, zi, zn * sizeof(double));
        for (size_t e = 0; e < zn; ++e) z[e] += zi[e];   /* the all-reduce */
    }
    free(zi);
    return macs;
}

/*
 * Unsharded MLP on the full matrices: act(X A) B, i.e. the P = 1 case.
 *   tanh / identity: a is d_in x d_ff, a_up must be NULL;
 *   SwiGLU:          a is gate (d_in x d_ff), a_up is up (d_in x d_ff).
 * b is d_ff x d_out.
 */
long long oracle_tp_mlp_unsharded(const float *x, int T, int d_in, int d_ff,
                                  int d_out, int act, const float *a,
                                  const float *a_up, const float *b, double *z)
{
    if (!args_ok(T, d_in, d_ff, d_out, act)) return -1;
    if ((act == ORACLE_ACT_SWIGLU) != (a_up != NULL)) return -1;
    return mlp_block(x, T, d_in, d_ff, d_out, act, a, a_up, (long)d_ff, b, z);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
