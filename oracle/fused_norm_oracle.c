/*
 * fused_norm_oracle.c -- the oracle for the tensor-parallel all-reduce followed
 * by the residual add and RMSNorm, every arithmetic step in fp64.
 *
 * TEST INFRASTRUCTURE ONLY, like tp_mlp_oracle.c (built into the same library,
 * with the same callers).  The CUDA library shares no code with it.
 *
 * What it computes, and where the pages say so:
 *
 *  - "7.4 推理侧并行", §7.4.2, optimisation 2 (custom all-reduce), its last
 *    point: the kernel that sums the ranks' outputs also does the residual
 *    add and the RMSNorm that come next, so the summed activations are not
 *    written to device memory and read back by a separate kernel.
 *  - The all-reduce sums the ranks' partial outputs Z_i of the row-parallel
 *    second projection ("大模型推理系统揭秘（07）", §1.2.3: Z = sum_i Y_i W_2i),
 *    in rank order as in tp_mlp_oracle.c.
 *
 * Readings taken where the pages are silent:
 *  - RMSNorm is the textbook one: RMSNorm(h)_j = h_j / sqrt(mean_k h_k^2 + eps)
 *    * gamma_j over the whole model width of a token row (no mean subtraction,
 *    no bias); eps is the caller's;
 *  - the residual add comes first: h = residual + sum_i Z_i is both the norm's
 *    input and the updated residual stream handed back to the caller.
 *
 * Inputs are fp32 arrays holding exact values; all sums and products are in
 * double.  Returns 0, or -1 on an argument error.
 */
#include <math.h>
#include <stddef.h>

/*
 * partials: P x T x d (rank-major, as tp_mlp_partials lays them out);
 * residual: T x d; gamma: d.  Writes y (T x d) and h (T x d).
 */
int oracle_allreduce_residual_rmsnorm(const float *partials, int P, int T, int d,
                                      const float *residual, const float *gamma,
                                      double eps, double *y, double *h)
{
    if (P < 1 || T < 0 || d < 1 || !(eps >= 0.0)) return -1;
    for (int t = 0; t < T; ++t) {
        double *ht = h + (size_t)t * d;
        /* the all-reduce (ranks in order), then the residual add */
        for (int j = 0; j < d; ++j) {
            double z = 0.0;
            for (int i = 0; i < P; ++i)
                z += (double)partials[((size_t)i * T + t) * d + j];
            ht[j] = (double)residual[(size_t)t * d + j] + z;
        }
        /* RMSNorm of the row */
        double sum_sq = 0.0;
        for (int j = 0; j < d; ++j) sum_sq += ht[j] * ht[j];
        const double rms = sqrt(sum_sq / (double)d + eps);
        for (int j = 0; j < d; ++j)
            y[(size_t)t * d + j] = ht[j] / rms * (double)gamma[j];
    }
    return 0;
}
