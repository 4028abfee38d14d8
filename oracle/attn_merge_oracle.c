/*
 * attn_merge_oracle.c -- the oracle for merging partial attention results of
 * KV shards (decode context parallelism), every arithmetic step in fp64.
 *
 * TEST INFRASTRUCTURE ONLY, like tp_mlp_oracle.c (built into the same library,
 * with the same callers).  The CUDA library shares no code with it.
 *
 * What it computes, and where the pages say so:
 *
 *  - "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 4) 上下文并行（CP）, decode
 *    context parallelism (DCP): the stored KV history is cut by sequence
 *    position; each rank attends over its own part and reports, per query, the
 *    local maximum score, the sum of exponentials taken relative to that
 *    maximum, and the exponential-weighted sum of the values.  The merge takes
 *    the global maximum, rescales every rank's sum and weighted sum by
 *    exp(local max - global max), adds them up, and divides the merged weighted
 *    sum by the merged sum.  The pages state that this reproduces attention over
 *    the unsplit history.
 *
 * Readings taken where the pages are silent:
 *  - scores are q . k times a caller-given scale (the usual 1/sqrt(D));
 *  - a rank with no keys for a row reports maximum -inf, sum 0 and weighted
 *    sum 0, and contributes nothing; a row for which every rank is empty merges
 *    to zeros;
 *  - one query row is one (token, head) pair; ranks are added in rank order.
 *
 * Inputs are fp32 arrays holding exact values; all arithmetic is in double.
 * Each entry point returns 0, or -1 on an argument error.
 */
#include <math.h>
#include <stddef.h>

/*
 * Rank-local step for `rows` query rows against `n_keys` keys:
 *   q: rows x D, k: n_keys x D, v: n_keys x D (one shard of the history).
 * Writes maximum[rows], exp_sum[rows], weighted[rows x D].
 */
int oracle_attention_partial(const float *q, const float *k, const float *v, int rows, int n_keys, int D,
                             double scale, double *maximum, double *exp_sum, double *weighted)
{
    if (rows < 0 || n_keys < 0 || D < 1) return -1;
    for (int r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int j = 0; j < n_keys; ++j) {
            double sc = 0.0;
            for (int e = 0; e < D; ++e) sc += (double)q[(size_t)r * D + e] * (double)k[(size_t)j * D + e];
            sc *= scale;
            if (sc > m) m = sc;
        }
        double s = 0.0;
        double *w = weighted + (size_t)r * D;
        for (int e = 0; e < D; ++e) w[e] = 0.0;
        for (int j = 0; j < n_keys; ++j) {
            double sc = 0.0;
            for (int e = 0; e < D; ++e) sc += (double)q[(size_t)r * D + e] * (double)k[(size_t)j * D + e];
            const double p = exp(sc * scale - m);
            s += p;
            for (int e = 0; e < D; ++e) w[e] += p * (double)v[(size_t)j * D + e];
        }
        maximum[r] = m;
        exp_sum[r] = s;
    }
    return 0;
}

/*
 * The merge, in the pages' order of steps, for P ranks and `rows` rows:
 *   maximum, exp_sum: P x rows; weighted: P x rows x D.  Writes out: rows x D.
 */
int oracle_merge_attention_partials(int P, int rows, int D, const float *maximum, const float *exp_sum,
                                    const float *weighted, double *out)
{
    if (P < 1 || rows < 0 || D < 1) return -1;
    for (int r = 0; r < rows; ++r) {
        double global_max = -INFINITY;
        for (int i = 0; i < P; ++i)
            if ((double)maximum[(size_t)i * rows + r] > global_max) global_max = maximum[(size_t)i * rows + r];
        double *o = out + (size_t)r * D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        if (global_max == -INFINITY) continue;            /* every rank empty */
        double denominator = 0.0;
        for (int i = 0; i < P; ++i) {
            const double m = maximum[(size_t)i * rows + r];
            const double scale = (m == -INFINITY) ? 0.0 : exp(m - global_max);
            denominator += scale * (double)exp_sum[(size_t)i * rows + r];
            for (int e = 0; e < D; ++e)
                o[e] += scale * (double)weighted[((size_t)i * rows + r) * D + e];   /* numerator */
        }
        for (int e = 0; e < D; ++e) o[e] /= denominator;
    }
    return 0;
}

/*
 * The plain definition the merge must reproduce: softmax attention of each
 * query row over all n_keys keys, out[r] = sum_j softmax_j(scale q_r . k_j) v_j
 * (the softmax taken relative to the row's maximum so that exp cannot overflow).
 */
int oracle_attention_full(const float *q, const float *k, const float *v, int rows, int n_keys, int D,
                          double scale, double *out)
{
    if (rows < 0 || n_keys < 1 || D < 1) return -1;
    for (int r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int j = 0; j < n_keys; ++j) {
            double sc = 0.0;
            for (int e = 0; e < D; ++e) sc += (double)q[(size_t)r * D + e] * (double)k[(size_t)j * D + e];
            if (sc * scale > m) m = sc * scale;
        }
        double z = 0.0;
        for (int j = 0; j < n_keys; ++j) {
            double sc = 0.0;
            for (int e = 0; e < D; ++e) sc += (double)q[(size_t)r * D + e] * (double)k[(size_t)j * D + e];
            z += exp(sc * scale - m);
        }
        double *o = out + (size_t)r * D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        for (int j = 0; j < n_keys; ++j) {
            double sc = 0.0;
            for (int e = 0; e < D; ++e) sc += (double)q[(size_t)r * D + e] * (double)k[(size_t)j * D + e];
            const double p = exp(sc * scale - m) / z;
            for (int e = 0; e < D; ++e) o[e] += p * (double)v[(size_t)j * D + e];
        }
    }
    return 0;
}
