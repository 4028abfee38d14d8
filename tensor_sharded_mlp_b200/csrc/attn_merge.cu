// attn_merge.cu -- merging the partial attention results of KV shards (decode
// context parallelism), one kernel.
//
// "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 4) 上下文并行（CP）: the KV
// history is cut by sequence position, each rank attends over its own part and
// reports per query row (one token and head) its maximum score m_i, the sum of
// exponentials relative to it s_i and the exponential-weighted sum of values
// w_i; the merge
//   M = max_i m_i,  c_i = exp(m_i - M),  out = (sum_i c_i w_i) / (sum_i c_i s_i)
// reproduces attention over the whole history.  A rank with no keys for the row
// reports m_i = -inf and contributes nothing; a row with every rank empty is 0.
//
// One warp per row: the lanes read the row's P maxima and sums (the same
// addresses, one transaction), then walk the row in groups of 4 elements with
// all P weighted groups in flight at once (P is a template argument): 16-byte
// loads for fp32, 8-byte loads for bf16.  The data is read once and is
// HBM-bound; there is nothing to reuse.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "vec_io.cuh"

namespace tpmlp {
namespace {

constexpr int kMergeThreads = 256;

template <typename T, int P>
__global__ void __launch_bounds__(kMergeThreads)
    attn_merge_kernel(const float *__restrict__ maximum, const float *__restrict__ exp_sum,
                      const T *__restrict__ weighted, int rows, int D, T *__restrict__ out) {
    pdl_allow_dependents();
    const int lane = threadIdx.x & 31;
    const long long r = ((long long)blockIdx.x * kMergeThreads + threadIdx.x) >> 5;
    pdl_wait_previous();   // the partials may come from the previous kernel
    if (r >= rows) return;
    float m[P];
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        m[i] = __ldg(maximum + (long long)i * rows + r);
        M = fmaxf(M, m[i]);
    }
    float c[P];
    float den = 0.f;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        c[i] = m[i] == -INFINITY ? 0.f : expf(m[i] - M);
        den += c[i] * __ldg(exp_sum + (long long)i * rows + r);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;   // every rank empty: zeros
    const long long rank_stride = (long long)rows * D;
    const T *wr = weighted + r * D;
    T *o = out + r * D;
    for (int g = lane; g < (D >> 2); g += 32) {
        float4 v[P];
#pragma unroll
        for (int i = 0; i < P; ++i) v[i] = load4(wr + i * rank_stride + 4 * g);
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < P; ++i) {
            a.x += c[i] * v[i].x; a.y += c[i] * v[i].y; a.z += c[i] * v[i].z; a.w += c[i] * v[i].w;
        }
        store4(o + 4 * g, make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv));
    }
}

template <typename T>
cudaError_t launch_t(int P, int rows, int D, const float *mx, const float *es, const void *w, void *out,
                     cudaStream_t st) {
    const dim3 grid((unsigned)((rows * 32LL + kMergeThreads - 1) / kMergeThreads));
    const T *wt = static_cast<const T *>(w);
    T *ot = static_cast<T *>(out);
    switch (P) {
        case 1: return launch_pdl(attn_merge_kernel<T, 1>, grid, dim3(kMergeThreads), 0, st, mx, es, wt, rows, D, ot);
        case 2: return launch_pdl(attn_merge_kernel<T, 2>, grid, dim3(kMergeThreads), 0, st, mx, es, wt, rows, D, ot);
        case 3: return launch_pdl(attn_merge_kernel<T, 3>, grid, dim3(kMergeThreads), 0, st, mx, es, wt, rows, D, ot);
        case 4: return launch_pdl(attn_merge_kernel<T, 4>, grid, dim3(kMergeThreads), 0, st, mx, es, wt, rows, D, ot);
        case 5: return launch_pdl(attn_merge_kernel<T, 5>, grid, dim3(kMergeThreads), 0, st, mx, es, wt, rows, D, ot);
        case 6: return launch_pdl(attn_merge_kernel<T, 6>, grid, dim3(kMergeThreads), 0, st, mx, es, wt, rows, D, ot);
        case 7: return launch_pdl(attn_merge_kernel<T, 7>, grid, dim3(kMergeThreads), 0, st, mx, es, wt, rows, D, ot);
        case 8: return launch_pdl(attn_merge_kernel<T, 8>, grid, dim3(kMergeThreads), 0, st, mx, es, wt, rows, D, ot);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attn_merge(int P, int rows, int D, const float *maximum, const float *exp_sum,
                              const void *weighted, int dtype, void *out, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (dtype == TP_MLP_F32) return launch_t<float>(P, rows, D, maximum, exp_sum, weighted, out, st);
    return launch_t<__nv_bfloat16>(P, rows, D, maximum, exp_sum, weighted, out, st);
}

}  // namespace tpmlp
