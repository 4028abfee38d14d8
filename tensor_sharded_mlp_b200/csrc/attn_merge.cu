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
// A row is walked by a group of L lanes (L a power of two up to 32, as many as
// the row has groups of V elements, so short rows share a warp); the lanes of
// a group read the row's P maxima and sums (the same addresses), then walk the
// row V elements at a time with all P weighted groups in flight at once (P is
// a template argument): 16-byte loads (fp32 V = 4, bf16 V = 8 when the row
// allows), else 8-byte bf16 loads (V = 4).  The lane's first groups are
// requested before the maxima come back, so a decode-sized row costs one
// memory round trip.  The data is read once and is HBM-bound; there is
// nothing to reuse.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "vec_io.cuh"

namespace tpmlp {
namespace {

constexpr int kMergeThreads = 256;

// V consecutive elements as loaded (16 bytes of fp32, 16 or 8 of bf16),
// widened to fp32 only where they are used, so the loads in flight hold as
// few registers as the data needs
template <typename T, int V> struct Packed;
template <> struct Packed<float, 4> { using type = float4; };
template <> struct Packed<__nv_bfloat16, 4> { using type = uint2; };
template <> struct Packed<__nv_bfloat16, 8> { using type = uint4; };
template <typename T, int V>
__device__ __forceinline__ typename Packed<T, V>::type load_packed(const T *p) {
    return *reinterpret_cast<const typename Packed<T, V>::type *>(p);
}
__device__ __forceinline__ void widen(float4 v, float *f) { f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w; }
__device__ __forceinline__ void widen(uint2 u, float *f) {
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
}
__device__ __forceinline__ void widen(uint4 u, float *f) {
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
    f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
}
__device__ __forceinline__ void store_v(float *p, const float *a) { store4(p, make_float4(a[0], a[1], a[2], a[3])); }
__device__ __forceinline__ void store_v(__nv_bfloat16 *p, const float *a, int n) {
    if (n == 4) {
        store4(p, make_float4(a[0], a[1], a[2], a[3]));
    } else {
        *reinterpret_cast<uint4 *>(p) = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                                   pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
    }
}
__device__ __forceinline__ void store_v(float *p, const float *a, int) { store_v(p, a); }

// lanes_log2 = log2(L); a warp covers 32 / L rows
template <typename T, int P, int V>
__global__ void __launch_bounds__(kMergeThreads)
    attn_merge_kernel(const float *__restrict__ maximum, const float *__restrict__ exp_sum,
                      const T *__restrict__ weighted, int rows, int D, int lanes_log2, T *__restrict__ out) {
    pdl_allow_dependents();
    const int lane = threadIdx.x & 31;
    const int L = 1 << lanes_log2;
    const int li = lane & (L - 1);
    const long long warp = ((long long)blockIdx.x * kMergeThreads + threadIdx.x) >> 5;
    const long long r = (warp << (5 - lanes_log2)) + (lane >> lanes_log2);
    pdl_wait_previous();   // the partials may come from the previous kernel
    if (r >= rows) return;
    const long long rank_stride = (long long)rows * D;
    const T *wr = weighted + r * D;
    T *o = out + r * D;
    const int G = D / V;
    typename Packed<T, V>::type v[P];
    if (li < G) {
#pragma unroll
        for (int i = 0; i < P; ++i) v[i] = load_packed<T, V>(wr + i * rank_stride + V * li);
    }
    float c[P], s[P];
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        c[i] = __ldg(maximum + (long long)i * rows + r);
        s[i] = __ldg(exp_sum + (long long)i * rows + r);
        M = fmaxf(M, c[i]);
    }
    float den = 0.f;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        c[i] = c[i] == -INFINITY ? 0.f : expf(c[i] - M);   // the rank's scale
        den += c[i] * s[i];
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;   // every rank empty: zeros
    for (int g = li; g < G; g += L) {
        if (g != li) {
#pragma unroll
            for (int i = 0; i < P; ++i) v[i] = load_packed<T, V>(wr + i * rank_stride + V * g);
        }
        float a[V];
#pragma unroll
        for (int k = 0; k < V; ++k) a[k] = 0.f;
#pragma unroll
        for (int i = 0; i < P; ++i) {
            float w[V];
            widen(v[i], w);
#pragma unroll
            for (int k = 0; k < V; ++k) a[k] += c[i] * w[k];
        }
#pragma unroll
        for (int k = 0; k < V; ++k) a[k] *= inv;
        store_v(o + V * g, a, V);
    }
}

template <typename T, int V>
cudaError_t launch_tv(int P, int rows, int D, const float *mx, const float *es, const T *w, T *out,
                      cudaStream_t st) {
    // lanes per row: the largest power of two up to 32 that the row's groups fill
    const int G = D / V;
    int lg = 0;
    while (lg < 5 && (2 << lg) <= G) ++lg;
    const long long warps = ((long long)rows + (32 >> lg) - 1) >> (5 - lg);
    const dim3 grid((unsigned)((warps * 32 + kMergeThreads - 1) / kMergeThreads));
    const dim3 block(kMergeThreads);
    switch (P) {
        case 1: return launch_pdl(attn_merge_kernel<T, 1, V>, grid, block, 0, st, mx, es, w, rows, D, lg, out);
        case 2: return launch_pdl(attn_merge_kernel<T, 2, V>, grid, block, 0, st, mx, es, w, rows, D, lg, out);
        case 3: return launch_pdl(attn_merge_kernel<T, 3, V>, grid, block, 0, st, mx, es, w, rows, D, lg, out);
        case 4: return launch_pdl(attn_merge_kernel<T, 4, V>, grid, block, 0, st, mx, es, w, rows, D, lg, out);
        case 5: return launch_pdl(attn_merge_kernel<T, 5, V>, grid, block, 0, st, mx, es, w, rows, D, lg, out);
        case 6: return launch_pdl(attn_merge_kernel<T, 6, V>, grid, block, 0, st, mx, es, w, rows, D, lg, out);
        case 7: return launch_pdl(attn_merge_kernel<T, 7, V>, grid, block, 0, st, mx, es, w, rows, D, lg, out);
        case 8: return launch_pdl(attn_merge_kernel<T, 8, V>, grid, block, 0, st, mx, es, w, rows, D, lg, out);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attn_merge(int P, int rows, int D, const float *maximum, const float *exp_sum,
                              const void *weighted, int dtype, void *out, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (dtype == TP_MLP_F32)
        return launch_tv<float, 4>(P, rows, D, maximum, exp_sum, static_cast<const float *>(weighted),
                                   static_cast<float *>(out), st);
    // 16-byte loads when every row starts on a 16-byte boundary (D % 8 == 0)
    const auto *wb = static_cast<const __nv_bfloat16 *>(weighted);
    auto *ob = static_cast<__nv_bfloat16 *>(out);
    if (D % 8 == 0) return launch_tv<__nv_bfloat16, 8>(P, rows, D, maximum, exp_sum, wb, ob, st);
    return launch_tv<__nv_bfloat16, 4>(P, rows, D, maximum, exp_sum, wb, ob, st);
}

}  // namespace tpmlp
