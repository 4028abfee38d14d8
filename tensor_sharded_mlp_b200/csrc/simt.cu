// simt.cu -- tiled CUDA-core kernels for the tensor-parallel MLP.
//
// These serve every shape, both dtypes (fp32 for exact-fp32 work, which the
// tensor cores cannot do -- tcgen05 has no full-fp32 kind), and both weight
// layouts: the per-rank shards as the pages pass them, and the packed K-major
// layout.  They are the general path; the GEMV and tcgen05 kernels are the
// fast paths for bf16.
//
// First projection, column-parallel ("大模型推理系统揭秘（07）", §1.2.2):
//   H[t][n] = act( sum_j X[t][j] * A_{n / f_s}[j][n % f_s] )           (+ up for SwiGLU)
// Second projection, row-parallel, with the ranks' partial sums fused into
// one accumulator (§1.2.3: Z = sum_i Y_i W_2i):
//   Z[t][c] = sum_i sum_{k < f_s} H[t][i f_s + k] * B_i[k][c]
// or, for the partials entry point, one rank's K range per grid z-slice.
#include "common.cuh"
#include "internal.h"

namespace tpmlp {
namespace {

constexpr int BT = 16;   // tokens per block tile
constexpr int BN = 64;   // output columns per block tile
constexpr int BK = 32;   // K per smem stage
constexpr int NTHR = 256;

// Load one element of the first-projection weight W(k, n) (n = global feature).
template <typename E, bool PACKED>
__device__ __forceinline__ float w1_at(const ShardPtrs &w, const Problem &p, int k, int n, bool up) {
    if (PACKED) {
        const E *base = static_cast<const E *>(w.p[0]);
        return to_f32(base[blk_offset(w1p_row(n, up, p.act), k, blk_kblocks(p.d_in))]);
    }
    const int shard = n / p.fs;
    const int j = n - shard * p.fs;
    const long lda = (p.act == TP_MLP_ACT_SWIGLU) ? 2L * p.fs : (long)p.fs;
    const E *a = static_cast<const E *>(w.p[shard]);
    return to_f32(a[(long)k * lda + j + (up ? p.fs : 0)]);
}

// Load one element of the second-projection weight W(k, c) (k = global feature).
template <typename E, bool PACKED>
__device__ __forceinline__ float w2_at(const ShardPtrs &w, const Problem &p, int k, int c) {
    if (PACKED) {
        const E *base = static_cast<const E *>(w.p[0]);
        return to_f32(base[blk_offset(c, k, blk_kblocks(p.d_ff))]);
    }
    const int shard = k / p.fs;
    const E *b = static_cast<const E *>(w.p[shard]);
    return to_f32(b[(long)(k - shard * p.fs) * p.d_out + c]);
}

template <typename E, bool PACKED>
__global__ void __launch_bounds__(NTHR) simt_first_proj(const E *__restrict__ x, ShardPtrs w,
                                                        Problem p, E *__restrict__ h) {
    __shared__ float xs[BK][BT + 1];
    __shared__ float wg[BK][BN + 1];
    __shared__ float wu[BK][BN + 1];
    const bool swiglu = p.act == TP_MLP_ACT_SWIGLU;
    const int tid = threadIdx.x;
    const int t0 = blockIdx.y * BT;
    const int n0 = blockIdx.x * BN;
    const int tt = tid / 16, tn = tid % 16;
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};

    for (int k0 = 0; k0 < p.d_in; k0 += BK) {
        for (int e = tid; e < BT * BK; e += NTHR) {
            const int t = e / BK, k = e % BK;
            const bool ok = (t0 + t < p.T) && (k0 + k < p.d_in);
            xs[k][t] = ok ? to_f32(x[(long)(t0 + t) * p.d_in + k0 + k]) : 0.f;
        }
        for (int e = tid; e < BK * BN; e += NTHR) {
            int k, n;
            if (PACKED) { n = e / BK; k = e % BK; } else { k = e / BN; n = e % BN; }
            const bool ok = (n0 + n < p.d_ff) && (k0 + k < p.d_in);
            wg[k][n] = ok ? w1_at<E, PACKED>(w, p, k0 + k, n0 + n, false) : 0.f;
            if (swiglu) wu[k][n] = ok ? w1_at<E, PACKED>(w, p, k0 + k, n0 + n, true) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < BK; ++k) {
            const float xv = xs[k][tt];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = fmaf(xv, wg[k][tn + 16 * j], acc[j]);
            if (swiglu) {
#pragma unroll
                for (int j = 0; j < 4; ++j) accu[j] = fmaf(xv, wu[k][tn + 16 * j], accu[j]);
            }
        }
        __syncthreads();
    }
    const int t = t0 + tt;
    if (t >= p.T) return;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int n = n0 + tn + 16 * j;
        if (n < p.d_ff) h[(long)t * p.d_ff + n] = from_f32<E>(activate<false>(p.act, acc[j], accu[j]));
    }
}

// out (E) when partials == nullptr; otherwise fp32 partials of rank blockIdx.z.
template <typename E, bool PACKED>
__global__ void __launch_bounds__(NTHR) simt_second_proj(const E *__restrict__ h, ShardPtrs w,
                                                         Problem p, E *__restrict__ out,
                                                         float *__restrict__ partials) {
    __shared__ float hs[BK][BT + 1];
    __shared__ float ws[BK][BN + 1];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.y * BT;
    const int c0 = blockIdx.x * BN;
    const int tt = tid / 16, tc = tid % 16;
    const int kb = partials ? blockIdx.z * p.fs : 0;
    const int ke = partials ? kb + p.fs : p.d_ff;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};

    for (int k0 = kb; k0 < ke; k0 += BK) {
        for (int e = tid; e < BT * BK; e += NTHR) {
            const int t = e / BK, k = e % BK;
            const bool ok = (t0 + t < p.T) && (k0 + k < ke);
            hs[k][t] = ok ? to_f32(h[(long)(t0 + t) * p.d_ff + k0 + k]) : 0.f;
        }
        for (int e = tid; e < BK * BN; e += NTHR) {
            int k, c;
            if (PACKED) { c = e / BK; k = e % BK; } else { k = e / BN; c = e % BN; }
            const bool ok = (c0 + c < p.d_out) && (k0 + k < ke);
            ws[k][c] = ok ? w2_at<E, PACKED>(w, p, k0 + k, c0 + c) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < BK; ++k) {
            const float hv = hs[k][tt];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = fmaf(hv, ws[k][tc + 16 * j], acc[j]);
        }
        __syncthreads();
    }
    const int t = t0 + tt;
    if (t >= p.T) return;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int c = c0 + tc + 16 * j;
        if (c >= p.d_out) continue;
        if (partials)
            partials[((long)blockIdx.z * p.T + t) * p.d_out + c] = acc[j];
        else
            out[(long)t * p.d_out + c] = from_f32<E>(acc[j]);
    }
}

template <typename E, bool PACKED>
cudaError_t launch_simt_typed(const Problem &p, const void *x, const ShardPtrs &w1,
                              const ShardPtrs &w2, void *h, void *out, float *partials,
                              cudaStream_t s, const Marks &marks) {
    const dim3 blk(NTHR);
    marks.mark(0, s);
    const dim3 g1((p.d_ff + BN - 1) / BN, (p.T + BT - 1) / BT);
    simt_first_proj<E, PACKED><<<g1, blk, 0, s>>>(static_cast<const E *>(x), w1, p,
                                                  static_cast<E *>(h));
    marks.mark(1, s);
    const dim3 g2((p.d_out + BN - 1) / BN, (p.T + BT - 1) / BT, partials ? p.tp : 1);
    simt_second_proj<E, PACKED><<<g2, blk, 0, s>>>(static_cast<const E *>(h), w2, p,
                                                   static_cast<E *>(out), partials);
    marks.mark(2, s);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt(const Problem &p, bool packed, const void *x, const ShardPtrs &w1,
                        const ShardPtrs &w2, void *h, void *out, float *partials,
                        cudaStream_t s, const Marks &m) {
    if (p.dtype == TP_MLP_F32)
        return packed ? launch_simt_typed<float, true>(p, x, w1, w2, h, out, partials, s, m)
                      : launch_simt_typed<float, false>(p, x, w1, w2, h, out, partials, s, m);
    return packed ? launch_simt_typed<__nv_bfloat16, true>(p, x, w1, w2, h, out, partials, s, m)
                  : launch_simt_typed<__nv_bfloat16, false>(p, x, w1, w2, h, out, partials, s, m);
}

}  // namespace tpmlp
