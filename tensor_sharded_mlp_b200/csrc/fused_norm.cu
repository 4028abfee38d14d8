// fused_norm.cu -- the tensor-parallel all-reduce followed by the residual add
// and RMSNorm, as one kernel.
//
// "7.4 推理侧并行", §7.4.2, optimisation 2 (custom all-reduce): the residual add
// and RMSNorm that follow the all-reduce are fused into it, so the summed
// activations are not written out and read back in between.  With every rank
// on one GPU the all-reduce is the sum of the ranks' fp32 partial outputs Z_i
// (tp_mlp_partials, "大模型推理系统揭秘（07）" §1.2.3).  Per token row t:
//   h            = residual[t] + sum_i Z_i[t]       (ranks in order, fp32)
//   residual_out = h
//   y            = h / sqrt(mean_j h_j^2 + eps) * gamma
//
// A row is cut into C contiguous chunks, one CTA each, and the C CTAs of a row
// form one thread-block cluster: each keeps its chunk of h in shared memory,
// adds up its part of sum(h^2), and reads the other CTAs' parts through
// distributed shared memory after a cluster barrier (a hardware barrier: no
// CTA spins on another).  C grows when there are few rows (decode), so that
// the grid still covers the SMs; with many rows C = 1.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"
#include "vec_io.cuh"

namespace tpmlp {
namespace {

using tc::smem_u32;

constexpr int kNormThreads = 256;

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a cluster barrier that publishes nothing: the arrive does not wait for this
// thread's earlier stores to complete (its earlier loads have completed, since
// their values were used before it)
__device__ __forceinline__ void cluster_sync_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
// float at the same shared-memory address in CTA `rank` of this cluster
__device__ __forceinline__ float ld_dsmem(const float *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// grid = rows * C CTAs, clusters of C; CTA (row, c) covers float4 groups
// [c * chunk4, min(d / 4, (c + 1) * chunk4)) of its row.
// P (ranks) is a template argument so that the P partial loads of a float4
// group are all in flight at once.
template <typename T, int P>
__global__ void __launch_bounds__(kNormThreads)
    allreduce_norm_kernel(const float *__restrict__ part, int rows, int d, int chunk4, const T *res,
                          const T *__restrict__ gamma, float eps, T *y, T *res_out) {
    extern __shared__ float4 hs[];   // this CTA's chunk of h
    __shared__ float warp_sq[kNormThreads / 32];
    __shared__ float cta_sq;         // read by the other CTAs of the cluster
    pdl_allow_dependents();
    const int C = (int)(gridDim.x / rows);
    const uint32_t c = cluster_ctarank();
    const int t = blockIdx.x / C;
    const int q0 = (int)c * chunk4, q1 = min(d >> 2, q0 + chunk4);
    const long long row = (long long)t * d;
    const long long rank_stride = (long long)rows * d;
    pdl_wait_previous();   // the partials may come from the previous kernel

    float sq = 0.f;
#pragma unroll 2
    for (int q = q0 + (int)threadIdx.x; q < q1; q += kNormThreads) {
        const float *pz = part + row + 4LL * q;
        float4 w[P];
#pragma unroll
        for (int i = 0; i < P; ++i) w[i] = load4_stream(pz + i * rank_stride);
        const float4 r = load4(res + row + 4LL * q);
        float4 z = w[0];
#pragma unroll
        for (int i = 1; i < P; ++i) {   // the all-reduce, ranks in order
            z.x += w[i].x; z.y += w[i].y; z.z += w[i].z; z.w += w[i].w;
        }
        const float4 h = make_float4(r.x + z.x, r.y + z.y, r.z + z.z, r.w + z.w);
        hs[q - q0] = h;
        sq += h.x * h.x + h.y * h.y + h.z * h.z + h.w * h.w;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) warp_sq[warp] = sq;
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kNormThreads / 32; ++w) s += warp_sq[w];
        cta_sq = s;
    }
    cluster_sync();   // every CTA's cta_sq is written (and hs is complete)
    float total = 0.f;
    for (int k = 0; k < C; ++k) total += ld_dsmem(&cta_sq, (uint32_t)k);   // same order in every CTA
    const float scale = rsqrtf(total / (float)d + eps);
    for (int q = q0 + (int)threadIdx.x; q < q1; q += kNormThreads) {
        const float4 h = hs[q - q0];
        const float4 g = load4(gamma + 4LL * q);
        store4(y + row + 4LL * q, make_float4(h.x * scale * g.x, h.y * scale * g.y, h.z * scale * g.z,
                                              h.w * scale * g.w));
        store4(res_out + row + 4LL * q, h);
    }
    cluster_sync_relaxed();   // no CTA leaves while another may still read its cta_sq
}

template <typename T, int P>
cudaError_t launch_typed(const float *part, int rows, int d, const void *res, const void *gamma, float eps,
                         void *y, void *res_out, int num_sms, cudaStream_t st) {
    const int d4 = d / 4;
    // CTAs per row: enough for about two CTAs per SM, at most 8 (a portable
    // cluster) and never more than the row has float4 groups per thread block
    int C = 1;
    while (C < kNormClusterMax && (long long)rows * C < 2LL * num_sms && d4 >= 2 * C * 32) C *= 2;
    const int chunk4 = (d4 + C - 1) / C;
    const size_t smem = (size_t)chunk4 * 16;
    auto kern = allreduce_norm_kernel<T, P>;
    // the attribute is set once per device, so to the largest chunk any call uses
    cudaError_t e = ensure_smem_attr(kern, (size_t)kNormMaxWidth * 4);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * C));
    cfg.blockDim = dim3(kNormThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, part, rows, d, chunk4, static_cast<const T *>(res),
                              static_cast<const T *>(gamma), eps, static_cast<T *>(y), static_cast<T *>(res_out));
}

template <typename T>
cudaError_t launch_p(const float *part, int P, int rows, int d, const void *res, const void *gamma, float eps,
                     void *y, void *res_out, int num_sms, cudaStream_t st) {
    switch (P) {
        case 1: return launch_typed<T, 1>(part, rows, d, res, gamma, eps, y, res_out, num_sms, st);
        case 2: return launch_typed<T, 2>(part, rows, d, res, gamma, eps, y, res_out, num_sms, st);
        case 3: return launch_typed<T, 3>(part, rows, d, res, gamma, eps, y, res_out, num_sms, st);
        case 4: return launch_typed<T, 4>(part, rows, d, res, gamma, eps, y, res_out, num_sms, st);
        case 5: return launch_typed<T, 5>(part, rows, d, res, gamma, eps, y, res_out, num_sms, st);
        case 6: return launch_typed<T, 6>(part, rows, d, res, gamma, eps, y, res_out, num_sms, st);
        case 7: return launch_typed<T, 7>(part, rows, d, res, gamma, eps, y, res_out, num_sms, st);
        case 8: return launch_typed<T, 8>(part, rows, d, res, gamma, eps, y, res_out, num_sms, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_allreduce_norm(const float *partials, int P, int rows, int d, const void *residual,
                                  const void *gamma, float eps, int dtype, void *y, void *residual_out,
                                  int num_sms, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (dtype == TP_MLP_F32) return launch_p<float>(partials, P, rows, d, residual, gamma, eps, y, residual_out,
                                                    num_sms, st);
    return launch_p<__nv_bfloat16>(partials, P, rows, d, residual, gamma, eps, y, residual_out, num_sms, st);
}

}  // namespace tpmlp
