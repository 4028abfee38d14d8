// gemv.cu -- decode path: the MLP for 1..4 tokens on packed bf16 weights.
//
// Decode is memory-bound: every weight is read once per step and each weight
// feeds only T multiply-adds ("7.4 推理侧并行", §7.4.1: at batch 1 the GEMM
// degenerates to a GEMV whose time is the weight read).  So these kernels are
// built to stream the K-major packed weights at HBM speed:
//   * one warp per output feature ("group"); each lane loads 16 bytes
//     (8 bf16) of every weight row per step with a non-allocating L1 load,
//     several steps in flight;
//   * X (or H) for the block's K chunk is staged once in shared memory as
//     fp32, permuted so that every lane's 2x16-byte read is conflict-free;
//   * warp-shuffle reduction of the per-lane sums;
//   * split-K over blockIdx.y when K is long: each split writes fp32 partial
//     sums to the workspace and the LAST block to finish a row range (found
//     with one atomic counter; nothing ever waits) adds the splits in a fixed
//     order, applies the epilogue and resets the counter.
// First projection (MODE 0): group n = feature n; rows w1p_row(n) (+ its up
// row for SwiGLU); H[t][n] = act(.).  Second projection (MODE 1): group c =
// output column c; one row of d_ff elements whose K loop runs over every
// rank's rows, so the rank sum happens in the accumulator; out[t][c].
#include "common.cuh"
#include "internal.h"

namespace tpmlp {
namespace {

constexpr int WARPS = 8;
constexpr int NTHR = WARPS * 32;
constexpr int KSTEP = 256;   // elements one warp covers per load step (32 lanes x 8)

struct GemvArgs {
    const __nv_bfloat16 *w;   // packed rows
    long ldw;                 // row length (elements) = K
    const __nv_bfloat16 *x;   // T x K activations (row-major, row stride K)
    int K;
    int Kc;                   // K chunk per split, a multiple of KSTEP
    int S;                    // splits
    int groups;               // output features
    int gpb;                  // groups per block
    int act, d_ff;            // for the first projection's row map / epilogue
    __nv_bfloat16 *out;       // T x groups
    float *part;              // S x groups x R x T partial sums (S > 1)
    unsigned *counters;       // one per blockIdx.x, zero between launches
};

// Position of element k (0 <= k < Kc) of the staged chunk: within each 256-wide
// step, lane l owns k = 8l..8l+7; its first four go to [l*4], its last four to
// [128 + l*4], so a warp's float4 reads are contiguous.
__device__ __forceinline__ int xs_pos(int k) {
    const int step = k / KSTEP, w = k % KSTEP;
    const int lane = w >> 3, half = (w >> 2) & 1, e = w & 3;
    return step * KSTEP + half * 128 + lane * 4 + e;
}

template <int T, int R>
__device__ __forceinline__ void fma8(float (&acc)[R][T], const uint4 (&wv)[R], const float4 (&xa)[T],
                                     const float4 (&xb)[T]) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float w0 = bf16lo(wv[r].x), w1 = bf16hi(wv[r].x), w2 = bf16lo(wv[r].y), w3 = bf16hi(wv[r].y);
        const float w4 = bf16lo(wv[r].z), w5 = bf16hi(wv[r].z), w6 = bf16lo(wv[r].w), w7 = bf16hi(wv[r].w);
#pragma unroll
        for (int t = 0; t < T; ++t) {
            float a = acc[r][t];
            a = fmaf(w0, xa[t].x, a); a = fmaf(w1, xa[t].y, a);
            a = fmaf(w2, xa[t].z, a); a = fmaf(w3, xa[t].w, a);
            a = fmaf(w4, xb[t].x, a); a = fmaf(w5, xb[t].y, a);
            a = fmaf(w6, xb[t].z, a); a = fmaf(w7, xb[t].w, a);
            acc[r][t] = a;
        }
    }
}

template <int T, int R, int MODE>
__device__ __forceinline__ void finish(const GemvArgs &a, int g, const float (&v)[R][T]) {
#pragma unroll
    for (int t = 0; t < T; ++t) {
        float y;
        if (MODE == 0) y = activate<true>(a.act, v[0][t], R > 1 ? v[R - 1][t] : 0.f);
        else y = v[0][t];
        a.out[(long)t * a.groups + g] = __float2bfloat16_rn(y);
    }
}

template <int T, int R, int MODE>
__global__ void __launch_bounds__(NTHR) gemv_kernel(GemvArgs a) {
    extern __shared__ float4 smem4[];
    float *xs = reinterpret_cast<float *>(smem4);
    __shared__ bool s_last;
    constexpr int U = (R == 1) ? 8 : 4;   // load steps in flight per row
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int s = blockIdx.y;
    const long kbase = (long)s * a.Kc;
    const int klen = (int)min((long)a.Kc, (long)a.K - kbase);
    const int kpad = (klen + KSTEP - 1) / KSTEP * KSTEP;

    const int g0 = blockIdx.x * a.gpb;
    const int g1 = min(a.groups, g0 + a.gpb);
    auto rows_of = [&](int g, const __nv_bfloat16 *(&row)[R]) {
        if (MODE == 0) {
            row[0] = a.w + w1p_row(g, false, a.d_ff, a.act) * a.ldw + kbase;
            if (R > 1) row[R - 1] = a.w + w1p_row(g, true, a.d_ff, a.act) * a.ldw + kbase;
        } else {
            row[0] = a.w + (long)g * a.ldw + kbase;
        }
    };
    auto load_bundle = [&](const __nv_bfloat16 *const (&row)[R], int k0, uint4 (&wv)[U][R]) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = k0 + u * KSTEP + lane * 8;
#pragma unroll
            for (int r = 0; r < R; ++r)
                wv[u][r] = (k < klen) ? ld_stream_v4(row[r] + k) : make_uint4(0, 0, 0, 0);
        }
    };

    // Prologue, independent of the previous kernel: let the next kernel launch,
    // pull this warp's first rows towards L2 and issue its first weight loads.
    pdl_allow_dependents();
    uint4 wv[U][R];
    {
        const int g = g0 + warp;
        if (g < g1) {
            const __nv_bfloat16 *row[R];
            rows_of(g, row);
            if (lane < R) prefetch_l2(row[lane], (uint32_t)klen * 2u);
            load_bundle(row, 0, wv);
        }
    }
    // X (or H) is produced by the previous kernel: wait for it, then stage
    // X[:, kbase : kbase + klen] (zero-padded to a whole step) as fp32.
    pdl_wait_previous();
    for (int t = 0; t < T; ++t) {
        const __nv_bfloat16 *xr = a.x + (long)t * a.K + kbase;
        for (int k = threadIdx.x; k < kpad; k += NTHR)
            xs[t * kpad + xs_pos(k)] = (k < klen) ? __bfloat162float(xr[k]) : 0.f;
    }
    __syncthreads();

    bool first = true;
    for (int g = g0 + warp; g < g1; g += WARPS) {
        const __nv_bfloat16 *row[R];
        rows_of(g, row);
        float acc[R][T];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < T; ++t) acc[r][t] = 0.f;

        for (int k0 = 0; k0 < klen; k0 += KSTEP * U) {
            if (!first) load_bundle(row, k0, wv);
            first = false;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int kk = k0 + u * KSTEP;
                if (kk >= kpad) break;
                float4 xa[T], xb[T];
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const float4 *xp = reinterpret_cast<const float4 *>(xs + t * kpad + kk);
                    xa[t] = xp[lane];
                    xb[t] = xp[32 + lane];
                }
                fma8<T, R>(acc, wv[u], xa, xb);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < T; ++t) {
                float v = acc[r][t];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                acc[r][t] = v;
            }
        if (lane == 0) {
            if (a.S == 1) {
                finish<T, R, MODE>(a, g, acc);
            } else {
                float *dst = a.part + (((long)s * a.groups + g) * R) * T;
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int t = 0; t < T; ++t) dst[r * T + t] = acc[r][t];
            }
        }
    }
    if (a.S == 1) return;

    // split-K: the last block of this row range to arrive reduces all splits
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(&a.counters[blockIdx.x], 1u);
        s_last = (prev == (unsigned)(a.S - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int g = g0 + threadIdx.x; g < g1; g += NTHR) {
        float v[R][T];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < T; ++t) v[r][t] = 0.f;
        for (int sp = 0; sp < a.S; ++sp) {
            const float *src = a.part + (((long)sp * a.groups + g) * R) * T;
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int t = 0; t < T; ++t) v[r][t] += __ldcg(src + r * T + t);
        }
        finish<T, R, MODE>(a, g, v);
    }
    if (threadIdx.x == 0) a.counters[blockIdx.x] = 0u;
}

template <int T, int R, int MODE>
cudaError_t launch_one(const GemvArgs &a, cudaStream_t st) {
    const size_t smem = (size_t)T * a.Kc * sizeof(float);
    auto kern = gemv_kernel<T, R, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((a.groups + a.gpb - 1) / a.gpb, a.S);
    return launch_pdl(kern, grid, dim3(NTHR), smem, st, a);
}

template <int R, int MODE>
cudaError_t launch_T(int T, const GemvArgs &a, cudaStream_t st) {
    switch (T) {
        case 1: return launch_one<1, R, MODE>(a, st);
        case 2: return launch_one<2, R, MODE>(a, st);
        case 3: return launch_one<3, R, MODE>(a, st);
        case 4: return launch_one<4, R, MODE>(a, st);
    }
    return cudaErrorInvalidValue;
}

// Split count: keep the staged chunk <= kSmemBudget and give the grid enough blocks.
constexpr size_t kSmemBudget = 48 * 1024;
constexpr int kGpb = 16;

void plan_split(int T, int K, int groups, int num_sms, int &S, int &Kc) {
    const long steps = (K + KSTEP - 1) / KSTEP;
    int s_smem = (int)(((size_t)T * steps * KSTEP * sizeof(float) + kSmemBudget - 1) / kSmemBudget);
    const int blocks = (groups + kGpb - 1) / kGpb;
    int s_occ = (int)((4L * num_sms + blocks - 1) / blocks);   // >= ~4 blocks per SM
    S = max(1, max(s_smem, s_occ));
    S = (int)min((long)S, steps);
    Kc = (int)(((steps + S - 1) / S) * KSTEP);
    S = (int)((K + Kc - 1) / Kc);
}

}  // namespace

bool gemv_supported(const Problem &p) {
    return p.dtype == TP_MLP_BF16 && p.T >= 1 && p.T <= kGemvMaxTokens && p.d_in % 8 == 0 &&
           p.d_ff % 8 == 0;
}

size_t gemv_workspace_bytes(const Problem &p, int num_sms) {
    if (!gemv_supported(p)) return 0;
    int S1, K1, S2, K2;
    plan_split(p.T, p.d_in, p.d_ff, num_sms, S1, K1);
    plan_split(p.T, p.d_ff, p.d_out, num_sms, S2, K2);
    const int R1 = p.act == TP_MLP_ACT_SWIGLU ? 2 : 1;
    const size_t a = S1 > 1 ? (size_t)S1 * p.d_ff * R1 * p.T * 4 : 0;
    const size_t b = S2 > 1 ? (size_t)S2 * p.d_out * p.T * 4 : 0;
    return align256(a > b ? a : b);
}

size_t gemv_counter_slots(const Problem &p) {
    const int m = p.d_ff > p.d_out ? p.d_ff : p.d_out;
    return (size_t)(m + kGpb - 1) / kGpb;
}

cudaError_t launch_gemv(const Problem &p, const void *x, const void *w1p, const void *w2p, void *h,
                        void *out, float *part, unsigned *counters, int num_sms, cudaStream_t st,
                        const Marks &marks, int *launches) {
    GemvArgs a{};
    a.act = p.act;
    a.d_ff = p.d_ff;
    a.gpb = kGpb;
    a.counters = counters;
    a.part = part;
    // first projection + activation -> H
    a.w = static_cast<const __nv_bfloat16 *>(w1p);
    a.ldw = p.d_in;
    a.x = static_cast<const __nv_bfloat16 *>(x);
    a.K = p.d_in;
    a.groups = p.d_ff;
    a.out = static_cast<__nv_bfloat16 *>(h);
    plan_split(p.T, a.K, a.groups, num_sms, a.S, a.Kc);
    marks.mark(0, st);
    cudaError_t e = (p.act == TP_MLP_ACT_SWIGLU) ? launch_T<2, 0>(p.T, a, st) : launch_T<1, 0>(p.T, a, st);
    if (e != cudaSuccess) return e;
    marks.mark(1, st);
    // second projection over all ranks' rows (rank sum in the accumulator) -> out
    a.w = static_cast<const __nv_bfloat16 *>(w2p);
    a.ldw = p.d_ff;
    a.x = static_cast<const __nv_bfloat16 *>(h);
    a.K = p.d_ff;
    a.groups = p.d_out;
    a.out = static_cast<__nv_bfloat16 *>(out);
    plan_split(p.T, a.K, a.groups, num_sms, a.S, a.Kc);
    e = launch_T<1, 1>(p.T, a, st);
    marks.mark(2, st);
    if (launches) *launches = 2;
    return e;
}

}  // namespace tpmlp
