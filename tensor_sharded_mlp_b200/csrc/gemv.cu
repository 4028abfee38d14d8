// gemv.cu -- decode path: the MLP for 1..4 tokens on packed bf16 weights.
//
// Decode is memory-bound: every weight is read once per step and feeds only T
// multiply-adds ("7.4 推理侧并行", §7.4.1: at batch 1 the GEMM degenerates to a
// GEMV whose time is the weight read).  These kernels stream the tile-blocked
// packed weights at HBM speed with CUDA-core arithmetic:
//   * the weight stream is split evenly over the SMs (streamk.cuh): every CTA
//     reads one contiguous run of 32 KB blocks (256 rows x 64 k);
//   * one producer thread moves the blocks into a ring of shared-memory
//     stages with bulk copies (cp.async.bulk, 128 KB in flight per SM);
//   * the activations a CTA needs (the k-blocks of its share: at most one
//     tile's K, as a cyclic window) are bulk-copied into shared memory once,
//     as soon as the previous kernel is done, instead of being read per block
//     from L2 (whose latency, under a full weight stream, held back the CTAs
//     that saw the most of it: the step took 9 % longer);
//   * eight compute warps take 32 rows each; per step a lane reads one
//     16-byte granule (8 weights) of one row, so a warp reads 512 contiguous
//     bytes, and multiplies it with the matching 8 activations of each token;
//   * the 8 lanes that share a row add their sums with warp shuffles;
//   * a tile shared with other CTAs is finished by the last CTA to arrive,
//     adding the fp32 partial slots in slot order (no CTA waits on another).
// First projection: rows are features (SwiGLU: gate rows 0..127 and up rows
// 128..255 of each tile), H[t][n] = act(.).  Second projection: rows are
// output columns c with K = d_ff running over every rank's rows, so the sum
// over ranks happens in the accumulation; out[t][c].
#include "common.cuh"
#include "internal.h"
#include "streamk.cuh"
#include "tc_ptx.cuh"

namespace tpmlp {
namespace {

using namespace tc;

constexpr int CWARPS = 8;                    // compute warps
constexpr int NTHR = (CWARPS + 1) * 32;      // + one producer warp
#ifndef TPMLP_GEMV_STAGES
#define TPMLP_GEMV_STAGES 4   // 4 measured best on B200: the smaller carve-out leaves L1 room for X/H
#endif
constexpr int STAGES = TPMLP_GEMV_STAGES;   // shared-memory ring depth (32 KB per stage)
constexpr uint32_t BLK_BYTES = kTileRows * kKBlock * 2;   // 32 KB

enum { MODE_FIRST = 0, MODE_SECOND = 1 };

struct GemvArgs {
    const __nv_bfloat16 *w;   // packed part (tile-blocked)
    const __nv_bfloat16 *x;   // T x K activations, row-major
    int K, KB;
    long long total;          // tiles * KB
    int slots;
    int mode, act;
    int out_cols;             // d_ff (H) or d_out
    __nv_bfloat16 *out;       // T x out_cols
    float *part;              // [tile][slot][T][256] fp32
    unsigned *tile_cnt;       // k-blocks done per tile, zero between launches
    int *status;
    int xwin;                 // k-blocks of X staged in shared memory per token (0: read X from L2)
};

struct GemvSmem {
    uint8_t *ring;
    uint64_t *full, *empty;
    float *rowsum;            // [T][256]
    volatile int *abort;
    int *flag;
    uint64_t *xbar;           // completes when the staged X has landed
    __nv_bfloat16 *xs;        // [T][xwin][64] staged X, k-block kb at slot (kb - first kb) mod KB
};

constexpr size_t kSmemFixed = 128 + STAGES * (size_t)BLK_BYTES + 2 * STAGES * 8 + 16 + 128;
constexpr size_t kSmemOptin = 227 * 1024;   // largest dynamic shared memory of one CTA on sm_100

template <int T>
__device__ __forceinline__ GemvSmem gemv_carve(uint8_t *raw) {
    GemvSmem s;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 127) & ~uintptr_t(127));
    s.ring = base;
    s.full = reinterpret_cast<uint64_t *>(base + STAGES * BLK_BYTES);
    s.empty = s.full + STAGES;
    s.rowsum = reinterpret_cast<float *>(s.empty + STAGES);
    s.abort = reinterpret_cast<volatile int *>(s.rowsum + T * kTileRows);
    s.flag = const_cast<int *>(s.abort) + 1;
    s.xbar = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(s.flag) + 12);
    s.xs = reinterpret_cast<__nv_bfloat16 *>(reinterpret_cast<uint8_t *>(s.xbar) + 128);
    return s;
}

size_t gemv_smem_bytes(int T, int xwin) {
    return kSmemFixed + (size_t)T * kTileRows * 4 + (size_t)T * xwin * kKBlock * 2;
}

// Thread 0 of the compute warps: bulk-copy the X this CTA's share reads into
// s.xs.  The share's k-blocks form the cyclic window [kbs, kbs + W) mod KB, at
// most two contiguous runs of every token's row of X.  The last block of a row
// may be partial (K % 64 != 0); the readers skip k >= K.
template <int T>
__device__ __forceinline__ void stage_x(const GemvArgs &a, const GemvSmem &s, int kbs, int W) {
    const int r1e = min(a.KB, kbs + W);
    const int r2e = kbs + W - a.KB;   // > 0: the window wraps to k-block 0
    const uint32_t n1 = (uint32_t)(min(r1e * kKBlock, a.K) - kbs * kKBlock) * 2;
    const uint32_t n2 = r2e > 0 ? (uint32_t)min(r2e * kKBlock, a.K) * 2 : 0u;
    const uint32_t xb = smem_u32(s.xbar);
    mbar_arrive_expect_tx(xb, T * (n1 + n2));
#pragma unroll
    for (int t = 0; t < T; ++t) {
        __nv_bfloat16 *row = s.xs + (size_t)t * a.xwin * kKBlock;
        bulk_load(smem_u32(row), a.x + (long)t * a.K + kbs * kKBlock, n1, xb);
        if (n2) bulk_load(smem_u32(row + (size_t)(a.KB - kbs) * kKBlock), a.x + (long)t * a.K, n2, xb);
    }
}

// Final value of row `row` of tile `tile` for all tokens, from s.rowsum.
template <int T>
__device__ __forceinline__ void finish_row(const GemvArgs &a, const GemvSmem &s, int tile, int row) {
    if (a.mode == MODE_FIRST && a.act == TP_MLP_ACT_SWIGLU) {
        if (row >= kSwigluBlock) return;
        const int n = tile * kSwigluBlock + row;
        if (n >= a.out_cols) return;
#pragma unroll
        for (int t = 0; t < T; ++t)
            a.out[(long)t * a.out_cols + n] =
                __float2bfloat16_rn(silu_fast(s.rowsum[t * kTileRows + row]) * s.rowsum[t * kTileRows + row + 128]);
    } else {
        const int n = tile * kTileRows + row;
        if (n >= a.out_cols) return;
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const float v = s.rowsum[t * kTileRows + row];
            a.out[(long)t * a.out_cols + n] =
                __float2bfloat16_rn(a.mode == MODE_FIRST ? activate<true>(a.act, v, 0.f) : v);
        }
    }
}

template <int T, bool XS>
__global__ void __launch_bounds__(NTHR, 1) gemv_kernel(GemvArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const GemvSmem s = gemv_carve<T>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(smem_u32(&s.full[i]), 1);
            mbar_init(smem_u32(&s.empty[i]), CWARPS);
        }
        mbar_init(smem_u32(s.xbar), 1);
        *s.abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_allow_dependents();

    const long long total = a.total, G = gridDim.x, c = blockIdx.x;
    const long long it_b = share_begin(c, total, G), it_e = share_begin(c + 1, total, G);
    const int KB = a.KB;

    if (warp == CWARPS) {
        // producer: weights do not depend on the previous kernel, so start at once
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            const uint8_t *src = reinterpret_cast<const uint8_t *>(a.w) + it_b * (long long)BLK_BYTES;
            for (long long it = it_b; it < it_e; ++it) {
                if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1, s.abort)) break;
                const uint32_t fb = smem_u32(&s.full[stage]);
                mbar_arrive_expect_tx(fb, BLK_BYTES);
                bulk_load(smem_u32(s.ring + stage * BLK_BYTES), src, BLK_BYTES, fb);
                src += BLK_BYTES;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else {
        pdl_wait_previous();   // X and the outputs belong to the previous kernel until it is done
        const int kbs = (int)(it_b % KB);
        bool xok = true;
        if (XS) {
            if (threadIdx.x == 0) stage_x<T>(a, s, kbs, (int)min((long long)KB, it_e - it_b));
            xok = mbar_wait(smem_u32(s.xbar), 0, s.abort);
            xok = !named_bar_or(1, CWARPS * 32, !xok);   // all compute threads alike
        }
        const int g = lane & 7;                         // granule (8 k) of the row
        const int rbase = warp * 32 + (lane >> 3);      // rows rbase + 4j, j = 0..7
        int stage = 0;
        uint32_t phase = 0;
        for (long long it = it_b; xok && it < it_e;) {
            const int tile = (int)(it / KB);
            const int kb0 = (int)(it - (long long)tile * KB);
            const int kb1 = (int)min((long long)KB, it_e - (long long)tile * KB);
            it = (long long)tile * KB + kb1;
            float acc[8][T];
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int t = 0; t < T; ++t) acc[j][t] = 0.f;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                // this lane's 8 activations of every token for k = kb*64 + 8g ..
                float xv[T][8];
                const int k = kb * kKBlock + g * 8;
                const int slot = kb - kbs + (kb < kbs ? KB : 0);
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    if (k < a.K) {   // K is a multiple of 8: a granule is all in or all out
                        const uint4 w4 =
                            XS ? *reinterpret_cast<const uint4 *>(s.xs + ((size_t)t * a.xwin + slot) * kKBlock + g * 8)
                               : __ldg(reinterpret_cast<const uint4 *>(a.x + (long)t * a.K + k));
                        xv[t][0] = bf16lo(w4.x); xv[t][1] = bf16hi(w4.x);
                        xv[t][2] = bf16lo(w4.y); xv[t][3] = bf16hi(w4.y);
                        xv[t][4] = bf16lo(w4.z); xv[t][5] = bf16hi(w4.z);
                        xv[t][6] = bf16lo(w4.w); xv[t][7] = bf16hi(w4.w);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) xv[t][i] = 0.f;
                    }
                }
                if (!mbar_wait(smem_u32(&s.full[stage]), phase, s.abort)) { ok = false; break; }
                const uint4 *blk = reinterpret_cast<const uint4 *>(s.ring + stage * BLK_BYTES);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 wv = blk[(rbase + 4 * j) * 8 + g];
                    const float w0 = bf16lo(wv.x), w1 = bf16hi(wv.x), w2 = bf16lo(wv.y), w3 = bf16hi(wv.y);
                    const float w4 = bf16lo(wv.z), w5 = bf16hi(wv.z), w6 = bf16lo(wv.w), w7 = bf16hi(wv.w);
#pragma unroll
                    for (int t = 0; t < T; ++t) {
                        float v = acc[j][t];
                        v = fmaf(w0, xv[t][0], v); v = fmaf(w1, xv[t][1], v);
                        v = fmaf(w2, xv[t][2], v); v = fmaf(w3, xv[t][3], v);
                        v = fmaf(w4, xv[t][4], v); v = fmaf(w5, xv[t][5], v);
                        v = fmaf(w6, xv[t][6], v); v = fmaf(w7, xv[t][7], v);
                        acc[j][t] = v;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&s.empty[stage]));
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            // leave together if a wait gave up in any warp (the barriers below need all)
            if (named_bar_or(1, CWARPS * 32, !ok)) break;
            // the 8 lanes of a row hold partial sums of its 8 granules
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    float v = acc[j][t];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    acc[j][t] = v;
                }
            if (g == 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
#pragma unroll
                    for (int t = 0; t < T; ++t) s.rowsum[t * kTileRows + rbase + 4 * j] = acc[j][t];
            }
            named_bar(1, CWARPS * 32);
            const int row = threadIdx.x;   // 0..255: one row per compute thread
            if (kb0 == 0 && kb1 == KB) {
                finish_row<T>(a, s, tile, row);
            } else {
                const int c_first = share_owner((long long)tile * KB, total, G);
                const int c_last = share_owner((long long)tile * KB + KB - 1, total, G);
                float *mine = a.part + ((long long)tile * a.slots + ((int)c - c_first)) * T * kTileRows;
#pragma unroll
                for (int t = 0; t < T; ++t) mine[t * kTileRows + row] = s.rowsum[t * kTileRows + row];
                __threadfence();
                named_bar(1, CWARPS * 32);
                if (threadIdx.x == 0) {
                    const unsigned done = atomicAdd(&a.tile_cnt[tile], (unsigned)(kb1 - kb0)) + (kb1 - kb0);
                    *s.flag = (done == (unsigned)KB);
                }
                named_bar(1, CWARPS * 32);
                if (*s.flag) {
                    __threadfence();
                    const float *tb = a.part + (long long)tile * a.slots * T * kTileRows;
#pragma unroll
                    for (int t = 0; t < T; ++t) {
                        float v = 0.f;
                        for (int sl = 0; sl <= c_last - c_first; ++sl)
                            v += __ldcg(tb + ((long long)sl * T + t) * kTileRows + row);
                        s.rowsum[t * kTileRows + row] = v;
                    }
                    named_bar(1, CWARPS * 32);
                    finish_row<T>(a, s, tile, row);
                    if (threadIdx.x == 0) a.tile_cnt[tile] = 0u;
                }
            }
            named_bar(1, CWARPS * 32);   // rowsum and the flag are reused by the next tile
        }
    }
    if (*s.abort) {
        // a bounded wait gave up: let bulk copies in flight land before the CTA exits
        if (threadIdx.x == 0) {
            const unsigned long long t0 = globaltimer();
            while (globaltimer() - t0 < 100000ull) {
            }
            atomicExch(a.status, 1);
        }
    }
    __syncthreads();
}

StreamKGeom gemv_geom(long long rows, int K, int num_sms) {
    return streamk_geom(blk_tiles(rows), blk_kblocks(K), num_sms);
}

template <int T, bool XS>
cudaError_t launch_one(const GemvArgs &a, int grid, cudaStream_t st) {
    const size_t smem = gemv_smem_bytes(T, XS ? a.xwin : 0);
    auto kern = gemv_kernel<T, XS>;
    cudaError_t e = ensure_smem_attr(kern, kSmemOptin);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(grid), dim3(NTHR), smem, st, a);
}

template <int T>
cudaError_t launch_one(const GemvArgs &a, int grid, cudaStream_t st) {
    return a.xwin > 0 ? launch_one<T, true>(a, grid, st) : launch_one<T, false>(a, grid, st);
}

cudaError_t launch_T(int T, const GemvArgs &a, int grid, cudaStream_t st) {
    switch (T) {
        case 1: return launch_one<1>(a, grid, st);
        case 2: return launch_one<2>(a, grid, st);
        case 3: return launch_one<3>(a, grid, st);
        case 4: return launch_one<4>(a, grid, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t run_part(const void *w, long long rows, int K, const void *x, int T, int mode, int act, void *out,
                     int out_cols, float *part, unsigned *cnt, int *status, int num_sms, cudaStream_t st) {
    const StreamKGeom g = gemv_geom(rows, K, num_sms);
    GemvArgs a{};
    a.w = static_cast<const __nv_bfloat16 *>(w);
    a.x = static_cast<const __nv_bfloat16 *>(x);
    a.K = K;
    a.KB = g.KB;
    a.total = g.total;
    a.slots = g.slots;
    a.mode = mode;
    a.act = act;
    a.out_cols = out_cols;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.part = part;
    a.tile_cnt = cnt;
    a.status = status;
    // a share spans at most ceil(total / grid) k-blocks, and the window never more than one tile's K
    a.xwin = (int)std::min<long long>(g.KB, (g.total + g.grid - 1) / g.grid);
    if (gemv_smem_bytes(T, a.xwin) > kSmemOptin) a.xwin = 0;
    return launch_T(T, a, g.grid, st);
}

}  // namespace

bool gemv_supported(const Problem &p) {
    return p.dtype == TP_MLP_BF16 && p.T >= 1 && p.T <= kGemvMaxTokens && p.d_in % 8 == 0 && p.d_ff % 8 == 0;
}

size_t gemv_workspace_bytes(const Problem &p, int num_sms) {
    if (!gemv_supported(p)) return 0;
    const StreamKGeom g1 = gemv_geom(w1p_rows(p.d_ff, p.act), p.d_in, num_sms);
    const StreamKGeom g2 = gemv_geom(p.d_out, p.d_ff, num_sms);
    const size_t m = std::max((size_t)g1.tiles * g1.slots, (size_t)g2.tiles * g2.slots);
    return align256(m * p.T * kTileRows * 4);
}

cudaError_t launch_gemv(const Problem &p, const void *x, const void *w1p, const void *w2p, void *h, void *out,
                        float *part, unsigned *counters, int *status, int num_sms, cudaStream_t st,
                        const Marks &marks, int *launches) {
    const long long rows1 = w1p_rows(p.d_ff, p.act);
    unsigned *cnt1 = counters, *cnt2 = counters + blk_tiles(rows1);
    marks.mark(0, st);
    cudaError_t e = run_part(w1p, rows1, p.d_in, x, p.T, MODE_FIRST, p.act, h, p.d_ff, part, cnt1, status,
                             num_sms, st);
    if (e != cudaSuccess) return e;
    marks.mark(1, st);
    e = run_part(w2p, p.d_out, p.d_ff, h, p.T, MODE_SECOND, p.act, out, p.d_out, part, cnt2, status, num_sms, st);
    marks.mark(2, st);
    if (launches) *launches = 2;
    return e;
}

}  // namespace tpmlp
