// tc_gemm.cu -- tensor-core path for bf16: tcgen05 MMA with TMEM accumulators,
// operands streamed by TMA through a shared-memory ring, warp-specialised.
//
// Both projections are GEMMs over the packed K-major weights W (rows x K):
//   first  ("大模型推理系统揭秘（07）", §1.2.2 column-parallel):  U = X W1^T,
//          H = tanh(U) or SiLU(U_gate) * U_up (§1.4.3), fused in the epilogue;
//   second (§1.2.2 row-parallel + §1.2.3 sum of partials):  Z = H W2^T, one
//          K loop over every rank's rows, so the ranks' partial sums accumulate
//          in TMEM and never reach HBM.
//
// Two tilings share the pipeline code:
//   wide   (many tokens, compute-bound): the MMA's M is 128 tokens and its N is
//          256 weight rows; persistent CTAs walk the tiles in groups of
//          kGroupM token tiles so a weight tile is reused from L2;
//   skinny (few tokens, memory-bound, the decode case "7.4 推理侧并行" §7.4.1
//          describes): operands swapped -- M is 128 weight rows (two MMAs per
//          256-row weight tile, or one per 128-row tile), N is the token count
//          rounded up to BT.  The weight stream is cut into equal contiguous
//          shares, one per CTA ("stream-K"), or -- with few tiles -- a whole
//          number of CTAs per tile; a tile split between CTAs is finished from
//          fp32 partial slots added in a fixed order, either by a reduction
//          kernel behind the GEMM (default) or by the last CTA to arrive.
//          Nothing waits on another CTA.
//
// Roles: warp 0 lane 0 issues TMA loads, warp 1 allocates TMEM and lane 0
// issues the MMAs, warps 2..5 run the epilogue (TMEM lanes 32*(warp%4)...).
// Every mbarrier wait is bounded (tc_ptx.cuh); a wait that runs out raises an
// abort flag that every role checks, and the CTA records it in a status word.
#include <cuda.h>

#include <string.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "streamk.cuh"
#include "tc_ptx.cuh"

namespace tpmlp {
namespace {

using namespace tc;

constexpr int BK = 64;              // K per stage: one 128-byte swizzle row of bf16
constexpr int NTHREADS = 192;
constexpr int kGroupM = 8;          // wide tiling: token tiles per raster group
constexpr int kWideStages = 4;

// EPI_PART: the second projection of one rank at a time, fp32 outputs
// (tp_mlp_partials: Z_i = H_i B_i without the sum over ranks).
// EPI_AR: the same per-rank second projection, then the one-shot all-reduce
// across ranks (cross-GPU tensor parallelism; see the cluster exit below).
enum { EPI_H_TANH = 0, EPI_H_SWIGLU = 1, EPI_H_IDENT = 2, EPI_OUT = 3, EPI_PART = 4, EPI_AR = 5 };

struct TcArgs {
    int rows_x;          // X rows (tokens)
    int rows_w;          // W rows
    int K, KB;           // K and ceil(K / BK)
    int epi;
    __nv_bfloat16 *out;  // H (T x d_ff) or out (T x d_out)
    int ldo;             // row stride of out = out_cols
    int out_cols;
    // skinny tiling (stream-K)
    long long total_iters;
    int slots;           // partial slots per weight tile
    float *part;         // [tile][slot][BT/4][256][4] fp32 (float4 per row and 4 tokens)
    unsigned *tile_cnt;  // k-blocks done per weight tile, zero between launches
    int split_mode;      // kSplitInKernel or kSplitSeparate (see internal.h)
    int grid;            // CTAs of the skinny launch (the stream-K split)
    int *status;         // set to 1 if a bounded wait ran out
    // first projection read straight from the per-rank shards: tile t covers
    // features of rank t / tps only (tps tiles per rank of fs features)
    int raw_first, tps, fs;
    // per-rank partials (EPI_PART): weight tile t is output tile t % otiles of
    // rank t / otiles, whose K loop is that rank's KB k-blocks of the full K
    // (k-block offset rank * KB); results go to pout[rank][token][column]
    int prank, otiles;
    float *pout;
    // skinny whole-CTA grids: the n CTAs sharing a tile form one thread-block
    // cluster and add their partials through distributed shared memory (0: off)
    int cluster_red;
    // one-shot all-reduce (EPI_AR): this launch computes ranks ar_rank0 ..
    // ar_rank0 + prank - 1 of ar_ranks; comm[p] is rank p's buffer as this
    // process sees it: [control: epoch, finished-CTA count (256 B) | flags:
    // ar_ranks x otiles x 8 u32 | recv: 2 (epoch parity) x ar_ranks x ar_rows
    // x ldo bf16].  outs[i]: the output of local rank i (tokens x ldo bf16).
    int ar_rank0, ar_ranks, ar_rows;
    size_t recv_off;
    uint8_t *comm[kMaxTp];
    __nv_bfloat16 *outs[kMaxTp];
    // sequence parallelism: rank o owns token rows [o sp_rows, (o + 1) sp_rows).
    // EPI_AR with sp_rows > 0 is a reduce-scatter: a row goes only to its
    // owner, which writes its own rows (outs[i]: sp_rows x ldo).  A first
    // projection with sp_wait != nullptr reads X gathered from every rank and
    // first waits until all ar_ranks arrival counts sp_wait[src] reach
    // calls * sp_per_src (calls = *sp_epoch + 1: this is the next
    // sequence-parallel call).
    int sp_rows;
    const unsigned *sp_wait;
    const unsigned *sp_epoch;
    unsigned sp_per_src;
};

// Weight tile and k-block of the full weight / activation that iteration
// (tile, kb) of a launch reads.  Only the per-rank partials remap them.
__device__ __forceinline__ int w_tile(const TcArgs &a, int tile) { return a.prank ? tile % a.otiles : tile; }
__device__ __forceinline__ int k_block(const TcArgs &a, int tile, int kb) {
    return a.prank ? (tile / a.otiles) * a.KB + kb : kb;
}
// Row t of rank (tile / otiles)'s fp32 partial output.
__device__ __forceinline__ float *part_row(const TcArgs &a, int tile, int t) {
    return a.pout + ((long)(tile / a.otiles) * a.rows_x + t) * a.ldo;
}

// --- thread-block clusters (split tiles added through distributed shared memory) ---
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Hardware cluster barrier (no spinning; not the .aligned form, so a warp whose
// lanes arrive apart is fine).  Every thread of every CTA of the cluster must
// arrive, on every path, or the others wait for ever: the skinny kernel calls
// it only from its common exit.
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// 16 bytes at the same shared-memory address in CTA `rank` of the cluster.
__device__ __forceinline__ float4 ld_cluster_f4(const void *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(remote)
                 : "memory");
    return v;
}

// --- the one-shot all-reduce across ranks (EPI_AR) ---------------------------------
__device__ __forceinline__ void st_release_sys(unsigned *p, unsigned v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_sys(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Per rank: [0] last finished epoch, [1] finished-CTA count, [2] sequence-
// parallel calls finished, [8 + src] rows of rank src gathered here by
// sequence-parallel calls (in CTAs of the gather; counts only grow).
constexpr int kArControlBytes = 256;
__device__ __forceinline__ unsigned *ar_control(const TcArgs &a, int p) {
    return reinterpret_cast<unsigned *>(a.comm[p]);
}
__device__ __forceinline__ unsigned *ar_flag(const TcArgs &a, int p, int src, int otile, int j) {
    return reinterpret_cast<unsigned *>(a.comm[p] + kArControlBytes) + ((size_t)src * a.otiles + otile) * 8 + j;
}
__device__ __forceinline__ __nv_bfloat16 *ar_recv_row(const TcArgs &a, unsigned epoch, int p, int src, int t) {
    return reinterpret_cast<__nv_bfloat16 *>(a.comm[p] + a.recv_off) +
           (((size_t)(epoch & 1u) * a.ar_ranks + src) * a.ar_rows + t) * a.ldo;
}

// Weight operand of one projection, for the producer's TMA loads.
//   packed: map[0] views the tile-blocked part; one 32 KB box per (tile, k-block).
//   raw:    per-rank row-major shards; four 64 (columns) x 64 (k rows) boxes per
//           (tile, k-block).  First projection: map[i] = A_i (tanh) or gate_i,
//           map[kMaxTp + i] = up_i; a tile is 256 features (tanh) or 128 gate +
//           the same 128 up features (SwiGLU) of one rank.  Second projection:
//           map[i] = B_i; a tile is 256 output columns, k-block kb comes from
//           rank kb / kbps.
struct WeightMaps {
    CUtensorMap map[2 * kMaxTp];
    int first, swiglu, tps, kbps;
};

// HALF: 128-row tiles (tile t = rows [128 (t % 2), +128) of 256-row block t / 2
// in the packed layout; two 64-column boxes in the shard form).
template <bool RAW, bool HALF = false>
__device__ __forceinline__ void load_w_tile(uint32_t dst, const WeightMaps &wm, int tile, int kb, int KB,
                                            uint32_t bar) {
    if (!RAW) {
        if (HALF)
            tma_load_2d(dst, &wm.map[0], 0, ((tile >> 1) * KB + kb) * 256 + (tile & 1) * 128, bar);
        else
            tma_load_2d(dst, &wm.map[0], 0, (tile * KB + kb) * 256, bar);
        return;
    }
    if (HALF) {   // tanh / identity first projection or the second projection: 128 columns
        if (wm.first) {
            const int i = tile / wm.tps, n0 = (tile - i * wm.tps) * 128;
#pragma unroll
            for (int q = 0; q < 2; ++q) tma_load_2d(dst + q * 8192, &wm.map[i], n0 + 64 * q, kb * BK, bar);
        } else {
            const int i = kb / wm.kbps, kl = kb - i * wm.kbps;
#pragma unroll
            for (int q = 0; q < 2; ++q) tma_load_2d(dst + q * 8192, &wm.map[i], tile * 128 + 64 * q, kl * BK, bar);
        }
        return;
    }
    if (wm.first) {
        const int per = wm.swiglu ? 128 : 256;
        const int i = tile / wm.tps, n0 = (tile - i * wm.tps) * per;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const CUtensorMap *m = (wm.swiglu && q >= 2) ? &wm.map[kMaxTp + i] : &wm.map[i];
            const int x = n0 + 64 * (wm.swiglu ? (q & 1) : q);
            tma_load_2d(dst + q * 8192, m, x, kb * BK, bar);
        }
    } else {
        const int i = kb / wm.kbps, kl = kb - i * wm.kbps;
#pragma unroll
        for (int q = 0; q < 4; ++q) tma_load_2d(dst + q * 8192, &wm.map[i], tile * 256 + 64 * q, kl * BK, bar);
    }
}

// Output column of element `local` (0 .. per-1) of weight tile `tile`, or -1 when
// it is padding.  per = 128 for the SwiGLU first projection, 256 otherwise.
__device__ __forceinline__ int tile_col(const TcArgs &a, int tile, int local, int per) {
    if (!a.raw_first) {
        const int n = tile * per + local;
        return n < a.out_cols ? n : -1;
    }
    const int i = tile / a.tps, l = (tile - i * a.tps) * per + local;
    return l < a.fs ? i * a.fs + l : -1;
}

__device__ __forceinline__ float act_out(int epi, float u) {
    if (epi == EPI_H_TANH) return tanh_fast(u);
    return u;   // identity / plain output
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Shared-memory carve-up common to both tilings.
struct Smem {
    uint8_t *a, *b;           // stage rings (1024-aligned)
    uint64_t *full, *empty;   // per stage
    uint64_t *tfull, *tempty; // per accumulator buffer (2)
    uint64_t *drain;          // abort path: waits for the MMAs in flight
    uint32_t *tmem_slot;
    volatile int *abort;
    int *flag;
};

template <int STAGES>
__device__ __forceinline__ Smem carve(uint8_t *raw, uint32_t a_bytes, uint32_t b_bytes) {
    Smem s;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.a = base;
    s.b = base + STAGES * a_bytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(s.b + STAGES * b_bytes);
    s.full = bars;
    s.empty = bars + STAGES;
    s.tfull = bars + 2 * STAGES;
    s.tempty = bars + 2 * STAGES + 2;
    s.drain = bars + 2 * STAGES + 4;
    s.tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
    s.abort = reinterpret_cast<volatile int *>(s.tmem_slot + 1);
    s.flag = reinterpret_cast<int *>(s.tmem_slot + 2);
    return s;
}

template <int STAGES>
constexpr size_t smem_bytes(uint32_t a_bytes, uint32_t b_bytes) {
    return 1024 + STAGES * (size_t)(a_bytes + b_bytes) + (2 * STAGES + 5) * 8 + 16;
}

// Setup shared by both kernels: barriers, TMEM (512 columns), descriptor prefetch.
template <int STAGES>
__device__ __forceinline__ uint32_t setup(const Smem &s, const CUtensorMap *m0, const CUtensorMap *m1) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(smem_u32(&s.full[i]), 1);
            mbar_init(smem_u32(&s.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&s.tfull[i]), 1);
            mbar_init(smem_u32(&s.tempty[i]), 4);
        }
        mbar_init(smem_u32(s.drain), 1);
        *s.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(m0);
        tma_prefetch_desc(m1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(s.tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *s.tmem_slot;
}

__device__ __forceinline__ void teardown(const Smem &s, uint32_t tmem_base, int *status) {
    if (*s.abort) {
        // A bounded wait gave up somewhere.  Before TMEM and shared memory are
        // released: let the MMA issuer's MMAs finish, and give TMA copies in
        // flight time to land (both bounded).
        if (threadIdx.x == 32) {
            mma_commit(smem_u32(s.drain));
            volatile int never = 0;
            mbar_wait(smem_u32(s.drain), 0, &never);
        }
        if (threadIdx.x == 0) {
            const unsigned long long t0 = globaltimer();
            while (globaltimer() - t0 < 100000ull) {
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
    if (threadIdx.x == 0 && *s.abort) atomicExch(status, 1);
}

// ============ wide tiling: 128*MH tokens x 256 weight rows per tile ============
// MH = 1: one M=128 MMA per 16-k step, two TMEM accumulator buffers (the
//         epilogue of one tile overlaps the next tile's MMAs), 4 stages.
// MH = 2: two M=128 MMAs share every weight tile (256 tokens per tile), so a
//         FLOP costs a third less operand traffic from L2; the 2 x 256-column
//         accumulator fills TMEM, so there is one buffer, 3 stages.

__device__ __forceinline__ void wide_tile(int u, int MT, int NT, int &mt, int &nt) {
    const int per_group = kGroupM * NT;
    const int g = u / per_group;
    const int gm = min(kGroupM, MT - g * kGroupM);
    const int r = u - g * per_group;
    nt = r / gm;
    mt = g * kGroupM + r % gm;
}

template <int MH>
struct WideCfg {
    static constexpr int STAGES = MH == 1 ? kWideStages : 3;
    static constexpr int NACC = MH == 1 ? 2 : 1;          // TMEM accumulator buffers
    static constexpr uint32_t A_BYTES = 128 * MH * BK * 2;
    static constexpr uint32_t B_BYTES = 256 * BK * 2;
};

// Epilogue of one 128-token half: TMEM lanes = tokens, columns 0..255 = weight rows.
// Output columns come in runs of 16 that are all valid or all padding, except
// at a packed part's ragged end (handled element by element).
__device__ __forceinline__ void wide_epilogue_part(const TcArgs &a, int row, int nt, uint32_t taddr) {
    const bool row_ok = row < a.rows_x;
    float *orow = row_ok ? part_row(a, nt, row) : nullptr;
    const int ot = w_tile(a, nt);
#pragma unroll 1
    for (int j = 0; j < 16; ++j) {
        float g[16];
        tmem_ld16(taddr + 16 * j, g);
        tmem_ld_wait();
        const int col = tile_col(a, ot, 16 * j, 256);
        if (!row_ok || col < 0) continue;
        if (col + 16 <= a.out_cols) {
            float4 *dst = reinterpret_cast<float4 *>(orow + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_float4(g[4 * i], g[4 * i + 1], g[4 * i + 2], g[4 * i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (col + i < a.out_cols) orow[col + i] = g[i];
        }
    }
}

__device__ __forceinline__ void wide_epilogue_half(const TcArgs &a, int row, int nt, uint32_t taddr) {
    if (a.epi == EPI_PART) {
        wide_epilogue_part(a, row, nt, taddr);
        return;
    }
    const bool row_ok = row < a.rows_x;
    __nv_bfloat16 *orow = a.out + (long)row * a.ldo;
    const bool swiglu = a.epi == EPI_H_SWIGLU;
    const int per = swiglu ? 128 : 256;
#pragma unroll 1
    for (int j = 0; j < per / 16; ++j) {
        float g[16], v[16];
        tmem_ld16(taddr + 16 * j, g);
        if (swiglu) tmem_ld16(taddr + 128 + 16 * j, v);
        tmem_ld_wait();
        const int col = tile_col(a, nt, 16 * j, per);
        if (!row_ok || col < 0) continue;
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = swiglu ? silu_fast(g[i]) * v[i] : act_out(a.epi, g[i]);
        if (a.raw_first || col + 16 <= a.out_cols) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
            uint4 *dst = reinterpret_cast<uint4 *>(orow + col);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)   // unrolled so y stays in registers
                if (col + i < a.out_cols) orow[col + i] = __float2bfloat16_rn(y[i]);
        }
    }
}

template <int MH, bool RAW>
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_wide_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ WeightMaps wm, TcArgs a) {
    using C = WideCfg<MH>;
    constexpr int STAGES = C::STAGES;
    constexpr int NACC = C::NACC;
    constexpr uint32_t A_BYTES = C::A_BYTES;   // X tile: 128*MH tokens
    constexpr uint32_t B_BYTES = C::B_BYTES;   // W tile: 256 rows
    extern __shared__ uint8_t smem_raw[];
    const Smem s = carve<STAGES>(smem_raw, A_BYTES, B_BYTES);
    const uint32_t tmem_base = setup<STAGES>(s, &tmX, &wm.map[0]);
    pdl_allow_dependents();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int MT = (a.rows_x + 128 * MH - 1) / (128 * MH), NT = a.rows_w;   // rows_w: weight tiles
    const int units = MT * NT;

    if (warp == 0) {
        if (lane == 0) {
            pdl_wait_previous();   // X / H come from the previous kernel
            int stage = 0;
            uint32_t phase = 0;
            for (int u = blockIdx.x; u < units; u += gridDim.x) {
                int mt, nt;
                wide_tile(u, MT, NT, mt, nt);
                for (int kb = 0; kb < a.KB; ++kb) {
                    if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1, s.abort)) goto done;
                    const uint32_t fb = smem_u32(&s.full[stage]);
                    mbar_arrive_expect_tx(fb, A_BYTES + B_BYTES);
                    const int gkb = k_block(a, nt, kb);
                    tma_load_2d(smem_u32(s.a + stage * A_BYTES), &tmX, gkb * BK, mt * 128 * MH, fb);
                    load_w_tile<RAW>(smem_u32(s.b + stage * B_BYTES), wm, w_tile(a, nt), gkb, a.KB, fb);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, 256) | (RAW ? kIdescBMajorMN : 0u);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < units; u += gridDim.x) {
                if (!mbar_wait(smem_u32(&s.tempty[acc]), acc_phase ^ 1, s.abort)) goto done;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * 256 * MH;
                for (int kb = 0; kb < a.KB; ++kb) {
                    if (!mbar_wait(smem_u32(&s.full[stage]), phase, s.abort)) goto done;
                    tc_fence_after();
                    const uint32_t sa = smem_u32(s.a + stage * A_BYTES);
                    const uint32_t sb = smem_u32(s.b + stage * B_BYTES);
                    // K-major: +32 bytes per 16 k (+2 in the address field); MN-major: +2048 bytes (+128)
                    const uint64_t db = RAW ? smem_desc_mnmajor_sw128(sb) : smem_desc_kmajor_sw128(sb);
                    constexpr uint32_t kstep_b = RAW ? 128 : 2;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
#pragma unroll
                        for (int h = 0; h < MH; ++h)      // token half h: rows 128h.. of the X tile
                            mma_bf16(d + h * 256, smem_desc_kmajor_sw128(sa + h * 128 * 128) + 2 * k,
                                     db + kstep_b * k, idesc, (kb | k) != 0);
                    }
                    mma_commit(smem_u32(&s.empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                mma_commit(smem_u32(&s.tfull[acc]));
                if (++acc == NACC) { acc = 0; acc_phase ^= 1; }
            }
        }
    } else {
        // epilogue: TMEM lane quadrant q holds tokens 32q..32q+31 of each 128-token half
        pdl_wait_previous();   // outputs may still be read by the previous kernel
        const int q = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            int mt, nt;
            wide_tile(u, MT, NT, mt, nt);
            if (!mbar_wait(smem_u32(&s.tfull[acc]), acc_phase, s.abort)) break;
            tc_fence_after();
#pragma unroll 1
            for (int h = 0; h < MH; ++h)
                wide_epilogue_half(a, mt * 128 * MH + h * 128 + q * 32 + lane, nt,
                                   tmem_base + (acc * MH + h) * 256 + ((uint32_t)(q * 32) << 16));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&s.tempty[acc]));
            if (++acc == NACC) { acc = 0; acc_phase ^= 1; }
        }
    }
done:
    teardown(s, tmem_base, a.status);
}

// ============ pair tiling: 256 tokens x 256 weight rows per pair of CTAs ============
// A cluster of two CTAs computes each tile with cta_group::2 MMAs (M = 256
// tokens, N = 256 weight rows).  CTA r of the pair loads tokens [128 r, 128 r
// + 128) of the tile and weight rows [128 r, 128 r + 128) -- 32 KB per stage,
// so 6 stages fit -- and holds its 128 tokens x 256 rows of the accumulator in
// its own TMEM: two buffers in 512 columns, so one tile's epilogue overlaps the
// next tile's MMAs (the 1-CTA 256-token tiling has room for one buffer only).
// Per FLOP the operands cost the same L2 traffic as the 256-token tiling, and
// each tensor core reads a third less shared memory.  The pair's first CTA
// issues the MMAs and owns the mbarriers that both CTAs' loads complete on;
// its commits arrive on the barriers of both CTAs, and both CTAs' epilogues
// hand the accumulator back to it.  Packed weights only.
// NB = 2: each unit is 256 tokens x 512 weight rows -- two weight tiles share
// every X stage (two M=256 MMAs per 16-k step), so a CTA loads 48 KB per stage
// for twice the FLOPs of 32 KB: a quarter less operand traffic per FLOP than
// the 1-CTA 256-token tiling, which lowers the power a prefill-size GEMM draws
// under the 1 kW cap.  Its two 256-column accumulators fill TMEM, so there is
// one buffer and the epilogue does not overlap the MMAs.
constexpr int kPairStages = 6;
constexpr int kPair2Stages = 4;

__device__ __forceinline__ void pair_teardown(const Smem &s, uint32_t tmem_base, uint32_t rank, int *status) {
    // The first CTA waits until its MMAs and their commits (which also arrive
    // in the other CTA) are done; then neither CTA leaves while the other may
    // still touch its shared memory or TMEM.
    if (threadIdx.x == 32 && rank == 0) {
        mma_commit_pair_local(smem_u32(s.drain));
        volatile int never = 0;
        mbar_wait(smem_u32(s.drain), 0, &never);
    }
    if (*s.abort && threadIdx.x == 0) {   // a bounded wait gave up: let copies in flight land
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 100000ull) {
        }
    }
    tc_fence_before();
    __syncwarp();
    cluster_barrier();
    if ((threadIdx.x >> 5) == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
    if (threadIdx.x == 0 && *s.abort) atomicExch(status, 1);
}

template <int STAGES, int NB>
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ WeightMaps wm, TcArgs a) {
    constexpr uint32_t A_BYTES = 128 * BK * 2;        // this CTA's 128 tokens of a stage
    constexpr uint32_t B_BYTES = NB * 128 * BK * 2;   // this CTA's 128 rows of each of NB weight tiles
    constexpr int NACC = NB == 1 ? 2 : 1;             // TMEM accumulator buffers (NB x 256 columns each)
    extern __shared__ uint8_t smem_raw[];
    const Smem s = carve<STAGES>(smem_raw, A_BYTES, B_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(smem_u32(&s.full[i]), 1);
            mbar_init(smem_u32(&s.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&s.tfull[i]), 1);
            mbar_init(smem_u32(&s.tempty[i]), 8);   // 4 epilogue warps in each CTA
        }
        mbar_init(smem_u32(s.drain), 1);
        *s.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&wm.map[0]);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(s.tmem_slot), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_barrier();   // both CTAs' barriers exist before anything arrives on them
    tc_fence_after();
    const uint32_t tmem_base = *s.tmem_slot;
    pdl_allow_dependents();

    const int MT = (a.rows_x + 255) / 256;
    const int NT = (a.rows_w + NB - 1) / NB;   // rows_w: 256-row weight tiles; a unit takes NB of them
    const int units = MT * NT;
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
    const int KB = a.KB;

    if (warp == 0) {
        if (lane == 0) {
            pdl_wait_previous();   // X / H come from the previous kernel
            const uint32_t full0 = cluster_addr(smem_u32(&s.full[0]), 0);   // the first CTA's full[0]
            int stage = 0;
            uint32_t phase = 0;
            for (int u = pair; u < units; u += npairs) {
                int mt, nt;
                wide_tile(u, MT, NT, mt, nt);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1, s.abort)) goto done;
                    if (rank == 0) mbar_arrive_expect_tx(smem_u32(&s.full[stage]), 2 * (A_BYTES + B_BYTES));
                    const uint32_t fb = full0 + 8u * stage;
                    tma_load_2d_pair(smem_u32(s.a + stage * A_BYTES), &tmX, kb * BK, mt * 256 + (int)rank * 128, fb);
#pragma unroll
                    for (int j = 0; j < NB; ++j) {   // a tile past the end loads the last one again (discarded)
                        const int wt = min(nt * NB + j, a.rows_w - 1);
                        tma_load_2d_pair(smem_u32(s.b + stage * B_BYTES + j * 16384), &wm.map[0], 0,
                                         (wt * KB + kb) * 256 + (int)rank * 128, fb);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = idesc_bf16_f32(256, 256);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int u = pair; u < units; u += npairs) {
                if (!mbar_wait(smem_u32(&s.tempty[acc]), acc_phase ^ 1, s.abort)) goto done;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * 256 * NB;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(smem_u32(&s.full[stage]), phase, s.abort)) goto done;
                    tc_fence_after();
                    const uint64_t da = smem_desc_kmajor_sw128(smem_u32(s.a + stage * A_BYTES));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
#pragma unroll
                        for (int j = 0; j < NB; ++j)
                            mma_bf16_pair(d + 256 * j, da + 2 * k,
                                          smem_desc_kmajor_sw128(smem_u32(s.b + stage * B_BYTES + j * 16384)) + 2 * k,
                                          idesc, (kb | k) != 0);
                    mma_commit_pair_both(smem_u32(&s.empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                mma_commit_pair_both(smem_u32(&s.tfull[acc]));
                if (++acc == NACC) { acc = 0; acc_phase ^= 1; }
            }
        }
    } else {
        // epilogue: TMEM lane quadrant q holds this CTA's tokens 32q..32q+31
        pdl_wait_previous();   // outputs may still be read by the previous kernel
        const int q = warp & 3;
        const uint32_t tempty0 = cluster_addr(smem_u32(&s.tempty[0]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = pair; u < units; u += npairs) {
            int mt, nt;
            wide_tile(u, MT, NT, mt, nt);
            if (!mbar_wait(smem_u32(&s.tfull[acc]), acc_phase, s.abort)) break;
            tc_fence_after();
#pragma unroll 1
            for (int j = 0; j < NB; ++j)
                if (nt * NB + j < a.rows_w)
                    wide_epilogue_half(a, mt * 256 + (int)rank * 128 + q * 32 + lane, nt * NB + j,
                                       tmem_base + (acc * NB + j) * 256 + ((uint32_t)(q * 32) << 16));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(tempty0 + 8u * acc);
            if (++acc == NACC) { acc = 0; acc_phase ^= 1; }
        }
    }
done:
    pair_teardown(s, tmem_base, rank, a.status);
}

// ================== skinny tiling: 256 weight rows x BT tokens, stream-K ==================

// Final epilogue of a skinny tile for 16 tokens t0..t0+15: v0 = rows r, v1 = rows 128 + r.
__device__ __forceinline__ void skinny_final16(const TcArgs &a, int tile, int r, int t0, const float (&v0)[16],
                                               const float (&v1)[16]) {
    const int T = a.rows_x;
    if (a.epi == EPI_PART) {
        const int ot = w_tile(a, tile);
        const int n0 = tile_col(a, ot, r, 256), n1 = tile_col(a, ot, r + 128, 256);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (t0 + i >= T) break;
            float *row = part_row(a, tile, t0 + i);
            if (n0 >= 0) row[n0] = v0[i];
            if (n1 >= 0) row[n1] = v1[i];
        }
        return;
    }
    if (a.epi == EPI_H_SWIGLU) {
        const int n = tile_col(a, tile, r, 128);
        if (n < 0) return;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (t0 + i < T) a.out[(long)(t0 + i) * a.ldo + n] = __float2bfloat16_rn(silu_fast(v0[i]) * v1[i]);
    } else {
        const int n0 = tile_col(a, tile, r, 256), n1 = tile_col(a, tile, r + 128, 256);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (t0 + i >= T) break;
            if (n0 >= 0) a.out[(long)(t0 + i) * a.ldo + n0] = __float2bfloat16_rn(act_out(a.epi, v0[i]));
            if (n1 >= 0) a.out[(long)(t0 + i) * a.ldo + n1] = __float2bfloat16_rn(act_out(a.epi, v1[i]));
        }
    }
}

// Final epilogue of 4 tokens t0..t0+3: v0 = row r, v1 = row 128 + r.
__device__ __forceinline__ void skinny_final4(const TcArgs &a, int tile, int r, int t0, float4 v0, float4 v1) {
    const float g[4] = {v0.x, v0.y, v0.z, v0.w}, u[4] = {v1.x, v1.y, v1.z, v1.w};
    const int T = a.rows_x;
    if (a.epi == EPI_PART) {
        const int ot = w_tile(a, tile);
        const int n0 = tile_col(a, ot, r, 256), n1 = tile_col(a, ot, r + 128, 256);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (t0 + i >= T) break;
            float *row = part_row(a, tile, t0 + i);
            if (n0 >= 0) row[n0] = g[i];
            if (n1 >= 0) row[n1] = u[i];
        }
        return;
    }
    if (a.epi == EPI_H_SWIGLU) {
        const int n = tile_col(a, tile, r, 128);
        if (n < 0) return;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (t0 + i < T) a.out[(long)(t0 + i) * a.ldo + n] = __float2bfloat16_rn(silu_fast(g[i]) * u[i]);
    } else {
        const int n0 = tile_col(a, tile, r, 256), n1 = tile_col(a, tile, r + 128, 256);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (t0 + i >= T) break;
            if (n0 >= 0) a.out[(long)(t0 + i) * a.ldo + n0] = __float2bfloat16_rn(act_out(a.epi, g[i]));
            if (n1 >= 0) a.out[(long)(t0 + i) * a.ldo + n1] = __float2bfloat16_rn(act_out(a.epi, u[i]));
        }
    }
}

// Final epilogue of a 128-row tile (tanh / identity / output): 4 tokens of row r.
__device__ __forceinline__ void skinny_final_half4(const TcArgs &a, int tile, int r, int t0, float4 v) {
    const int n = tile_col(a, tile, r, 128);
    if (n < 0) return;
    const float g[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (t0 + i < a.rows_x) a.out[(long)(t0 + i) * a.ldo + n] = __float2bfloat16_rn(act_out(a.epi, g[i]));
}

// Whole 128-row tile: the epilogue warps stage the BT x 128 bf16 outputs (after
// the activation) in shared memory, one column per thread, then write them out
// as 16-byte pieces of 8 columns of one token -- a sixteenth of the stores of
// one 2-byte column per thread.  `so` holds BT rows of 128 columns.  Output
// widths are multiples of 8, so a piece is all real columns or all padding and
// is 16-byte aligned.  Runs on the 128 epilogue threads (named barrier 1).
__device__ __forceinline__ void skinny_store_staged(const TcArgs &a, int tile, int BT, const __nv_bfloat16 *so) {
    const int et = threadIdx.x - 64;                 // 0..127
    for (int c = et; c < BT * 16; c += 128) {
        const int t = c >> 4, j = c & 15;
        const int col = tile_col(a, tile, 8 * j, 128);
        if (t < a.rows_x && col >= 0)
            *reinterpret_cast<uint4 *>(a.out + (long)t * a.ldo + col) =
                *reinterpret_cast<const uint4 *>(so + t * 128 + 8 * j);
    }
}

// One-shot all-reduce of a 256-row tile across ranks (EPI_AR), run by the 128
// epilogue threads of CTA j of the tile's cluster once every CTA of the
// cluster has staged its partial sums ("7.4 推理侧并行" §7.4.2, optimisation
// 2: each rank sends its whole partial to every other rank and every rank
// adds them up itself, in one step).
//   1. For the token quads j, j + n, ... of the tile: add the cluster's slots
//      (this rank's Z_i for those tokens), round to bf16 and store them into
//      every rank's receive buffer (plain stores; over NVLink for a peer),
//      row block `me` of the buffer half chosen by the epoch's parity.
//   2. Fence at system scope, then publish: flag (me, tile, j) = epoch in
//      every rank's buffer.
//   3. Wait (bounded) until the same unit's flag from every rank has this
//      epoch in our own buffer, then add the ranks' rows in rank order (fp32)
//      and write the output.
// The epoch is kept on the device (graph replays need no new arguments): each
// rank's buffer holds the last finished epoch, every CTA reads it at its start
// and works on the next one, and the last CTA of the rank to finish stores it.
// Flags only grow (the epoch goes up by one per call), so nothing is reset;
// the two buffer halves keep a fast rank from overwriting rows a slow rank is
// still reading: a rank reaches epoch e + 2 only after seeing every rank's
// epoch e + 1 flags, which those ranks set after finishing epoch e.
template <int BT>
__device__ __forceinline__ void ar_exchange(const TcArgs &a, const Smem &s, int tile, unsigned epoch) {
    const int r = threadIdx.x - 64;
    const uint32_t n = (uint32_t)a.cluster_red, j = cluster_rank();
    const int li = tile / a.otiles, otile = tile - li * a.otiles, me = a.ar_rank0 + li;
    const int col0 = tile_col(a, otile, r, 256), col1 = tile_col(a, otile, r + 128, 256);
    const float4 *st4 = reinterpret_cast<const float4 *>(s.a);
    const int T = a.rows_x;
    for (int qd = (int)j; qd < BT / 4 && qd * 4 < T; qd += (int)n) {
        float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
        for (uint32_t src = 0; src < n; ++src) {
            const float4 g = ld_cluster_f4(st4 + qd * 256 + r, src);
            const float4 h = ld_cluster_f4(st4 + qd * 256 + 128 + r, src);
            s0.x += g.x; s0.y += g.y; s0.z += g.z; s0.w += g.w;
            s1.x += h.x; s1.y += h.y; s1.z += h.z; s1.w += h.w;
        }
        const float v0[4] = {s0.x, s0.y, s0.z, s0.w}, v1[4] = {s1.x, s1.y, s1.z, s1.w};
        if (a.sp_rows) {   // reduce-scatter: row t goes to its owner only, as the owner's row t - owner * sp_rows
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = qd * 4 + i;
                if (t >= T) break;
                const int owner = t / a.sp_rows;
                __nv_bfloat16 *row = ar_recv_row(a, epoch, owner, me, t - owner * a.sp_rows);
                if (col0 >= 0) row[col0] = __float2bfloat16_rn(v0[i]);
                if (col1 >= 0) row[col1] = __float2bfloat16_rn(v1[i]);
            }
            continue;
        }
        for (int p = 0; p < a.ar_ranks; ++p)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = qd * 4 + i;
                if (t >= T) break;
                __nv_bfloat16 *row = ar_recv_row(a, epoch, p, me, t);
                if (col0 >= 0) row[col0] = __float2bfloat16_rn(v0[i]);
                if (col1 >= 0) row[col1] = __float2bfloat16_rn(v1[i]);
            }
    }
    __threadfence_system();
    named_bar(1, 128);
    if (threadIdx.x == 64) {
        for (int p = 0; p < a.ar_ranks; ++p) st_release_sys(ar_flag(a, p, me, otile, (int)j), epoch);
        bool ok = true;
        const unsigned long long t0 = globaltimer();
        for (int src = 0; src < a.ar_ranks && ok; ++src) {
            const unsigned *f = ar_flag(a, me, src, otile, (int)j);
            while (ld_acquire_sys(f) != epoch) {
                if (globaltimer() - t0 > kWaitLimitNs) {
                    ok = false;
                    *s.abort = 1;
                    break;
                }
            }
        }
        *s.flag = ok ? 1 : 0;
    }
    named_bar(1, 128);
    if (!*s.flag) return;
    __threadfence();
    __nv_bfloat16 *out = a.outs[li];
    for (int qd = (int)j; qd < BT / 4 && qd * 4 < T; qd += (int)n)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int t = qd * 4 + i;
            if (t >= T) break;
            if (a.sp_rows) {   // reduce-scatter: only the rows this rank owns, as its local rows
                if (t / a.sp_rows != me) continue;
                t -= me * a.sp_rows;
            }
            float z0 = 0.f, z1 = 0.f;
            for (int src = 0; src < a.ar_ranks; ++src) {
                const unsigned short *row =
                    reinterpret_cast<const unsigned short *>(ar_recv_row(a, epoch, me, src, t));
                if (col0 >= 0) z0 += __bfloat162float(__ushort_as_bfloat16(__ldcg(row + col0)));
                if (col1 >= 0) z1 += __bfloat162float(__ushort_as_bfloat16(__ldcg(row + col1)));
            }
            if (col0 >= 0) out[(long)t * a.ldo + col0] = __float2bfloat16_rn(z0);
            if (col1 >= 0) out[(long)t * a.ldo + col1] = __float2bfloat16_rn(z1);
        }
}

// HALF: 128-row weight tiles, one M=128 MMA per 16-k step (never SwiGLU's first
// projection, whose gate and up rows must share a tile); split tiles always go
// to skinny_reduce_kernel.
template <int BT, int STAGES, bool RAW, bool HALF>
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_skinny_kernel(const __grid_constant__ WeightMaps wm, const __grid_constant__ CUtensorMap tmX, TcArgs a) {
    constexpr uint32_t W_BYTES = (HALF ? 128 : 256) * BK * 2;   // 256 weight rows: two M=128 halves
    constexpr uint32_t X_BYTES = BT * BK * 2;
    extern __shared__ uint8_t smem_raw[];
    const Smem s = carve<STAGES>(smem_raw, W_BYTES, X_BYTES);
    // HALF: BT x 128 bf16 output staging after the barrier block (16-byte aligned)
    __nv_bfloat16 *stage_out = reinterpret_cast<__nv_bfloat16 *>(
        (reinterpret_cast<uintptr_t>(s.tmem_slot) + 16 + 15) & ~uintptr_t(15));
    const uint32_t tmem_base = setup<STAGES>(s, &wm.map[0], &tmX);
    pdl_allow_dependents();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long total = a.total_iters, G = gridDim.x, c = blockIdx.x;
    const long long it_b = share_begin(c, total, G), it_e = share_begin(c + 1, total, G);
    const int KB = a.KB;
    constexpr int ROWS = HALF ? 128 : 256;   // rows of a weight tile; a partial slot is [token/4][ROWS][4]
    int cl_tile = -1;                         // cluster route: the tile this CTA staged in shared memory

    if (a.epi == EPI_AR && threadIdx.x == 0) {   // this call's epoch, read before any CTA of it finishes
        const int li = (int)(blockIdx.x / ((unsigned)a.cluster_red * a.otiles));
        s.tmem_slot[3] = *reinterpret_cast<volatile unsigned *>(ar_control(a, a.ar_rank0 + li)) + 1u;
    }
    if (warp == 0) {
        if (lane == 0) {
            // The weights do not depend on the previous kernel; X does.  Every
            // stage gets its weight block before the wait (each barrier expects
            // the weight and X bytes, so a stage completes only with both); then
            // the producer waits and adds the X boxes.  (Prefetching further
            // blocks into L2 here measured slower.)
            const int npre = (int)min((long long)STAGES, it_e - it_b);
            for (int i = 0; i < npre; ++i) {
                const long long it = it_b + i;
                const int tile = (int)(it / KB), kb = (int)(it - (long long)tile * KB);
                const uint32_t fb = smem_u32(&s.full[i]);
                mbar_arrive_expect_tx(fb, W_BYTES + X_BYTES);   // first use of stage i: it is empty
                load_w_tile<RAW, HALF>(smem_u32(s.a + i * W_BYTES), wm, w_tile(a, tile), k_block(a, tile, kb), KB,
                                       fb);
            }
            pdl_wait_previous();
            if (a.sp_wait) {
                // X is gathered from every rank: wait until every rank's rows have
                // arrived (bounded), then order those generic-proxy stores before
                // this thread's TMA reads of them.
                const unsigned need = (*reinterpret_cast<const volatile unsigned *>(a.sp_epoch) + 1u) * a.sp_per_src;
                const unsigned long long t0 = globaltimer();
                for (int src = 0; src < a.ar_ranks; ++src)
                    while (ld_acquire_sys(a.sp_wait + src) < need) {
                        if (globaltimer() - t0 > kWaitLimitNs) {
                            *s.abort = 1;
                            goto done;
                        }
                    }
                asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            for (int i = 0; i < npre; ++i) {
                const long long it = it_b + i;
                const int tile = (int)(it / KB), kb = (int)(it - (long long)tile * KB);
                tma_load_2d(smem_u32(s.b + i * X_BYTES), &tmX, k_block(a, tile, kb) * BK, 0, smem_u32(&s.full[i]));
            }
            int stage = npre % STAGES;
            uint32_t phase = npre == STAGES ? 1u : 0u;
            for (long long it = it_b + npre; it < it_e; ++it) {
                const int tile = (int)(it / KB), kb = (int)(it - (long long)tile * KB);
                if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1, s.abort)) goto done;
                const uint32_t fb = smem_u32(&s.full[stage]);
                mbar_arrive_expect_tx(fb, W_BYTES + X_BYTES);
                const int gkb = k_block(a, tile, kb);
                load_w_tile<RAW, HALF>(smem_u32(s.a + stage * W_BYTES), wm, w_tile(a, tile), gkb, KB, fb);
                tma_load_2d(smem_u32(s.b + stage * X_BYTES), &tmX, gkb * BK, 0, fb);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, BT) | (RAW ? kIdescAMajorMN : 0u);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (long long it = it_b; it < it_e;) {
                const int tile = (int)(it / KB);
                const int kb0 = (int)(it - (long long)tile * KB);
                const int kb1 = (int)min((long long)KB, it_e - (long long)tile * KB);
                if (!mbar_wait(smem_u32(&s.tempty[acc]), acc_phase ^ 1, s.abort)) goto done;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * (2 * BT), d1 = d0 + BT;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(smem_u32(&s.full[stage]), phase, s.abort)) goto done;
                    tc_fence_after();
                    const uint32_t wa = smem_u32(s.a + stage * W_BYTES);
                    // rows 128..255 of the tile: K-major 16 KB in; MN-major atoms 2-3, 16 KB in
                    const uint64_t dw0 = RAW ? smem_desc_mnmajor_sw128(wa) : smem_desc_kmajor_sw128(wa);
                    const uint64_t dw1 =
                        RAW ? smem_desc_mnmajor_sw128(wa + 16384) : smem_desc_kmajor_sw128(wa + 128 * 128);
                    constexpr uint32_t kstep_w = RAW ? 128 : 2;
                    const uint64_t dx = smem_desc_kmajor_sw128(smem_u32(s.b + stage * X_BYTES));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint32_t accum = (kb != kb0 || k != 0) ? 1u : 0u;
                        mma_bf16(d0, dw0 + kstep_w * k, dx + 2 * k, idesc, accum);
                        if (!HALF) mma_bf16(d1, dw1 + kstep_w * k, dx + 2 * k, idesc, accum);
                    }
                    mma_commit(smem_u32(&s.empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                mma_commit(smem_u32(&s.tfull[acc]));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
                it = (long long)tile * KB + kb1;
            }
        }
    } else {
        pdl_wait_previous();
        const int q = warp & 3;
        const int r = q * 32 + lane;   // row within each 128-row half
        int acc = 0;
        uint32_t acc_phase = 0;
        for (long long it = it_b; it < it_e;) {
            const int tile = (int)(it / KB);
            const int kb0 = (int)(it - (long long)tile * KB);
            const int kb1 = (int)min((long long)KB, it_e - (long long)tile * KB);
            it = (long long)tile * KB + kb1;
            // all 128 epilogue threads leave alike if the wait gave up in any
            if (named_bar_or(1, 128, !mbar_wait(smem_u32(&s.tfull[acc]), acc_phase, s.abort))) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + acc * (2 * BT) + ((uint32_t)(q * 32) << 16);
            // (the cluster route stages even a whole tile: the all-reduce needs it there)
            const bool whole = (kb0 == 0 && kb1 == KB) && !a.cluster_red;
            if (whole) {
#pragma unroll 1
                for (int t0 = 0; t0 < BT; t0 += 16) {
                    float v0[16], v1[16];
                    tmem_ld16(taddr + t0, v0);
                    if (!HALF) tmem_ld16(taddr + BT + t0, v1);
                    tmem_ld_wait();
                    if (HALF) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            stage_out[(t0 + i) * 128 + r] = __float2bfloat16_rn(act_out(a.epi, v0[i]));
                    } else {
                        skinny_final16(a, tile, r, t0, v0, v1);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&s.tempty[acc]));
                if (HALF) {
                    named_bar(1, 128);   // the whole tile is staged
                    skinny_store_staged(a, tile, BT, stage_out);
                    named_bar(1, 128);   // staging is free for the next tile
                }
            } else {
                // this CTA's share of the tile -> its partial slot, laid out
                // [token/4][row][token%4]: each lane stores float4s, a warp 512 B at a time
                const int c_first = share_owner((long long)tile * KB, total, G);
                const int c_last = share_owner((long long)tile * KB + KB - 1, total, G);
                const int slot = (int)c - c_first;
                // cluster route: the slot is this CTA's own ring (every MMA that read it is done)
                float4 *base = a.cluster_red
                                   ? reinterpret_cast<float4 *>(s.a)
                                   : reinterpret_cast<float4 *>(a.part + ((long long)tile * a.slots + slot) * ROWS * BT);
#pragma unroll 1
                for (int t0 = 0; t0 < BT; t0 += 16) {
                    float v0[16], v1[16];
                    tmem_ld16(taddr + t0, v0);
                    if (!HALF) tmem_ld16(taddr + BT + t0, v1);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int qd = t0 / 4 + q;
                        base[qd * ROWS + r] = make_float4(v0[4 * q], v0[4 * q + 1], v0[4 * q + 2], v0[4 * q + 3]);
                        if (!HALF)
                            base[qd * ROWS + 128 + r] =
                                make_float4(v1[4 * q], v1[4 * q + 1], v1[4 * q + 2], v1[4 * q + 3]);
                    }
                }
                // the accumulator is copied out: hand TMEM back to the MMA before the fixup
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&s.tempty[acc]));
                if (a.cluster_red) {   // added across the cluster at the exit
                    cl_tile = tile;
                    acc ^= 1;
                    if (acc == 0) acc_phase ^= 1;
                    continue;
                }
                if (HALF || a.split_mode == kSplitSeparate) {   // skinny_reduce_kernel adds the slots
                    acc ^= 1;
                    if (acc == 0) acc_phase ^= 1;
                    continue;
                }
                __threadfence();
                named_bar(1, 128);
                if (threadIdx.x == 64) {
                    const unsigned done_kb = atomicAdd(&a.tile_cnt[tile], (unsigned)(kb1 - kb0)) + (kb1 - kb0);
                    *s.flag = (done_kb == (unsigned)KB);
                }
                named_bar(1, 128);
                if (*s.flag) {
                    // Last to arrive: add the n slots in slot order.  Each thread walks
                    // whole float4 positions (row r, 4 tokens) so the loads of several
                    // positions and slots are in flight together.
                    __threadfence();
                    const float4 *tb = reinterpret_cast<const float4 *>(a.part + (long long)tile * a.slots * 256 * BT);
                    const int n = c_last - c_first + 1;
                    constexpr long SLOT4 = 256L * BT / 4;   // float4s per slot
                    constexpr int NPOS = (BT / 4) * 128;     // (token quad, row pair) positions
                    constexpr int U = 4;
#pragma unroll 1
                    for (int p0 = threadIdx.x - 64; p0 < NPOS; p0 += 128 * U) {
                        float4 s0[U], s1[U];
#pragma unroll
                        for (int u = 0; u < U; ++u) s0[u] = s1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                        for (int sl = 0; sl < n; ++sl) {
#pragma unroll
                            for (int u = 0; u < U; ++u) {
                                const int pos = p0 + u * 128;
                                if (pos < NPOS) {
                                    const long o = sl * SLOT4 + (long)(pos >> 7) * 256 + (pos & 127);
                                    const float4 g = __ldcg(tb + o), h = __ldcg(tb + o + 128);
                                    s0[u].x += g.x; s0[u].y += g.y; s0[u].z += g.z; s0[u].w += g.w;
                                    s1[u].x += h.x; s1[u].y += h.y; s1[u].z += h.z; s1[u].w += h.w;
                                }
                            }
                        }
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            const int pos = p0 + u * 128;
                            if (pos < NPOS) skinny_final4(a, tile, pos & 127, (pos >> 7) * 4, s0[u], s1[u]);
                        }
                    }
                    if (threadIdx.x == 64) a.tile_cnt[tile] = 0u;
                }
                named_bar(1, 128);   // the flag is reused by the next split tile
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    }
done:
    if (a.cluster_red) {
        // The n CTAs of a tile (one cluster; cluster rank = slot) have staged
        // their partial sums in their rings.  Every thread of every CTA passes
        // both barriers, whatever happened before.  CTA j then adds, for token
        // quads j, j + n, ..., the n slots in slot order -- the order of
        // skinny_reduce_kernel, so both routes give the same bits -- and
        // applies the epilogue; the second barrier keeps each ring alive until
        // the cluster has read it.
        __syncwarp();
        cluster_barrier();
        if constexpr (!HALF) {
            if (a.epi == EPI_AR) {
                // After the barrier nobody sets the abort flag any more, so `go`
                // is the same in every thread of the CTA (the named barriers
                // below need all 128 epilogue threads or none).
                const unsigned epoch = s.tmem_slot[3];
                const bool go = cl_tile >= 0 && !*s.abort;
                if (go && threadIdx.x >= 64) ar_exchange<BT>(a, s, cl_tile, epoch);
                cluster_barrier();
                if (threadIdx.x == 0) {   // the rank's last CTA to finish records the epoch as done
                    const int li = (int)(blockIdx.x / ((unsigned)a.cluster_red * a.otiles));
                    unsigned *ctl = ar_control(a, a.ar_rank0 + li);
                    __threadfence();
                    if (atomicAdd(ctl + 1, 1u) + 1u == (unsigned)a.cluster_red * a.otiles) {
                        ctl[1] = 0u;
                        if (a.sp_rows) ctl[2] += 1u;
                        __threadfence();
                        atomicExch(ctl, epoch);
                    }
                }
                goto exit;
            }
        }
        if (cl_tile >= 0 && threadIdx.x >= 64) {
            const int r = threadIdx.x - 64;
            const uint32_t n = (uint32_t)a.cluster_red, j = cluster_rank();
            const float4 *st4 = reinterpret_cast<const float4 *>(s.a);
            for (int qd = (int)j; qd < BT / 4 && qd * 4 < a.rows_x; qd += (int)n) {
                float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
                for (uint32_t src = 0; src < n; ++src) {
                    const float4 g = ld_cluster_f4(st4 + qd * ROWS + r, src);
                    s0.x += g.x; s0.y += g.y; s0.z += g.z; s0.w += g.w;
                    if (!HALF) {
                        const float4 h = ld_cluster_f4(st4 + qd * ROWS + 128 + r, src);
                        s1.x += h.x; s1.y += h.y; s1.z += h.z; s1.w += h.w;
                    }
                }
                if (HALF)
                    skinny_final_half4(a, cl_tile, r, qd * 4, s0);
                else
                    skinny_final4(a, cl_tile, r, qd * 4, s0, s1);
            }
        }
        cluster_barrier();
    }
exit:
    teardown(s, tmem_base, a.status);
}

// Split tiles of the skinny tiling finished by a kernel of their own: the
// last-arriver fixup above leaves one CTA to read every slot of a tile, which
// at 128 tokens is ~0.4-1.2 MB of latency-bound reads at the very end of the
// kernel.  Here one CTA of 128 threads takes one (tile, 4-token group), thread
// r adds rows r and 128 + r over the slots in slot order -- the fixup's order,
// so both routes give the same bits -- and applies the same epilogue.  Launched
// behind the skinny kernel with programmatic dependent launch; tiles one CTA
// finished whole are skipped.
// HALF: 128-row tiles, slots [token/4][128][4], one row per thread.
template <bool HALF>
__global__ void __launch_bounds__(128) skinny_reduce_kernel(TcArgs a, int BT) {
    pdl_allow_dependents();
    constexpr int ROWS = HALF ? 128 : 256;
    const int quads = BT / 4;
    const int units = a.rows_w * quads;   // rows_w: weight tiles
    const int r = threadIdx.x;
    const long long SLOT4 = (long long)ROWS / 4 * BT;   // float4s per slot (ROWS rows x BT tokens)
    bool waited = false;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int tile = u / quads, qd = u - tile * quads;
        const long long it0 = (long long)tile * a.KB;
        const int c_first = share_owner(it0, a.total_iters, a.grid);
        const int n = share_owner(it0 + a.KB - 1, a.total_iters, a.grid) - c_first + 1;
        if (n == 1 || qd * 4 >= a.rows_x) continue;
        if (!waited) {
            pdl_wait_previous();
            waited = true;
        }
        const float4 *p =
            reinterpret_cast<const float4 *>(a.part) + (long long)tile * a.slots * SLOT4 + qd * ROWS + r;
        float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
#pragma unroll 4
        for (int sl = 0; sl < n; ++sl) {
            const float4 g = __ldcg(p + sl * SLOT4);
            s0.x += g.x; s0.y += g.y; s0.z += g.z; s0.w += g.w;
            if (!HALF) {
                const float4 h = __ldcg(p + sl * SLOT4 + 128);
                s1.x += h.x; s1.y += h.y; s1.z += h.z; s1.w += h.w;
            }
        }
        if (HALF)
            skinny_final_half4(a, tile, r, qd * 4, s0);
        else
            skinny_final4(a, tile, r, qd * 4, s0, s1);
    }
}

// ===== fused skinny tiling: both projections in one persistent launch =====
// A skinny projection is a weight stream of 20-140 us.  Run as two kernels,
// the second projection's CTAs can start only when the first one's leave
// their SMs (each holds most of an SM's shared memory), refill their rings
// from nothing (~3.5 us before the first MMA at 16-128 tokens) and wait for a
// kernel that adds split tiles in between.  Here every CTA streams its share
// of the first projection's weights and then, in the same ring, its share of
// the second's: those blocks do not depend on H and arrive while the first
// projection's last tiles finish.  Only the X operand of the second
// projection (H) waits -- for a device counter that reaches the number of
// first-projection tiles once each tile's H is stored: a whole tile by its
// CTA, a split tile by the last of its CTAs to arrive, which adds the slots
// (in slot order, as skinny_reduce_kernel does).  Split tiles of the second
// projection go to skinny_reduce_kernel, launched behind: finished inside the
// kernel, by the last CTA of each tile, they left those few CTAs a long
// latency-bound tail (sweep, 128 tokens: 64.9 against 54.3 us); added by the
// whole grid after a grid-wide count, they kept every SM busy to the end,
// where the reduction kernel lets the next launch's CTAs start streaming
// (60.7 against 54.9 us).  Every
// CTA of the grid (one per SM at most) must be resident at once for the
// counter to be reached; the wait is bounded, so a grid that cannot be fails
// with a status instead of hanging.  The last CTA past the wait resets it.
struct FusedMaps {
    WeightMaps w1, w2;    // packed parts (map[0]) or the per-rank shards (RAW), as for the skinny kernel
    CUtensorMap x, h;     // X (T x d_in) and H (T x d_ff): boxes of BT rows x 64 k
    unsigned *h_done;     // first-projection tiles whose H is stored, this launch
    unsigned *exits;      // CTAs past their wait on h_done, this launch
    unsigned h_tiles;     // first-projection tiles
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Last CTA of a split tile: add its n slots in slot order (the order of
// skinny_reduce_kernel, so both routes give the same bits) and apply the
// epilogue.  Each thread walks whole float4 positions (row r, 4 tokens), U of
// them at a time, so the loads of several positions and slots are in flight
// together.  Runs on the 128 epilogue threads.
template <int BT, bool HALF>
__device__ __forceinline__ void fixup_tile(const TcArgs &a, int tile, int n) {
    constexpr int ROWS = HALF ? 128 : 256;
    constexpr long SLOT4 = (long)ROWS * BT / 4;   // float4s per slot
    constexpr int NPOS = (BT / 4) * 128;           // (token quad, row) positions
    constexpr int U = 4;
    const float4 *tb = reinterpret_cast<const float4 *>(a.part + (long long)tile * a.slots * ROWS * BT);
#pragma unroll 1
    for (int p0 = threadIdx.x - 64; p0 < NPOS; p0 += 128 * U) {
        float4 s0[U], s1[U];
#pragma unroll
        for (int u = 0; u < U; ++u) s0[u] = s1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
        for (int sl = 0; sl < n; ++sl) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int pos = p0 + u * 128;
                if (pos < NPOS) {
                    const long o = sl * SLOT4 + (long)(pos >> 7) * ROWS + (pos & 127);
                    const float4 g = __ldcg(tb + o);
                    s0[u].x += g.x; s0[u].y += g.y; s0[u].z += g.z; s0[u].w += g.w;
                    if (!HALF) {
                        const float4 h = __ldcg(tb + o + 128);
                        s1[u].x += h.x; s1[u].y += h.y; s1[u].z += h.z; s1[u].w += h.w;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int pos = p0 + u * 128;
            if (pos >= NPOS) continue;
            if (HALF)
                skinny_final_half4(a, tile, pos & 127, (pos >> 7) * 4, s0[u]);
            else
                skinny_final4(a, tile, pos & 127, (pos >> 7) * 4, s0[u], s1[u]);
        }
    }
}

// One unit of the fused kernel's epilogue (this CTA's k-blocks kb0..kb1 of
// weight tile `tile`), on the 128 epilogue threads.  h_done != nullptr: a
// first-projection unit, whose tile is counted once its H is final.
// stage_out: where a whole 128-row tile is staged for 16-byte stores, or
// nullptr (2-byte stores straight from the accumulator).  Returns false if a
// wait gave up.
template <int BT, bool HALF>
__device__ __forceinline__ bool fused_unit(const TcArgs &a, const Smem &s, __nv_bfloat16 *stage_out,
                                           uint32_t tmem_base, int tile, int kb0, int kb1, int &acc,
                                           uint32_t &acc_phase, int c, unsigned *h_done) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;
    const int r = q * 32 + lane;   // row within each 128-row half
    constexpr int ROWS = HALF ? 128 : 256;
    // all 128 threads leave alike if the wait gave up in any (the barriers below need all)
    if (named_bar_or(1, 128, !mbar_wait(smem_u32(&s.tfull[acc]), acc_phase, s.abort))) return false;
    tc_fence_after();
    const uint32_t taddr = tmem_base + acc * (2 * BT) + ((uint32_t)(q * 32) << 16);
    bool final_here = true;   // this CTA wrote the tile's final values
    if (kb0 == 0 && kb1 == a.KB) {
#pragma unroll 1
        for (int t0 = 0; t0 < BT; t0 += 16) {
            float v0[16], v1[16];
            tmem_ld16(taddr + t0, v0);
            if (!HALF) tmem_ld16(taddr + BT + t0, v1);
            tmem_ld_wait();
            if (HALF && stage_out) {
#pragma unroll
                for (int i = 0; i < 16; ++i) stage_out[(t0 + i) * 128 + r] = __float2bfloat16_rn(act_out(a.epi, v0[i]));
            } else if (HALF) {
                const int n = tile_col(a, tile, r, 128);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (n >= 0 && t0 + i < a.rows_x)
                        a.out[(long)(t0 + i) * a.ldo + n] = __float2bfloat16_rn(act_out(a.epi, v0[i]));
            } else {
                skinny_final16(a, tile, r, t0, v0, v1);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&s.tempty[acc]));
        if (HALF && stage_out) {
            named_bar(1, 128);   // the whole tile is staged
            skinny_store_staged(a, tile, BT, stage_out);
            // the staging area is a ring stage's X box, which TMA fills next
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
    } else {
        // this CTA's share of the tile -> its slot, [token/4][row][token%4]
        const long long it0 = (long long)tile * a.KB;
        const int c_first = share_owner(it0, a.total_iters, a.grid);
        float4 *base = reinterpret_cast<float4 *>(a.part + ((long long)tile * a.slots + (c - c_first)) * ROWS * BT);
#pragma unroll 1
        for (int t0 = 0; t0 < BT; t0 += 16) {
            float v0[16], v1[16];
            tmem_ld16(taddr + t0, v0);
            if (!HALF) tmem_ld16(taddr + BT + t0, v1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int qd = t0 / 4 + j;
                base[qd * ROWS + r] = make_float4(v0[4 * j], v0[4 * j + 1], v0[4 * j + 2], v0[4 * j + 3]);
                if (!HALF)
                    base[qd * ROWS + 128 + r] = make_float4(v1[4 * j], v1[4 * j + 1], v1[4 * j + 2], v1[4 * j + 3]);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&s.tempty[acc]));
        if (a.split_mode != kSplitInKernel) {
            final_here = false;   // skinny_reduce_kernel adds the slots
        } else {
            // the last CTA of the tile to arrive adds its n slots in slot order
            __threadfence();
            named_bar(1, 128);
            if (threadIdx.x == 64) {
                const unsigned done_kb = atomicAdd(&a.tile_cnt[tile], (unsigned)(kb1 - kb0)) + (kb1 - kb0);
                *s.flag = (done_kb == (unsigned)a.KB);
            }
            named_bar(1, 128);
            final_here = *s.flag != 0;
            if (final_here) {
                __threadfence();
                fixup_tile<BT, HALF>(a, tile, share_owner(it0 + a.KB - 1, a.total_iters, a.grid) - c_first + 1);
                if (threadIdx.x == 64) a.tile_cnt[tile] = 0u;
            }
        }
    }
    if (h_done) __threadfence();   // H of this tile before the count that publishes it
    named_bar(1, 128);             // staging and the flag are free for the next unit
    if (h_done && final_here && threadIdx.x == 64) atomicAdd(h_done, 1u);
    acc ^= 1;
    if (acc == 0) acc_phase ^= 1;
    return true;
}

// HALF: 128-row tiles in both projections (tanh / identity); otherwise 256.
// RAW: the shard form, per-rank tensors read MN-major (always 256-row tiles).
template <int BT, int STAGES, bool HALF, bool RAW>
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_fused_kernel(const __grid_constant__ FusedMaps m, const __grid_constant__ TcArgs a1,
                    const __grid_constant__ TcArgs a2) {
    constexpr uint32_t W_BYTES = (HALF ? 128 : 256) * BK * 2;
    constexpr uint32_t X_BYTES = BT * BK * 2;
    extern __shared__ uint8_t smem_raw[];
    const Smem s = carve<STAGES>(smem_raw, W_BYTES, X_BYTES);
    // A whole 128-row tile is staged for its stores in the ring's X boxes
    // (BT x 128 bf16 = two of them): only for the CTA's last first-projection
    // unit, after which no X box is read or filled until that unit's H is
    // published.  Other whole 128-row tiles are stored straight from TMEM.
    static_assert(STAGES >= 2, "staging needs two X boxes");
    __nv_bfloat16 *const stage_x = reinterpret_cast<__nv_bfloat16 *>(s.b);
    const uint32_t tmem_base = setup<STAGES>(s, &m.w1.map[0], &m.x);
    pdl_allow_dependents();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const long long b1 = share_begin(c, a1.total_iters, a1.grid), e1 = share_begin(c + 1, a1.total_iters, a1.grid);
    long long b2 = 0, e2 = 0;   // CTAs beyond the second projection's grid have no share of it
    if (c < a2.grid) {
        b2 = share_begin(c, a2.total_iters, a2.grid);
        e2 = share_begin(c + 1, a2.total_iters, a2.grid);
    }

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&m.w2.map[0]);
            tma_prefetch_desc(&m.h);
            // first projection: the weights of the first stages before the
            // wait on the previous kernel, then X
            const int npre = (int)min((long long)STAGES, e1 - b1);
            for (int i = 0; i < npre; ++i) {
                const long long it = b1 + i;
                const int tile = (int)(it / a1.KB), kb = (int)(it - (long long)tile * a1.KB);
                const uint32_t fb = smem_u32(&s.full[i]);
                mbar_arrive_expect_tx(fb, W_BYTES + X_BYTES);
                load_w_tile<RAW, HALF>(smem_u32(s.a + i * W_BYTES), m.w1, tile, kb, a1.KB, fb);
            }
            pdl_wait_previous();
            for (int i = 0; i < npre; ++i) {
                const long long it = b1 + i;
                const int kb = (int)(it - it / a1.KB * a1.KB);
                tma_load_2d(smem_u32(s.b + i * X_BYTES), &m.x, kb * BK, 0, smem_u32(&s.full[i]));
            }
            int stage = npre % STAGES;
            uint32_t phase = npre == STAGES ? 1u : 0u;
            for (long long it = b1 + npre; it < e1; ++it) {
                const int tile = (int)(it / a1.KB), kb = (int)(it - (long long)tile * a1.KB);
                if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1, s.abort)) goto done;
                const uint32_t fb = smem_u32(&s.full[stage]);
                mbar_arrive_expect_tx(fb, W_BYTES + X_BYTES);
                load_w_tile<RAW, HALF>(smem_u32(s.a + stage * W_BYTES), m.w1, tile, kb, a1.KB, fb);
                tma_load_2d(smem_u32(s.b + stage * X_BYTES), &m.x, kb * BK, 0, fb);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            // second projection: weights into the stages as they free up, H
            // once every first-projection tile has been stored
            const int npre2 = (int)min((long long)STAGES, e2 - b2);
            const int stage0 = stage;
            for (int i = 0; i < npre2; ++i) {
                const long long it = b2 + i;
                const int tile = (int)(it / a2.KB), kb = (int)(it - (long long)tile * a2.KB);
                if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1, s.abort)) goto done;
                const uint32_t fb = smem_u32(&s.full[stage]);
                mbar_arrive_expect_tx(fb, W_BYTES + X_BYTES);
                load_w_tile<RAW, HALF>(smem_u32(s.a + stage * W_BYTES), m.w2, tile, kb, a2.KB, fb);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            {
                // every CTA waits (also one without a share of the second
                // projection), so that the last to pass can reset both words
                const unsigned long long t0 = globaltimer();
                while (ld_acquire_gpu(m.h_done) < m.h_tiles) {
                    if (*s.abort) goto done;
                    if (globaltimer() - t0 > kWaitLimitNs) {
                        *s.abort = 1;
                        goto done;
                    }
                }
                if (atomicAdd(m.exits, 1u) == gridDim.x - 1) {   // every CTA is past the wait
                    atomicExch(m.h_done, 0u);
                    atomicExch(m.exits, 0u);
                }
            }
            if (npre2 > 0) {
                // H was written with generic stores: order them before this thread's TMA reads
                asm volatile("fence.proxy.async.global;" ::: "memory");
                int sx = stage0;
                for (int i = 0; i < npre2; ++i) {
                    const long long it = b2 + i;
                    const int kb = (int)(it - it / a2.KB * a2.KB);
                    tma_load_2d(smem_u32(s.b + sx * X_BYTES), &m.h, kb * BK, 0, smem_u32(&s.full[sx]));
                    if (++sx == STAGES) sx = 0;
                }
            }
            for (long long it = b2 + npre2; it < e2; ++it) {
                const int tile = (int)(it / a2.KB), kb = (int)(it - (long long)tile * a2.KB);
                if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1, s.abort)) goto done;
                const uint32_t fb = smem_u32(&s.full[stage]);
                mbar_arrive_expect_tx(fb, W_BYTES + X_BYTES);
                load_w_tile<RAW, HALF>(smem_u32(s.a + stage * W_BYTES), m.w2, tile, kb, a2.KB, fb);
                tma_load_2d(smem_u32(s.b + stage * X_BYTES), &m.h, kb * BK, 0, fb);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, BT) | (RAW ? kIdescAMajorMN : 0u);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int ph = 0; ph < 2; ++ph) {
                const int KB = ph ? a2.KB : a1.KB;
                const long long ie = ph ? e2 : e1;
                for (long long it = ph ? b2 : b1; it < ie;) {
                    const int tile = (int)(it / KB);
                    const int kb0 = (int)(it - (long long)tile * KB);
                    const int kb1 = (int)min((long long)KB, ie - (long long)tile * KB);
                    if (!mbar_wait(smem_u32(&s.tempty[acc]), acc_phase ^ 1, s.abort)) goto done;
                    tc_fence_after();
                    const uint32_t d0 = tmem_base + acc * (2 * BT), d1 = d0 + BT;
                    for (int kb = kb0; kb < kb1; ++kb) {
                        if (!mbar_wait(smem_u32(&s.full[stage]), phase, s.abort)) goto done;
                        tc_fence_after();
                        const uint32_t wa = smem_u32(s.a + stage * W_BYTES);
                        // rows 128..255 of the tile: K-major 16 KB in; MN-major atoms 2-3, 16 KB in
                        const uint64_t dw0 = RAW ? smem_desc_mnmajor_sw128(wa) : smem_desc_kmajor_sw128(wa);
                        const uint64_t dw1 =
                            RAW ? smem_desc_mnmajor_sw128(wa + 16384) : smem_desc_kmajor_sw128(wa + 128 * 128);
                        constexpr uint32_t kstep_w = RAW ? 128 : 2;
                        const uint64_t dx = smem_desc_kmajor_sw128(smem_u32(s.b + stage * X_BYTES));
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k) {
                            const uint32_t accum = (kb != kb0 || k != 0) ? 1u : 0u;
                            mma_bf16(d0, dw0 + kstep_w * k, dx + 2 * k, idesc, accum);
                            if (!HALF) mma_bf16(d1, dw1 + kstep_w * k, dx + 2 * k, idesc, accum);
                        }
                        mma_commit(smem_u32(&s.empty[stage]));
                        if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    }
                    mma_commit(smem_u32(&s.tfull[acc]));
                    acc ^= 1;
                    if (acc == 0) acc_phase ^= 1;
                    it = (long long)tile * KB + kb1;
                }
            }
        }
    } else {
        pdl_wait_previous();
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int ph = 0; ph < 2 && ok; ++ph) {
            const TcArgs &a = ph ? a2 : a1;
            const long long ie = ph ? e2 : e1;
            for (long long it = ph ? b2 : b1; it < ie && ok;) {
                const int tile = (int)(it / a.KB);
                const int kb0 = (int)(it - (long long)tile * a.KB);
                const int kb1 = (int)min((long long)a.KB, ie - (long long)tile * a.KB);
                it = (long long)tile * a.KB + kb1;
                ok = fused_unit<BT, HALF>(a, s, ph == 0 && it == ie ? stage_x : nullptr, tmem_base, tile, kb0, kb1,
                                          acc, acc_phase, c, ph ? nullptr : m.h_done);
            }
        }
    }
done:
    teardown(s, tmem_base, a1.status);
}

// ======================================= host side =======================================

typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                    CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

PFN_encodeTiled encode_fn() {
    static PFN_encodeTiled fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(p);
    }
    return fn;
}

// 2-D bf16 tensor (inner x rows, rows `row_bytes` apart), box = 64 (inner) x box_rows,
// 128-byte swizzle, out-of-range elements read as zero.
bool make_map2d(CUtensorMap *m, const void *base, long long inner, long long rows, long long row_bytes,
                int box_rows) {
    PFN_encodeTiled enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Activations: K-major rows x K, row stride K; box = 64 (K) x box_rows.
bool make_map(CUtensorMap *m, const void *base, int K, int rows, int box_rows) {
    return make_map2d(m, base, K, rows, (long long)K * 2, box_rows);
}

// One projection's weight operand and its tile geometry.
struct WeightOperand {
    WeightMaps wm;
    bool raw, half;
    int tiles, KB;
    int raw_first, tps, fs;
    int prank, otiles;   // per-rank partials: tiles = prank * otiles, KB = one rank's k-blocks
};

// Token-tile widths from which the skinny tiling uses 128-row weight tiles
// (packed layout) and whole CTAs per tile (below); both measured best from the
// narrowest width on (sweep at 16 / 64 / 128 tokens: 54.4 -> 49.9, 63.6 ->
// 52.9, 68.4 -> 58.0 us; decode batch 32: 226 -> 222.5 us).
#ifndef TPMLP_SKINNY_HALF_MIN_BT
#define TPMLP_SKINNY_HALF_MIN_BT 16
#endif
#ifndef TPMLP_SKINNY_ALIGN_MIN_BT
#define TPMLP_SKINNY_ALIGN_MIN_BT 16
#endif

// Weight tiles of projection `proj` (0 first, 1 second) in the packed layout or
// the shard form, of 256 rows or (half) 128 rows.
long long skinny_tiles(const Problem &p, int proj, bool raw, bool half) {
    if (proj == 1) return half ? (p.d_out + 127) / 128 : blk_tiles(p.d_out);
    if (!raw) {
        const long long rows = w1p_rows(p.d_ff, p.act);
        return half ? (rows + 127) / 128 : blk_tiles(rows);
    }
    const int per = (p.act == TP_MLP_ACT_SWIGLU || half) ? 128 : 256;
    return (long long)p.tp * ((p.fs + per - 1) / per);
}

// Packed part (tile-blocked): a 2-D view of rows of 64 bf16 (128 B); one box of
// 256 rows = one 32 KB (tile, k-block) block, or of 128 rows = half of one.
bool weight_packed(WeightOperand *w, const Problem &p, int proj, const void *base, bool half) {
    memset(w, 0, sizeof(*w));
    const long long rows_w = proj == 0 ? w1p_rows(p.d_ff, p.act) : p.d_out;
    const int K = proj == 0 ? p.d_in : p.d_ff;
    w->half = half;
    w->tiles = (int)skinny_tiles(p, proj, false, half);
    w->KB = (int)blk_kblocks(K);
    const long long rows = blk_tiles(rows_w) * w->KB * kTileRows;
    return make_map2d(&w->wm.map[0], base, kKBlock, rows, kKBlock * 2, half ? kTileRows / 2 : kTileRows);
}

// First projection straight from the shards A_i (d_in x lda row-major, lda = f_s
// or 2 f_s for [gate_i | up_i]): maps over each rank's f_s columns, boxes of
// 64 columns x 64 k rows.
bool weight_raw_first(WeightOperand *w, const Problem &p, const ShardPtrs &A, bool half) {
    memset(w, 0, sizeof(*w));
    const bool sw = p.act == TP_MLP_ACT_SWIGLU;
    const long long lda = sw ? 2LL * p.fs : p.fs;
    const int per = (sw || half) ? 128 : 256;
    w->raw = true;
    w->half = half;
    w->tps = (p.fs + per - 1) / per;
    w->tiles = (int)skinny_tiles(p, 0, true, half);
    w->KB = (int)blk_kblocks(p.d_in);
    w->raw_first = 1;
    w->fs = p.fs;
    w->wm.first = 1;
    w->wm.swiglu = sw;
    w->wm.tps = w->tps;
    for (int i = 0; i < p.tp; ++i) {
        const __nv_bfloat16 *a = static_cast<const __nv_bfloat16 *>(A.p[i]);
        if (!make_map2d(&w->wm.map[i], a, p.fs, p.d_in, lda * 2, BK)) return false;
        if (sw && !make_map2d(&w->wm.map[kMaxTp + i], a + p.fs, p.fs, p.d_in, lda * 2, BK)) return false;
    }
    return true;
}

// Second projection straight from the shards B_i (f_s x d_out row-major); the K
// loop runs over rank 0's rows, then rank 1's, ... (needs f_s % 64 == 0).
// per_rank: one weight tile per (rank, output tile), each with its rank's
// k-blocks only (the per-rank partials), tiles rank-major.
bool weight_raw_second(WeightOperand *w, const Problem &p, const ShardPtrs &B, bool half, bool per_rank = false) {
    memset(w, 0, sizeof(*w));
    w->raw = true;
    w->half = half;
    w->tiles = (int)skinny_tiles(p, 1, true, half);
    w->KB = p.d_ff / BK;
    if (per_rank) {
        w->prank = p.tp;
        w->otiles = w->tiles;
        w->tiles *= p.tp;
        w->KB = p.fs / BK;
    }
    w->wm.kbps = p.fs / BK;
    for (int i = 0; i < p.tp; ++i)
        if (!make_map2d(&w->wm.map[i], B.p[i], p.d_out, p.fs, (long long)p.d_out * 2, BK)) return false;
    return true;
}

int skinny_bt(int T) { return T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : 128; }

// Split tiles of whole-CTA grids can be added across a thread-block cluster
// (tp_mlp_splitk CLUSTER).  Measured on B200 it is 0.6-2 us slower per step
// than skinny_reduce_kernel for the forward (sweep 16-128 tokens, decode batch
// 32), so AUTO keeps the reduction kernel; the cross-GPU exchange needs the
// cluster (its units finish inside the kernel).

// Ring depth of the skinny kernel per token width: 128-row tiles (SKH) and
// 256-row tiles (SK).  Each stage holds one weight block and one X box, so the
// wider the token tile, the fewer stages fit in shared memory.  More is not
// better on a grid of every SM: with 148 CTAs of 6 x 36 KB in flight (decode,
// 32 tokens) HBM is oversubscribed and serves the SMs unevenly -- equal shares
// finished 102-142 us after the start -- while 4 stages (21 MB in flight over
// the GPU) finished in 121-135 us: 3 % off the step at 2-32 tokens.  Fewer
// than 4 lets two CTAs share an SM, which was far slower.
#ifndef TPMLP_SKH_S16
#define TPMLP_SKH_S16 8
#endif
#ifndef TPMLP_SKH_S32
#define TPMLP_SKH_S32 8
#endif
#ifndef TPMLP_SKH_S64
#define TPMLP_SKH_S64 8
#endif
#ifndef TPMLP_SKH_S128
#define TPMLP_SKH_S128 6
#endif
#ifndef TPMLP_SK_S16
#define TPMLP_SK_S16 4
#endif
#ifndef TPMLP_SK_S32
#define TPMLP_SK_S32 4
#endif
#ifndef TPMLP_SK_S64
#define TPMLP_SK_S64 4
#endif
#ifndef TPMLP_SK_S128
#define TPMLP_SK_S128 4
#endif

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
    return ensure_smem_attr(kern, bytes);
}

// Whether `clusters` clusters of `n` CTAs of this kernel (smem bytes each) can
// all be resident at once (the cluster route needs them in one wave).  The
// answer is cached per kernel, cluster size and device.
template <typename K>
bool clusters_fit(K kern, size_t smem, int n, int clusters) {
    struct Entry {
        const void *fn;
        int n, dev, max_active;
    };
    static Entry cache[64];
    static int cached = 0;
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const void *fn = reinterpret_cast<const void *>(kern);
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < cached; ++i)
            if (cache[i].fn == fn && cache[i].n == n && cache[i].dev == dev) return cache[i].max_active >= clusters;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n * clusters);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)n;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_active = 0;
    if (cudaOccupancyMaxActiveClusters(&max_active, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        max_active = 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (cached < 64) cache[cached++] = Entry{fn, n, dev, max_active};
    return max_active >= clusters;
}

template <int BT, int STAGES, bool RAW, bool HALF>
cudaError_t launch_skinny_kern(const WeightOperand &w, const CUtensorMap &mx, TcArgs a, int grid, cudaStream_t st,
                               int *cluster_used) {
    // HALF adds the epilogue's BT x 128 bf16 staging (+16 for its alignment)
    const size_t smem = smem_bytes<STAGES>((HALF ? 128 : 256) * BK * 2, BT * BK * 2) + (HALF ? BT * 256 + 16 : 0);
    auto kern = tc_skinny_kernel<BT, STAGES, RAW, HALF>;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    // the cluster route stages a (HALF ? 128 : 256) x BT fp32 slot in the ring
    static_assert((size_t)(HALF ? 128 : 256) * BT * 4 <= (size_t)STAGES * ((HALF ? 128 : 256) + BT) * BK * 2,
                  "ring too small to stage a split tile");
    const int n = a.cluster_red;
    if (n >= 2 && clusters_fit(kern, smem, n, grid / n)) {
        *cluster_used = n;
        return launch_pdl_cluster(kern, dim3(grid), dim3(NTHREADS), smem, st, (unsigned)n, w.wm, mx, a);
    }
    a.cluster_red = 0;
    *cluster_used = 0;
    return launch_pdl(kern, dim3(grid), dim3(NTHREADS), smem, st, w.wm, mx, a);
}

template <int BT, int STAGES, bool HALF>
cudaError_t launch_skinny_bt(const WeightOperand &w, const CUtensorMap &mx, const TcArgs &a, int grid,
                             cudaStream_t st, int *cluster_used) {
    if (w.raw) return launch_skinny_kern<BT, STAGES, true, HALF>(w, mx, a, grid, st, cluster_used);
    return launch_skinny_kern<BT, STAGES, false, HALF>(w, mx, a, grid, st, cluster_used);
}

// Auto: the reduction kernel.  On B200 it measured faster at every width (16 to
// 128 tokens: 4-42 % of the step), even where the last-arriver fixup reads only
// two 32 KB slots, because the fixup sits at the end of the GEMM's critical path.
int resolve_split(int mode) { return mode == kSplitAuto || mode == kSplitCluster ? kSplitSeparate : mode; }

// 128-row tiles: never for SwiGLU's first projection (gate and up share a
// tile), the in-kernel fixup (256-row slots only) or the shard form, whose
// 64-column boxes of row-major shards then fetch 256-byte row pieces (T = 128:
// 66.6 us with 256-row tiles, 74.1 with 128).
bool skinny_half(int proj, int act, int BT, int split_mode, bool raw) {
    if (raw || resolve_split(split_mode) == kSplitInKernel) return false;
    if (proj == 0 && act == TP_MLP_ACT_SWIGLU) return false;
    return BT >= TPMLP_SKINNY_HALF_MIN_BT;
}

// Grid of a skinny projection.  Normally every SM, the weight stream cut into
// equal shares (stream-K).  With fewer tiles than SMs and wide token tiles,
// whose split-tile slots are large, a whole number s of CTAs per tile instead:
// every CTA then stays inside one tile, each tile has exactly s slots, and with
// as many tiles as SMs (s = 1) nothing is split at all -- provided that keeps
// at least 80 % of the SMs busy.
int skinny_grid(int tiles, int KB, int BT, int num_sms) {
    if (BT >= TPMLP_SKINNY_ALIGN_MIN_BT && tiles <= num_sms) {
        const int s = std::min(num_sms / tiles, KB);
        if (s >= 1 && 5LL * tiles * s >= 4LL * num_sms) return tiles * s;
    }
    return num_sms;
}

StreamKGeom skinny_geom(int tiles, int KB, int BT, int num_sms) {
    return streamk_geom(tiles, KB, skinny_grid(tiles, KB, BT, num_sms));
}

// One projection with the skinny tiling; x: T x K activations.
// Gather wait of a sequence-parallel first projection (see TcArgs::sp_wait).
struct SpWait {
    const unsigned *counts, *epoch;
    unsigned per_src;
    int ranks;
};

cudaError_t run_skinny(const WeightOperand &w, const void *x, int T, int K, int epi, void *out, int out_cols,
                       float *part, unsigned *cnt, int *status, int num_sms, cudaStream_t st, int split_mode,
                       int *launches, int ldo = 0, const SpWait *spw = nullptr) {
    const int BT = skinny_bt(T);
    CUtensorMap mx;
    if (!make_map(&mx, x, K, T, BT)) return cudaErrorInvalidValue;
    const StreamKGeom g = skinny_geom(w.tiles, w.KB, BT, num_sms);
    TcArgs a{};
    a.rows_x = T;
    a.rows_w = w.tiles;
    a.K = K;
    a.KB = g.KB;
    a.epi = epi;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.ldo = ldo ? ldo : out_cols;
    a.out_cols = out_cols;
    a.total_iters = g.total;
    a.slots = g.slots;
    a.part = part;
    a.tile_cnt = cnt;
    a.split_mode = g.slots > 1 ? (w.half ? kSplitSeparate : resolve_split(split_mode)) : kSplitInKernel;
    a.grid = g.grid;
    a.status = status;
    a.raw_first = w.raw_first;
    a.tps = w.tps;
    a.fs = w.fs;
    a.prank = w.prank;
    a.otiles = w.otiles;
    if (spw) {
        a.sp_wait = spw->counts;
        a.sp_epoch = spw->epoch;
        a.sp_per_src = spw->per_src;
        a.ar_ranks = spw->ranks;
    }
    if (epi == EPI_PART) {
        a.pout = static_cast<float *>(out);
        a.out = nullptr;
        if (g.slots > 1) a.split_mode = kSplitSeparate;   // the counters cover whole-K tiles only
    }
    // A whole number n of CTAs per tile (2..8), each inside one tile: the n
    // CTAs of a tile become one cluster and add their partials through
    // distributed shared memory, if all the clusters fit on the GPU at once.
    const int per_tile = g.grid / g.tiles;
    if (split_mode == kSplitCluster && g.slots > 1 && g.grid % g.tiles == 0 && per_tile >= 2 && per_tile <= 8)
        a.cluster_red = per_tile;
    int cl = 0;
    cudaError_t e;
    // a 128-row tile stage holds half the weights, so the ring gets more stages
    if (w.half) {
        switch (BT) {
            case 16: e = launch_skinny_bt<16, TPMLP_SKH_S16, true>(w, mx, a, g.grid, st, &cl); break;
            case 32: e = launch_skinny_bt<32, TPMLP_SKH_S32, true>(w, mx, a, g.grid, st, &cl); break;
            case 64: e = launch_skinny_bt<64, TPMLP_SKH_S64, true>(w, mx, a, g.grid, st, &cl); break;
            default: e = launch_skinny_bt<128, TPMLP_SKH_S128, true>(w, mx, a, g.grid, st, &cl); break;
        }
    } else {
        switch (BT) {
            case 16: e = launch_skinny_bt<16, TPMLP_SK_S16, false>(w, mx, a, g.grid, st, &cl); break;
            case 32: e = launch_skinny_bt<32, TPMLP_SK_S32, false>(w, mx, a, g.grid, st, &cl); break;
            case 64: e = launch_skinny_bt<64, TPMLP_SK_S64, false>(w, mx, a, g.grid, st, &cl); break;
            default: e = launch_skinny_bt<128, TPMLP_SK_S128, false>(w, mx, a, g.grid, st, &cl); break;
        }
    }
    ++*launches;
    if (e != cudaSuccess || cl || a.split_mode != kSplitSeparate) return e;
    ++*launches;
    // one CTA per unit: a grid capped at 2 CTAs per SM (so the next GEMM's CTAs
    // fit beside the waiting ones) measured 20-30 % slower at 32-128 tokens
    const dim3 rgrid(g.tiles * (BT / 4));
    return w.half ? launch_pdl(skinny_reduce_kernel<true>, rgrid, dim3(128), 0, st, a, BT)
                  : launch_pdl(skinny_reduce_kernel<false>, rgrid, dim3(128), 0, st, a, BT);
}

template <int MH>
cudaError_t run_wide(const WeightOperand &w, const void *x, int T, int K, int epi, void *out, int out_cols,
                     int *status, int num_sms, cudaStream_t st) {
    using C = WideCfg<MH>;
    CUtensorMap mx;
    if (!make_map(&mx, x, K, T, 128 * MH)) return cudaErrorInvalidValue;
    TcArgs a{};
    a.rows_x = T;
    a.rows_w = w.tiles;
    a.K = K;
    a.KB = w.KB;
    a.epi = epi;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.ldo = out_cols;
    a.out_cols = out_cols;
    a.status = status;
    a.raw_first = w.raw_first;
    a.tps = w.tps;
    a.fs = w.fs;
    a.prank = w.prank;
    a.otiles = w.otiles;
    if (epi == EPI_PART) {
        a.pout = static_cast<float *>(out);
        a.out = nullptr;
    }
    const int units = ((T + 128 * MH - 1) / (128 * MH)) * w.tiles;
    const int grid = std::min(units, num_sms);
    const size_t smem = smem_bytes<C::STAGES>(C::A_BYTES, C::B_BYTES);
    if (w.raw) {
        auto kern = tc_wide_kernel<MH, true>;
        cudaError_t e = set_smem(kern, smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, dim3(grid), dim3(NTHREADS), smem, st, mx, w.wm, a);
    }
    auto kern = tc_wide_kernel<MH, false>;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(grid), dim3(NTHREADS), smem, st, mx, w.wm, a);
}

// The pair tiling (packed weights): clusters of 2 CTAs, one 256 x 256 tile per
// pair at a time, persistent over the tiles.
template <int NB>
cudaError_t run_pair(const Problem &p, int proj, const void *wbase, const void *x, int T, int K, int epi,
                     void *out, int out_cols, int *status, int num_sms, cudaStream_t st) {
    WeightOperand w;
    if (!weight_packed(&w, p, proj, wbase, true)) return cudaErrorInvalidValue;   // 128-row boxes
    const long long rows_w = proj == 0 ? w1p_rows(p.d_ff, p.act) : p.d_out;
    CUtensorMap mx;
    if (!make_map(&mx, x, K, T, 128)) return cudaErrorInvalidValue;
    TcArgs a{};
    a.rows_x = T;
    a.rows_w = (int)blk_tiles(rows_w);
    a.K = K;
    a.KB = w.KB;
    a.epi = epi;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.ldo = out_cols;
    a.out_cols = out_cols;
    a.status = status;
    const int units = ((T + 255) / 256) * ((a.rows_w + NB - 1) / NB);
    const int pairs = std::max(1, std::min(units, num_sms / 2));
    constexpr int S = NB == 1 ? kPairStages : kPair2Stages;
    const size_t smem = smem_bytes<S>(128 * BK * 2, NB * 128 * BK * 2);
    auto kern = tc_pair_kernel<S, NB>;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl_cluster(kern, dim3(2 * pairs), dim3(NTHREADS), smem, st, 2u, mx, w.wm, a);
}

// Weight tiles per pair unit for one projection of the pair tiling: two
// (tc_pair_kernel<NB = 2>: each X stage feeds two 256-row tiles, a third less
// operand traffic per FLOP) unless the units then fill the pairs' waves worse:
// wave efficiency units / (waves x pairs) at least that of one tile per unit,
// less 2 %.  Sweep d 4096 / f 16384, tp 8: 2100 / 4096 tokens 400 / 857 us
// against 409 / 873 with one tile per unit (4096: 0.4 s windows); equal at
// 512-1024 tokens, where the rule keeps one tile for the second projection
// (two-tile units would leave 42 of 74 pairs idle: 171 against 117 us).
#ifndef TPMLP_PAIR_AUTO_NB
#define TPMLP_PAIR_AUTO_NB 1
#endif
int pair_tiles_per_unit(const Problem &p, int proj, int num_sms) {
    if (!TPMLP_PAIR_AUTO_NB) return 1;
    const long long MT = (p.T + 255) / 256;
    const long long tiles = blk_tiles(proj == 0 ? w1p_rows(p.d_ff, p.act) : p.d_out);
    const long long pairs = std::max(1, num_sms / 2);
    auto eff = [&](long long units) { return (double)units / (double)(((units + pairs - 1) / pairs) * pairs); };
    return eff(MT * ((tiles + 1) / 2)) >= eff(MT * tiles) - 0.02 ? 2 : 1;
}

int first_epi(int act) {
    return act == TP_MLP_ACT_SWIGLU ? EPI_H_SWIGLU : act == TP_MLP_ACT_TANH ? EPI_H_TANH : EPI_H_IDENT;
}

// Ring depth of the fused kernel: the skinny kernel's, except at 128 tokens,
// where the fused kernel's epilogue staging leaves room for a seventh stage
// (sweep d 4096 / f 16384, 128 tokens: 54.5 against 54.9 us with six).  More
// stages at 16-64 tokens measured no faster (8 -> 10-11 at 16 and 32, 8 -> 9
// at 64), and deeper 256-row rings slower (decode, 2-32 tokens: +9-12 us).
#ifndef TPMLP_FZH_S16
#define TPMLP_FZH_S16 TPMLP_SKH_S16
#endif
#ifndef TPMLP_FZH_S32
#define TPMLP_FZH_S32 TPMLP_SKH_S32
#endif
#ifndef TPMLP_FZH_S64
#define TPMLP_FZH_S64 TPMLP_SKH_S64
#endif
#ifndef TPMLP_FZH_S128
#define TPMLP_FZH_S128 7
#endif
#ifndef TPMLP_FZ_S16
#define TPMLP_FZ_S16 TPMLP_SK_S16
#endif
#ifndef TPMLP_FZ_S32
#define TPMLP_FZ_S32 TPMLP_SK_S32
#endif
#ifndef TPMLP_FZ_S64
#define TPMLP_FZ_S64 TPMLP_SK_S64
#endif
#ifndef TPMLP_FZ_S128
#define TPMLP_FZ_S128 TPMLP_SK_S128
#endif

// Fused skinny tiling: one grid for both projections, the first projection's
// (skinny_grid); the second is split evenly over the same CTAs.
struct FusedGeom {
    StreamKGeom g1, g2;
};
FusedGeom fused_geom(const Problem &p, bool half, bool raw, int num_sms) {
    const int BT = skinny_bt(p.T);
    FusedGeom f;
    f.g1 = skinny_geom((int)skinny_tiles(p, 0, raw, half), (int)blk_kblocks(p.d_in), BT, num_sms);
    f.g2 = streamk_geom(skinny_tiles(p, 1, raw, half), blk_kblocks(p.d_ff), f.g1.grid);
    return f;
}
// 128-row tiles for tanh / identity when no first-projection tile is split
// (a split 128-row tile has no in-kernel finish); 256 otherwise, and always for
// SwiGLU (gate and up share a tile).
bool fused_half(const Problem &p, int num_sms) {
    return p.act != TP_MLP_ACT_SWIGLU && skinny_bt(p.T) >= TPMLP_SKINNY_HALF_MIN_BT &&
           fused_geom(p, true, false, num_sms).g1.slots == 1;
}

// raw: the shard form (256-row tiles, f_s % 64 == 0, as for the skinny kernel).
bool fused_ok(const Problem &p, bool raw) {
    return (raw ? tc_raw_supported(p) : tc_supported(p)) && p.T >= 1 && p.T <= kTcSkinnyMaxTokens;
}

template <int BT, int STAGES, bool HALF, bool RAW = false>
cudaError_t launch_fused_kern(const FusedMaps &m, const TcArgs &a1, const TcArgs &a2, cudaStream_t st) {
    const size_t smem = smem_bytes<STAGES>((HALF ? 128 : 256) * BK * 2, BT * BK * 2);
    auto kern = tc_fused_kernel<BT, STAGES, HALF, RAW>;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(a1.grid), dim3(NTHREADS), smem, st, m, a1, a2);
}

// Both projections of the skinny tiling in one launch (packed weights, or the
// per-rank shards when rawA / rawB are given), then skinny_reduce_kernel for
// the second projection's split tiles.  Marks: 0 before, 1 after the fused
// kernel, 2 after the reduction.
cudaError_t run_fused(const Problem &p, const void *x, const void *w1p, const void *w2p, const ShardPtrs *rawA,
                      const ShardPtrs *rawB, void *h, void *out, float *part, unsigned *counters, int *status,
                      int num_sms, cudaStream_t st, const Marks &marks, int *launches) {
    *launches = 0;
    const bool raw = rawA != nullptr;
    if (!fused_ok(p, raw)) return cudaErrorNotSupported;
    const int BT = skinny_bt(p.T);
    const bool half = !raw && fused_half(p, num_sms);
    const FusedGeom f = fused_geom(p, half, raw, num_sms);
    WeightOperand w1, w2;
    if (raw) {
        if (!weight_raw_first(&w1, p, *rawA, false) || !weight_raw_second(&w2, p, *rawB, false, false))
            return cudaErrorInvalidValue;
    } else if (!weight_packed(&w1, p, 0, w1p, half) || !weight_packed(&w2, p, 1, w2p, half)) {
        return cudaErrorInvalidValue;
    }
    if (w1.tiles != f.g1.tiles || w1.KB != f.g1.KB || w2.tiles != f.g2.tiles || w2.KB != f.g2.KB)
        return cudaErrorInvalidValue;   // the operands' tiling must be the geometry's
    FusedMaps m;
    memset(&m, 0, sizeof(m));
    m.w1 = w1.wm;
    m.w2 = w2.wm;
    if (!make_map(&m.x, x, p.d_in, p.T, BT) || !make_map(&m.h, h, p.d_ff, p.T, BT)) return cudaErrorInvalidValue;
    m.h_done = counters + fused_counter_offset(p);
    m.exits = m.h_done + 1;
    m.h_tiles = (unsigned)f.g1.tiles;
    TcArgs a1{}, a2{};
    for (TcArgs *a : {&a1, &a2}) {
        a->rows_x = p.T;
        a->part = part;
        a->status = status;
    }
    a1.rows_w = f.g1.tiles;
    a1.K = p.d_in;
    a1.KB = f.g1.KB;
    a1.raw_first = w1.raw_first;   // the shard form's tiles map to features per rank
    a1.tps = w1.tps;
    a1.fs = w1.fs;
    a1.epi = first_epi(p.act);
    a1.out = static_cast<__nv_bfloat16 *>(h);
    a1.ldo = a1.out_cols = p.d_ff;
    a1.total_iters = f.g1.total;
    a1.slots = f.g1.slots;
    a1.tile_cnt = counters;
    a1.split_mode = kSplitInKernel;
    a1.grid = f.g1.grid;
    a2.rows_w = f.g2.tiles;
    a2.K = p.d_ff;
    a2.KB = f.g2.KB;
    a2.epi = EPI_OUT;
    a2.out = static_cast<__nv_bfloat16 *>(out);
    a2.ldo = a2.out_cols = p.d_out;
    a2.total_iters = f.g2.total;
    a2.slots = f.g2.slots;
    a2.split_mode = kSplitSeparate;
    a2.grid = f.g2.grid;
    marks.mark(0, st);
    cudaError_t e;
    if (raw) {
        switch (BT) {
            case 16: e = launch_fused_kern<16, TPMLP_FZ_S16, false, true>(m, a1, a2, st); break;
            case 32: e = launch_fused_kern<32, TPMLP_FZ_S32, false, true>(m, a1, a2, st); break;
            case 64: e = launch_fused_kern<64, TPMLP_FZ_S64, false, true>(m, a1, a2, st); break;
            default: e = launch_fused_kern<128, TPMLP_FZ_S128, false, true>(m, a1, a2, st); break;
        }
    } else if (half) {
        switch (BT) {
            case 16: e = launch_fused_kern<16, TPMLP_FZH_S16, true>(m, a1, a2, st); break;
            case 32: e = launch_fused_kern<32, TPMLP_FZH_S32, true>(m, a1, a2, st); break;
            case 64: e = launch_fused_kern<64, TPMLP_FZH_S64, true>(m, a1, a2, st); break;
            default: e = launch_fused_kern<128, TPMLP_FZH_S128, true>(m, a1, a2, st); break;
        }
    } else {
        switch (BT) {
            case 16: e = launch_fused_kern<16, TPMLP_FZ_S16, false>(m, a1, a2, st); break;
            case 32: e = launch_fused_kern<32, TPMLP_FZ_S32, false>(m, a1, a2, st); break;
            case 64: e = launch_fused_kern<64, TPMLP_FZ_S64, false>(m, a1, a2, st); break;
            default: e = launch_fused_kern<128, TPMLP_FZ_S128, false>(m, a1, a2, st); break;
        }
    }
    if (e != cudaSuccess) return e;
    ++*launches;
    marks.mark(1, st);
    if (f.g2.slots > 1) {
        const dim3 rgrid(f.g2.tiles * (BT / 4));
        e = half ? launch_pdl(skinny_reduce_kernel<true>, rgrid, dim3(128), 0, st, a2, BT)
                 : launch_pdl(skinny_reduce_kernel<false>, rgrid, dim3(128), 0, st, a2, BT);
        if (e == cudaSuccess) ++*launches;
    }
    marks.mark(2, st);
    return e;
}

// Launch with thread-block clusters and without programmatic overlap.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                           unsigned cluster, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The second projection of the local ranks fused with the one-shot all-reduce:
// n CTAs per tile (the largest n <= 8 whose clusters all fit on the GPU at
// once -- every CTA must be resident, since units wait on other ranks).
template <int BT, int STAGES>
cudaError_t launch_ar_bt(const WeightOperand &w, const CUtensorMap &mx, TcArgs a, int num_sms, cudaStream_t st) {
    const size_t smem = smem_bytes<STAGES>(256 * BK * 2, BT * BK * 2);
    auto kern = tc_skinny_kernel<BT, STAGES, true, false>;
    cudaError_t e = set_smem(kern, smem);
    if (e != cudaSuccess) return e;
    for (int n = std::min({8, num_sms / std::max(1, w.tiles), w.KB}); n >= 1; --n) {
        if (!clusters_fit(kern, smem, n, w.tiles)) continue;
        const int grid = w.tiles * n;
        a.grid = grid;
        a.slots = n;
        a.cluster_red = n;
        return launch_cluster(kern, dim3(grid), dim3(NTHREADS), smem, st, (unsigned)n, w.wm, mx, a);
    }
    return cudaErrorNotSupported;
}

// All-gather of the ranks' token rows (sequence parallelism): CTA (c, i) of
// local rank src = rank0 + i copies its share of x_i (rows x d bf16) into
// every rank's gather buffer at rows [src * rows, (src + 1) * rows), then
// counts itself in at every rank (release at system scope: a rank that sees
// the count also sees the rows).  Nothing here waits.
struct GatherArgs {
    const uint4 *x[kMaxTp];
    uint8_t *comm[kMaxTp];
    size_t gather_off;
    int rank0, ranks, rows, d;
};

__global__ void __launch_bounds__(256) sp_gather_kernel(GatherArgs g) {
    const int li = blockIdx.y, src = g.rank0 + li;
    const long long n16 = (long long)g.rows * g.d / 8;   // 16-byte pieces of one rank's rows
    const long long per = (n16 + gridDim.x - 1) / gridDim.x;
    const long long b = (long long)blockIdx.x * per, e = min(n16, b + per);
    const uint4 *x = g.x[li];
    for (int p = 0; p < g.ranks; ++p) {
        uint4 *dst = reinterpret_cast<uint4 *>(g.comm[p] + g.gather_off) + (long long)src * n16;
        for (long long k = b + threadIdx.x; k < e; k += blockDim.x) dst[k] = x[k];
    }
    __threadfence_system();
    __syncthreads();
    if (threadIdx.x == 0)
        for (int p = 0; p < g.ranks; ++p)
            asm volatile("red.release.sys.global.add.u32 [%0], 1;" ::"l"(reinterpret_cast<unsigned *>(g.comm[p]) + 8 + src)
                         : "memory");
}

constexpr int kGatherCtas = 16;   // per local rank

}  // namespace

cudaError_t launch_xgpu_sp(const Problem &p, int rank0, int nranks, const void *const *x_local, const ShardPtrs &A,
                           const ShardPtrs &B, void *h, float *part, unsigned *counters, int *status, int num_sms,
                           cudaStream_t st, const XgpuArgs &xa, size_t gather_off, int *launches) {
    *launches = 0;
    if (p.T < 1 || p.T > kTcSkinnyMaxTokens || p.T % p.tp || nranks < 1 || rank0 < 0 || rank0 + nranks > p.tp)
        return cudaErrorInvalidValue;
    const int rows = p.T / p.tp;
    // 1. all-gather of the token rows (no programmatic overlap: it must start
    //    after the previous call's exchange has finished and counted its epoch)
    GatherArgs g{};
    for (int i = 0; i < nranks; ++i) g.x[i] = static_cast<const uint4 *>(x_local[i]);
    for (int r = 0; r < p.tp; ++r) g.comm[r] = static_cast<uint8_t *>(xa.comm[r]);
    g.gather_off = gather_off;
    g.rank0 = rank0;
    g.ranks = p.tp;
    g.rows = rows;
    g.d = p.d_in;
    sp_gather_kernel<<<dim3(kGatherCtas, nranks), 256, 0, st>>>(g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
    // 2. each local rank's first projection on its gathered X, into its columns of H
    Problem p1 = p;
    p1.tp = 1;
    p1.d_ff = p.fs;
    const int ldh = nranks * p.fs;
    for (int i = 0; i < nranks; ++i) {
        ShardPtrs a1;
        memset(&a1, 0, sizeof(a1));
        a1.p[0] = A.p[i];
        WeightOperand w1;
        if (!weight_raw_first(&w1, p1, a1, false)) return cudaErrorInvalidValue;
        const unsigned *ctl = static_cast<const unsigned *>(xa.comm[rank0 + i]);
        const SpWait spw{ctl + 8, ctl + 2, (unsigned)kGatherCtas, p.tp};
        int n = 0;
        e = run_skinny(w1, static_cast<const uint8_t *>(xa.comm[rank0 + i]) + gather_off, p.T, p.d_in,
                       first_epi(p.act), static_cast<__nv_bfloat16 *>(h) + (size_t)i * p.fs, p.fs, part, counters,
                       status, num_sms, st, kSplitAuto, &n, ldh, &spw);
        *launches += n;
        if (e != cudaSuccess) return e;
    }
    // 3. second projection + reduce-scatter
    Problem pl = p;
    pl.tp = nranks;
    pl.d_ff = ldh;
    WeightOperand w2;
    if (!weight_raw_second(&w2, pl, B, false, true)) return cudaErrorInvalidValue;
    const int BT = skinny_bt(p.T);
    CUtensorMap mx;
    if (!make_map(&mx, h, ldh, p.T, BT)) return cudaErrorInvalidValue;
    TcArgs a{};
    a.rows_x = p.T;
    a.rows_w = w2.tiles;
    a.K = ldh;
    a.KB = w2.KB;
    a.epi = EPI_AR;
    a.ldo = p.d_out;
    a.out_cols = p.d_out;
    a.total_iters = (long long)w2.tiles * w2.KB;
    a.split_mode = kSplitSeparate;
    a.status = status;
    a.prank = w2.prank;
    a.otiles = w2.otiles;
    a.ar_rank0 = rank0;
    a.ar_ranks = p.tp;
    a.ar_rows = xa.rows;
    a.recv_off = xa.recv_off;
    a.sp_rows = rows;
    for (int r = 0; r < p.tp; ++r) a.comm[r] = static_cast<uint8_t *>(xa.comm[r]);
    for (int i = 0; i < nranks; ++i) a.outs[i] = static_cast<__nv_bfloat16 *>(xa.outs[i]);
    switch (BT) {
        case 16: e = launch_ar_bt<16, TPMLP_SK_S16>(w2, mx, a, num_sms, st); break;
        case 32: e = launch_ar_bt<32, TPMLP_SK_S32>(w2, mx, a, num_sms, st); break;
        case 64: e = launch_ar_bt<64, TPMLP_SK_S64>(w2, mx, a, num_sms, st); break;
        default: e = launch_ar_bt<128, TPMLP_SK_S128>(w2, mx, a, num_sms, st); break;
    }
    if (e == cudaSuccess) ++*launches;
    return e;
}

cudaError_t launch_xgpu(const Problem &p, int rank0, int nranks, const void *x, const ShardPtrs &A,
                        const ShardPtrs &B, void *h, float *part, unsigned *counters, int *status, int num_sms,
                        cudaStream_t st, const XgpuArgs &xa, int *launches) {
    *launches = 0;
    if (p.T < 1 || p.T > kTcSkinnyMaxTokens || nranks < 1 || rank0 < 0 || rank0 + nranks > p.tp)
        return cudaErrorInvalidValue;
    // the local ranks side by side: H = [act(x A_rank0) | ... ], K of the second
    // projection = nranks * f_s, tile t of it = output tile t % otiles of rank t / otiles
    Problem pl = p;
    pl.tp = nranks;
    pl.d_ff = nranks * p.fs;
    WeightOperand w1, w2;
    if (!weight_raw_first(&w1, pl, A, false) || !weight_raw_second(&w2, pl, B, false, true))
        return cudaErrorInvalidValue;
    cudaError_t e = run_skinny(w1, x, p.T, p.d_in, first_epi(p.act), h, pl.d_ff, part, counters, status, num_sms,
                               st, kSplitAuto, launches);
    if (e != cudaSuccess) return e;
    const int BT = skinny_bt(p.T);
    CUtensorMap mx;
    if (!make_map(&mx, h, pl.d_ff, p.T, BT)) return cudaErrorInvalidValue;
    TcArgs a{};
    a.rows_x = p.T;
    a.rows_w = w2.tiles;
    a.K = pl.d_ff;
    a.KB = w2.KB;
    a.epi = EPI_AR;
    a.ldo = p.d_out;
    a.out_cols = p.d_out;
    a.total_iters = (long long)w2.tiles * w2.KB;
    a.split_mode = kSplitSeparate;
    a.status = status;
    a.prank = w2.prank;
    a.otiles = w2.otiles;
    a.ar_rank0 = rank0;
    a.ar_ranks = p.tp;
    a.ar_rows = xa.rows;
    a.recv_off = xa.recv_off;
    for (int i = 0; i < p.tp; ++i) a.comm[i] = static_cast<uint8_t *>(xa.comm[i]);
    for (int i = 0; i < nranks; ++i) a.outs[i] = static_cast<__nv_bfloat16 *>(xa.outs[i]);
    switch (BT) {
        case 16: e = launch_ar_bt<16, TPMLP_SK_S16>(w2, mx, a, num_sms, st); break;
        case 32: e = launch_ar_bt<32, TPMLP_SK_S32>(w2, mx, a, num_sms, st); break;
        case 64: e = launch_ar_bt<64, TPMLP_SK_S64>(w2, mx, a, num_sms, st); break;
        default: e = launch_ar_bt<128, TPMLP_SK_S128>(w2, mx, a, num_sms, st); break;
    }
    if (e == cudaSuccess) ++*launches;
    return e;
}

bool fused_supported(const Problem &p, bool raw) { return fused_ok(p, raw); }

size_t xgpu_header_bytes(const Problem &p) {
    return kArControlBytes + align256((size_t)p.tp * blk_tiles(p.d_out) * 8 * 4);
}

bool tc_supported(const Problem &p) {
    return p.dtype == TP_MLP_BF16 && p.d_in % 8 == 0 && p.d_ff % 8 == 0 && p.d_out % 8 == 0 &&
           encode_fn() != nullptr;
}

bool tc_raw_supported(const Problem &p) { return tc_supported(p) && p.fs % BK == 0; }

// Counters serve the in-kernel fixup of the skinny kernel, which only runs
// 256-row tiles: the first projection's tiles (either layout) then the
// second's; then the fused kernel's two words (stored H tiles, CTAs past the
// wait).
size_t fused_counter_offset(const Problem &p) {
    return (size_t)(std::max(skinny_tiles(p, 0, false, false), skinny_tiles(p, 0, true, false)) +
                    blk_tiles(p.d_out));
}
size_t tile_counter_slots(const Problem &p) { return fused_counter_offset(p) + 2; }

// Split-tile scratch: the largest over both layouts, both projections and both
// tile heights, since the split mode may change after the workspace is sized.
size_t tc_workspace_bytes(const Problem &p, int num_sms) {
    if (p.T < 1 || p.T > kTcSkinnyMaxTokens) return 0;
    const int BT = skinny_bt(p.T);
    size_t m = 0;
    for (int raw = 0; raw < 2; ++raw)
        for (int proj = 0; proj < 2; ++proj)
            for (int half = 0; half < 2; ++half) {
                if (half && proj == 0 && p.act == TP_MLP_ACT_SWIGLU) continue;
                const long long tiles = skinny_tiles(p, proj, raw, half);
                const StreamKGeom g = skinny_geom((int)tiles, (int)blk_kblocks(proj ? p.d_ff : p.d_in), BT, num_sms);
                m = std::max(m, (size_t)g.tiles * g.slots * (half ? 128 : 256) * BT * 4);
            }
    if (p.fs % BK == 0) {   // per-rank partials: tp x the output tiles, one rank's k-blocks each
        const long long tiles = p.tp * skinny_tiles(p, 1, true, false);
        const StreamKGeom g = skinny_geom((int)tiles, p.fs / BK, BT, num_sms);
        m = std::max(m, (size_t)g.tiles * g.slots * 256 * BT * 4);
    }
    for (int v = 0; v < 3; ++v) {   // fused: the second projection on the first one's grid
        const bool half = v == 1, raw = v == 2;
        if (raw && p.fs % BK) continue;
        const FusedGeom f = fused_geom(p, half, raw, num_sms);
        m = std::max(m, (size_t)f.g2.tiles * f.g2.slots * (half ? 128 : 256) * BT * 4);
    }
    return align256(m);
}

cudaError_t launch_tc(const Problem &p, int tiling, const void *x, const void *w1p, const void *w2p,
                      const ShardPtrs *rawA, const ShardPtrs *rawB, void *h, void *out, float *part,
                      unsigned *counters, int *status, int num_sms, cudaStream_t st, const Marks &marks,
                      int split_mode, int *launches, float *partials) {
    *launches = 0;
    WeightOperand w1, w2;
    const bool raw = rawA != nullptr;
    if (partials && !raw) return cudaErrorInvalidValue;   // per-rank partials come from the shard form
    if (tiling == kTilingFused) {   // the forward only (no per-rank partials)
        if (partials) return cudaErrorNotSupported;
        return run_fused(p, x, w1p, w2p, rawA, rawB, h, out, part, counters, status, num_sms, st, marks, launches);
    }
    if (tiling == kTilingPair || tiling == kTilingPair2) {   // packed weights only
        if (raw || partials) return cudaErrorNotSupported;
        auto nb = [&](int proj) { return tiling == kTilingPair2 ? 2 : pair_tiles_per_unit(p, proj, num_sms); };
        marks.mark(0, st);
        cudaError_t e = (nb(0) == 2 ? run_pair<2> : run_pair<1>)(p, 0, w1p, x, p.T, p.d_in, first_epi(p.act), h,
                                                                   p.d_ff, status, num_sms, st);
        if (e != cudaSuccess) return e;
        marks.mark(1, st);
        e = (nb(1) == 2 ? run_pair<2> : run_pair<1>)(p, 1, w2p, h, p.T, p.d_ff, EPI_OUT, out, p.d_out, status,
                                                     num_sms, st);
        marks.mark(2, st);
        *launches = 2;
        return e;
    }
    const bool skinny = tiling == kTilingSkinny;
    const int BT = skinny_bt(p.T);
    const bool half1 = skinny && skinny_half(0, p.act, BT, split_mode, raw);
    const bool half2 = skinny && skinny_half(1, p.act, BT, split_mode, raw);
    const int epi2 = partials ? EPI_PART : EPI_OUT;
    void *out2 = partials ? static_cast<void *>(partials) : out;
    if (raw) {
        if (!weight_raw_first(&w1, p, *rawA, half1) || !weight_raw_second(&w2, p, *rawB, half2, partials != nullptr))
            return cudaErrorInvalidValue;
    } else if (!weight_packed(&w1, p, 0, w1p, half1) || !weight_packed(&w2, p, 1, w2p, half2)) {
        return cudaErrorInvalidValue;
    }
    cudaError_t e;
    marks.mark(0, st);
    if (skinny) {
        unsigned *cnt1 = counters;
        unsigned *cnt2 = counters + std::max(skinny_tiles(p, 0, false, false), skinny_tiles(p, 0, true, false));
        e = run_skinny(w1, x, p.T, p.d_in, first_epi(p.act), h, p.d_ff, part, cnt1, status, num_sms, st,
                       split_mode, launches);
        if (e != cudaSuccess) return e;
        marks.mark(1, st);
        e = run_skinny(w2, h, p.T, p.d_ff, epi2, out2, p.d_out, part, cnt2, status, num_sms, st, split_mode,
                       launches);
    } else {
        auto wide = tiling == kTilingWide256 ? run_wide<2> : run_wide<1>;
        e = wide(w1, x, p.T, p.d_in, first_epi(p.act), h, p.d_ff, status, num_sms, st);
        if (e != cudaSuccess) return e;
        marks.mark(1, st);
        e = wide(w2, h, p.T, p.d_ff, epi2, out2, p.d_out, status, num_sms, st);
        *launches = 2;
    }
    marks.mark(2, st);
    return e;
}

}  // namespace tpmlp
