// pack.cu -- the shard-layout packer: a bit-exact reordering of the per-rank
// shards into the K-major layout the fast kernels stream.
//
// Shards as the pages define them ("大模型推理系统揭秘（07）", §1.2.2–§1.2.3):
// rank i holds the column block A[:, i f_s:(i+1) f_s] of the first weight and
// the row block B[i f_s:(i+1) f_s, :] of the second.  The packed buffer holds
//   part 1: row w1p_row(n) = column n of A (gate/up paired in 256-row tiles
//           for SwiGLU), K = d_in;
//   part 2: row c = column c of B over all ranks' rows in rank order, K = d_ff;
// each part tile-blocked (common.cuh): 256 rows x 64 k per contiguous block.
// Packing zeroes the buffer first (padding must read as zero), then both
// directions are 32x32 tiled transposes through shared memory so that reads
// and writes are coalesced.  Elements are moved as raw bits.
#include "common.cuh"
#include "internal.h"

namespace tpmlp {
namespace {

constexpr int TILE = 32;
constexpr int ROWS = 8;   // threadIdx.y extent

// Address of logical element (k, n) of a part, in the shard form and in the packed form.
// part 0: first projection gate (or only) block; part 1: up block; part 2: second projection.
template <typename U>
__device__ __forceinline__ U *shard_addr(const ShardPtrs &sh, const Problem &p, int part, int k, int n) {
    if (part < 2) {
        const int shard = n / p.fs;
        const long lda = (p.act == TP_MLP_ACT_SWIGLU) ? 2L * p.fs : (long)p.fs;
        U *a = static_cast<U *>(const_cast<void *>(sh.p[shard]));
        return a + (long)k * lda + (n - shard * p.fs) + (part == 1 ? p.fs : 0);
    }
    const int shard = k / p.fs;
    U *b = static_cast<U *>(const_cast<void *>(sh.p[shard]));
    return b + (long)(k - shard * p.fs) * p.d_out + n;
}

template <typename U>
__device__ __forceinline__ U *packed_addr(U *w1p, U *w2p, const Problem &p, int part, int k, int n) {
    if (part < 2) return w1p + blk_offset(w1p_row(n, part == 1, p.act), k, blk_kblocks(p.d_in));
    return w2p + blk_offset(n, k, blk_kblocks(p.d_ff));
}

// grid: (ceil(N / 32), ceil(K / 32)), block (32, 8).  K/N of the part:
// parts 0/1: K = d_in, N = d_ff; part 2: K = d_ff, N = d_out.
template <typename U, bool UNPACK>
__global__ void __launch_bounds__(TILE *ROWS) transpose_part(ShardPtrs sh, U *w1p, U *w2p, Problem p, int part) {
    __shared__ U tile[TILE][TILE + 1];
    const int K = part < 2 ? p.d_in : p.d_ff;
    const int N = part < 2 ? p.d_ff : p.d_out;
    const int n0 = blockIdx.x * TILE, k0 = blockIdx.y * TILE;
    const int tx = threadIdx.x, ty = threadIdx.y;
    if (!UNPACK) {
        // read shard rows (n fastest), write packed rows (k fastest)
        for (int i = ty; i < TILE; i += ROWS) {
            const int k = k0 + i, n = n0 + tx;
            if (k < K && n < N) tile[i][tx] = *shard_addr<U>(sh, p, part, k, n);
        }
        __syncthreads();
        for (int i = ty; i < TILE; i += ROWS) {
            const int n = n0 + i, k = k0 + tx;
            if (k < K && n < N) *packed_addr<U>(w1p, w2p, p, part, k, n) = tile[tx][i];
        }
    } else {
        for (int i = ty; i < TILE; i += ROWS) {
            const int n = n0 + i, k = k0 + tx;
            if (k < K && n < N) tile[tx][i] = *packed_addr<U>(w1p, w2p, p, part, k, n);
        }
        __syncthreads();
        for (int i = ty; i < TILE; i += ROWS) {
            const int k = k0 + i, n = n0 + tx;
            if (k < K && n < N) *shard_addr<U>(sh, p, part, k, n) = tile[i][tx];
        }
    }
}

template <typename U, bool UNPACK>
cudaError_t run_parts(const Problem &p, const ShardPtrs &a, const ShardPtrs &b, void *packed,
                      cudaStream_t s) {
    U *w1p = static_cast<U *>(packed);
    U *w2p = reinterpret_cast<U *>(static_cast<char *>(packed) + packed_part2_offset(p));
    const dim3 blk(TILE, ROWS);
    if (!UNPACK) {
        cudaError_t e = cudaMemsetAsync(packed, 0, packed_total_bytes(p), s);
        if (e != cudaSuccess) return e;
    }
    const int nparts1 = p.act == TP_MLP_ACT_SWIGLU ? 2 : 1;
    for (int part = 0; part < nparts1; ++part) {
        const dim3 g((p.d_ff + TILE - 1) / TILE, (p.d_in + TILE - 1) / TILE);
        transpose_part<U, UNPACK><<<g, blk, 0, s>>>(a, w1p, w2p, p, part);
    }
    const dim3 g2((p.d_out + TILE - 1) / TILE, (p.d_ff + TILE - 1) / TILE);
    transpose_part<U, UNPACK><<<g2, blk, 0, s>>>(b, w1p, w2p, p, 2);
    return cudaGetLastError();
}

}  // namespace

size_t packed_part2_offset(const Problem &p) {
    const size_t e = p.dtype == TP_MLP_F32 ? 4 : 2;
    return align256(part_elems(w1p_rows(p.d_ff, p.act), p.d_in) * e);
}

size_t packed_total_bytes(const Problem &p) {
    const size_t e = p.dtype == TP_MLP_F32 ? 4 : 2;
    return packed_part2_offset(p) + align256(part_elems(p.d_out, p.d_ff) * e);
}

cudaError_t launch_pack(const Problem &p, const ShardPtrs &a, const ShardPtrs &b, void *packed,
                        bool unpack, cudaStream_t s) {
    if (p.dtype == TP_MLP_F32)
        return unpack ? run_parts<uint32_t, true>(p, a, b, packed, s)
                      : run_parts<uint32_t, false>(p, a, b, packed, s);
    return unpack ? run_parts<uint16_t, true>(p, a, b, packed, s)
                  : run_parts<uint16_t, false>(p, a, b, packed, s);
}

}  // namespace tpmlp
