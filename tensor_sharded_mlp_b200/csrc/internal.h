// internal.h -- launchers shared between the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace tpmlp {

struct Problem;
struct ShardPtrs;

// Caller-owned events recorded around the kernels of one call (timing hook).
struct Marks {
    cudaEvent_t ev[8];
    int n;
    void mark(int i, cudaStream_t s) const {
        if (i < n && ev[i]) cudaEventRecord(ev[i], s);
    }
};

// tp_mlp.cu: a device pointer, 16-byte aligned, inside one device allocation
// that holds `bytes` from it (a tp_mlp_status code; TP_MLP_OK when it does).
int check_dev(const void *p, size_t bytes);

// simt.cu: tiled CUDA-core path, any shape, both dtypes, shard or packed layout.
// h: T x d_ff scratch (dtype).  partials != nullptr selects the per-rank output.
cudaError_t launch_simt(const Problem &p, bool packed, const void *x, const ShardPtrs &w1,
                        const ShardPtrs &w2, void *h, void *out, float *partials, cudaStream_t s,
                        const Marks &marks);

// pack.cu: shard-layout packer.
size_t packed_part2_offset(const Problem &p);
size_t packed_total_bytes(const Problem &p);
cudaError_t launch_pack(const Problem &p, const ShardPtrs &a, const ShardPtrs &b, void *packed,
                        bool unpack, cudaStream_t s);

// selftest.cu: a bounded wait that runs out, recorded in *status.
cudaError_t launch_bounded_wait_selftest(int *status, unsigned wait_us, cudaStream_t st);

// fused_norm.cu: the rank sum of fp32 partials (P x rows x d) + residual add +
// RMSNorm, one kernel (clusters of up to kNormClusterMax CTAs per row).
constexpr int kNormClusterMax = 8;
constexpr int kNormMaxWidth = 49152;   // h of a row chunk lives in shared memory
cudaError_t launch_allreduce_norm(const float *partials, int P, int rows, int d, const void *residual,
                                  const void *gamma, float eps, int dtype, void *y, void *residual_out,
                                  int num_sms, cudaStream_t st);

// attn_merge.cu: merge of P ranks' partial attention results (maximum,
// exp_sum: P x rows fp32; weighted: P x rows x D of dtype) into rows x D.
constexpr int kMergeMaxHeadDim = 4096;
cudaError_t launch_attn_merge(int P, int rows, int D, const float *maximum, const float *exp_sum,
                              const void *weighted, int dtype, void *out, cudaStream_t st);

// copy.cu: `bytes` from src to dst by a kernel (either side may be page-locked
// host memory mapped into the device's address space); copies above
// kCopyKernelMaxBytes go to the copy engine instead.
constexpr size_t kCopyKernelMaxBytes = 1u << 20;
cudaError_t launch_copy(void *dst, const void *src, size_t bytes, int num_sms, cudaStream_t st);

// Split-tile counters the GEMV and tcgen05 skinny kernels need (one per
// weight tile of both parts; first part's tiles first).
size_t tile_counter_slots(const Problem &p);
size_t fused_counter_offset(const Problem &p);   // the fused skinny kernel's two words

// gemv.cu: decode path, packed bf16, 1..kGemvMaxTokens tokens.
constexpr int kGemvMaxTokens = 4;
bool gemv_supported(const Problem &p);
size_t gemv_workspace_bytes(const Problem &p, int num_sms);
cudaError_t launch_gemv(const Problem &p, const void *x, const void *w1p, const void *w2p, void *h, void *out,
                        float *part, unsigned *counters, int *status, int num_sms, cudaStream_t st,
                        const Marks &marks, int *launches);

// tc_gemm.cu: tcgen05 path, packed bf16.  skinny: tokens <= kTcSkinnyMaxTokens.
constexpr int kTcSkinnyMaxTokens = 128;
constexpr int kTcWide256MinTokens = 2048;   // auto, shard form: 256-token tiles from here on
// auto, packed weights: pairs of CTAs (cta_group::2) from kTcPairMinTokens to
// kTcPairMaxTokens tokens, one or two 256-row weight tiles per unit chosen per
// projection by wave efficiency (tc_gemm.cu, pair_tiles_per_unit), and two
// tiles per unit (256 x 512) above (measured on B200, sweep d 4096 / f 16384:
// T=1024 198-205 us pair vs 228 us 128-token tiles and 264 us two-tile pairs
// on both projections; prefill d 8192 / f 28672, T=8192, power-capped at ~1.2
// GHz: two-tile pairs 8.56-8.58 ms, 1-CTA 256-token tiles 8.69-8.74, one-tile
// pairs 8.88-8.93).
constexpr int kTcPairMinTokens = 512;
constexpr int kTcPairMaxTokens = 4096;
// kTilingFused: the skinny tiling with both projections in one persistent
// launch (packed weights or the shard form, 1..kTcSkinnyMaxTokens tokens;
// fused_supported).
enum { kTilingSkinny = 0, kTilingWide128 = 1, kTilingWide256 = 2, kTilingPair = 3, kTilingPair2 = 4, kTilingFused = 5 };
bool tc_supported(const Problem &p);
bool fused_supported(const Problem &p, bool raw);   // raw: the shard form
bool tc_raw_supported(const Problem &p);   // also needs f_s % 64 == 0
size_t tc_workspace_bytes(const Problem &p, int num_sms);
// Split tiles of the skinny tiling (values of tp_mlp_splitk): finished by the
// last CTA to arrive, inside the GEMM kernel, or by a reduction kernel behind it.
enum { kSplitAuto = 0, kSplitInKernel = 1, kSplitSeparate = 2, kSplitCluster = 3 };
// Packed weights (w1p/w2p), or the per-rank shards when rawA/rawB are given.
// *launches receives the number of kernels launched.  partials != nullptr
// (shard form only): the second projection writes each rank's fp32 partial
// output to partials[rank][token][column] instead of the sum to out.
cudaError_t launch_tc(const Problem &p, int tiling, const void *x, const void *w1p, const void *w2p,
                      const ShardPtrs *rawA, const ShardPtrs *rawB, void *h, void *out, float *part,
                      unsigned *counters, int *status, int num_sms, cudaStream_t st, const Marks &marks,
                      int split_mode, int *launches, float *partials = nullptr);

// tc_gemm.cu: tensor parallelism across GPUs with the one-shot all-reduce
// fused into the second projection (bf16, f_s % 64 == 0, 1..128 tokens).
// Ranks rank0 .. rank0 + nranks - 1 of p.tp run here (one per GPU, or every
// rank on one GPU); comm[r] is rank r's exchange buffer as this process sees
// it: [control + flags (xgpu_header_bytes) | receive rows: 2 x tp x rows x
// d_out bf16], zeroed before its first use.  The call count (epoch) lives in
// the control words, so launches can be captured in a CUDA graph.
struct XgpuArgs {
    void *comm[kMaxTp];
    void *outs[kMaxTp];     // output of local rank i (tokens x d_out bf16)
    size_t recv_off;        // = xgpu_header_bytes(p)
    int rows;               // receive rows per (half, rank): the handle's max tokens
};
size_t xgpu_header_bytes(const Problem &p);
// Sequence-parallel variant: x_local[i] holds local rank i's T / tp token
// rows; they are gathered into every rank's buffer at gather_off (T x d_in
// bf16) before the first projection, and the second projection's exchange is
// a reduce-scatter: outs[i] gets rank i's own T / tp rows.  T % tp == 0.
cudaError_t launch_xgpu_sp(const Problem &p, int rank0, int nranks, const void *const *x_local, const ShardPtrs &A,
                           const ShardPtrs &B, void *h, float *part, unsigned *counters, int *status, int num_sms,
                           cudaStream_t st, const XgpuArgs &xa, size_t gather_off, int *launches);
// h: tokens x (nranks * f_s) scratch; part / counters: split-tile scratch of
// the first projection.  cudaErrorNotSupported: the clusters do not all fit.
cudaError_t launch_xgpu(const Problem &p, int rank0, int nranks, const void *x, const ShardPtrs &A,
                        const ShardPtrs &B, void *h, float *part, unsigned *counters, int *status, int num_sms,
                        cudaStream_t st, const XgpuArgs &xa, int *launches);

}  // namespace tpmlp
