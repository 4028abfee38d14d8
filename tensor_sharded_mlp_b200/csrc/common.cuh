// common.cuh -- small device/host helpers shared by the CUDA kernels of the
// tensor-parallel MLP library.  No MLP arithmetic lives here.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/tp_mlp.h"

namespace tpmlp {

constexpr int kMaxTp = 8;
constexpr int kSwigluBlock = 128;   // gate/up interleave granularity of the packed layout

// Per-rank shard pointers, passed to kernels by value.
struct ShardPtrs {
    const void *p[kMaxTp];
};

// Problem description shared by every launcher.
struct Problem {
    int T;        // tokens
    int d_in;     // d_model
    int d_ff;     // sum of shard widths
    int d_out;
    int tp;
    int fs;       // d_ff / tp
    int act;      // tp_mlp_act
    int dtype;    // tp_mlp_dtype
};

// --- element conversion ------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename E> __device__ __forceinline__ E from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Two bf16 packed in a 32-bit word -> two floats (exact: bf16 is the top half of fp32).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// --- activations ---------------------------------------------------------------
// Precise forms (fp32 path, 1e-5 tolerance): the library's tanhf / expf.
// SiLU(g) = g * sigma(g) = g / (1 + e^{-g}); large negative g: e^{-g} -> inf, result -> -0.
__device__ __forceinline__ float silu_precise(float g) { return g / (1.0f + expf(-g)); }
// Fast forms (bf16 paths, whose H is rounded to bf16 anyway): the hardware
// tanh approximation (one instruction, relative error about 2^-11, below bf16's
// 2^-9 rounding), and SiLU through sigma(g) = (1 + tanh(g/2)) / 2.
__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float silu_fast(float g) { return g * fmaf(0.5f, tanh_fast(0.5f * g), 0.5f); }

template <bool kFast>
__device__ __forceinline__ float activate(int act, float u, float v) {
    if (act == TP_MLP_ACT_TANH) return kFast ? tanh_fast(u) : tanhf(u);
    if (act == TP_MLP_ACT_SWIGLU) return (kFast ? silu_fast(u) : silu_precise(u)) * v;
    return u;
}

// --- packed layout (shard-layout packer) --------------------------------------------
// Each part of the packed buffer is a matrix of "rows" (one per output of its
// projection) by K, stored tile-blocked: rows in tiles of kTileRows, K in
// blocks of kKBlock, block (tile, kb) = kTileRows x kKBlock elements stored
// contiguously (row-major inside), blocks of one tile consecutive in kb, tiles
// consecutive.  So a tile x k-block is one contiguous piece (32 KB in bf16)
// and a run of consecutive (tile, kb) pairs is one contiguous range of memory.
// Padding (rows past the end, k past the end, absent SwiGLU features) is zero.
constexpr int kTileRows = 256;
constexpr int kKBlock = 64;

// Row of the first-projection part holding feature n (0 <= n < d_ff); `up`
// selects the up row of a SwiGLU feature.  SwiGLU: tile b holds the gate rows
// of features 128b..128b+127 in rows 0..127 and their up rows in rows 128..255.
__host__ __device__ __forceinline__ long w1p_row(int n, bool up, int act) {
    if (act != TP_MLP_ACT_SWIGLU) return n;
    const int b = n / kSwigluBlock;
    return (long)kTileRows * b + (up ? kSwigluBlock : 0) + (n - b * kSwigluBlock);
}
// Logical rows of the first-projection part.
__host__ __device__ __forceinline__ long w1p_rows(int d_ff, int act) {
    return act == TP_MLP_ACT_SWIGLU ? (long)kTileRows * ((d_ff + kSwigluBlock - 1) / kSwigluBlock) : (long)d_ff;
}
__host__ __device__ __forceinline__ long blk_tiles(long rows) { return (rows + kTileRows - 1) / kTileRows; }
__host__ __device__ __forceinline__ long blk_kblocks(long K) { return (K + kKBlock - 1) / kKBlock; }
// Element offset of (row, k) inside a part whose K spans KB blocks.
__host__ __device__ __forceinline__ long blk_offset(long row, long k, long KB) {
    return (((row / kTileRows) * KB + k / kKBlock) * kTileRows + (row % kTileRows)) * kKBlock + (k % kKBlock);
}
// Elements of a part (padded to whole tiles and k-blocks).
__host__ __device__ __forceinline__ size_t part_elems(long rows, long K) {
    return (size_t)blk_tiles(rows) * blk_kblocks(K) * kTileRows * kKBlock;
}
__host__ __device__ __forceinline__ size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// --- cache-hinted loads ----------------------------------------------------------
// 16-byte streaming load: read-only, not kept in L1 (weights are read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// --- programmatic dependent launch (PDL) -----------------------------------------
// Let the next kernel in the stream start its independent prologue now.
__device__ __forceinline__ void pdl_allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until the previous kernel in the stream has completed and its writes are
// visible (returns at once when there is no programmatic dependency).
__device__ __forceinline__ void pdl_wait_previous() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Bulk prefetch of [p, p + bytes) into L2 (p and bytes multiples of 16).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and device
// (a per-device property; repeating it on every launch costs host time).
// Registry keyed by the kernel's address (host code only).
bool smem_attr_done(const void *fn, int dev);
void smem_attr_mark(const void *fn, int dev);

template <typename K>
cudaError_t ensure_smem_attr(K kern, size_t bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    const void *fn = reinterpret_cast<const void *>(kern);
    if (smem_attr_done(fn, dev)) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) smem_attr_mark(fn, dev);
    return e;
}

// Launch with the programmatic-stream-serialization attribute, so the kernel may
// begin while the previous kernel in the stream drains (it must call
// pdl_wait_previous() before touching that kernel's outputs).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The same with thread-block clusters of `cluster` CTAs along x (gridDim.x must
// be a multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               unsigned cluster, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace tpmlp
