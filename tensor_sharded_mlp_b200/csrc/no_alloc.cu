// no_alloc.cu -- a decode forward that needs no caller-provided workspace.
//
// Some callers cannot allocate device memory at all: code running inside a
// host callback or a custom allocator hook, plugins whose host process owns
// every allocation, or sandboxes where cudaMalloc is forbidden.  The regular
// entry points need a workspace from the caller for the intermediate
// activation H and the split-K scratch.  This file offers one entry point
// that keeps that scratch in a fixed array in device memory instead, compiled
// into the library.  Every GPU on which the library is loaded holds that array
// (kStaticScratchBytes) until the process exits.
//
// The array is shared by every call, in every thread and on every stream, and
// keeps whatever the last call left in it.  Two calls whose kernels overlap on
// the GPU therefore race and corrupt each other's results; callers must order
// them (one stream, or events).  The split-K counters that must start at zero
// are cleared by each call, on its stream, before its kernels run.
//
// Layout of the array: [status word, 256 bytes | split-tile counters | H |
// split-K partial sums].  The status word sits at a fixed place that no call
// clears; a kernel that gives up a bounded wait sets it, and
// tp_mlp_decode_static_status reads and clears it.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace tpmlp {
namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;   // 8 MiB
constexpr size_t kStatusBytes = 256;                // the status word's slot at the front

// The scratch itself.  Host code may not use this name as an address (on the
// host it is only a stand-in); it asks the runtime for the device address.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices];
int g_num_sms[kMaxDevices];

// Once per device, with that device current: look up the array's device
// address and the SM count.  Returns false if the runtime refuses.
bool device_setup(int dev, void **ptr, int *sms) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return false;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return false;
        g_num_sms[dev] = n;
        g_scratch_ptr[dev] = p;
    }
    *ptr = g_scratch_ptr[dev];
    *sms = g_num_sms[dev];
    return true;
}

}  // namespace
}  // namespace tpmlp

using namespace tpmlp;

extern "C" int tp_mlp_decode_forward_static(int d_model, int d_ff, int d_out, int tp_degree, int act,
                                            const void *x, int tokens, const void *packed, void *out,
                                            tp_mlp_stream_t stream) {
    if (act != TP_MLP_ACT_TANH && act != TP_MLP_ACT_SWIGLU && act != TP_MLP_ACT_IDENTITY)
        return TP_MLP_ERR_INVALID_ARG;
    if (d_model < 1 || d_ff < 1 || d_out < 1 || tp_degree < 1 || tp_degree > kMaxTp || d_ff % tp_degree)
        return TP_MLP_ERR_SHAPE;
    if (tokens < 0 || tokens > kGemvMaxTokens) return TP_MLP_ERR_SHAPE;
    if (tokens == 0) return TP_MLP_OK;
    if (!x || !packed || !out) return TP_MLP_ERR_INVALID_ARG;
    if (((uintptr_t)x | (uintptr_t)packed | (uintptr_t)out) & 15u) return TP_MLP_ERR_ALIGNMENT;
    Problem p;
    p.T = tokens;
    p.d_in = d_model;
    p.d_ff = d_ff;
    p.d_out = d_out;
    p.tp = tp_degree;
    p.fs = d_ff / tp_degree;
    p.act = act;
    p.dtype = TP_MLP_BF16;
    if (!gemv_supported(p)) return TP_MLP_ERR_UNSUPPORTED;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TP_MLP_ERR_CUDA;
    void *scratch = nullptr;
    int sms = 0;
    if (!device_setup(dev, &scratch, &sms)) return TP_MLP_ERR_CUDA;

    // scratch layout: [status word | split-tile counters | H (tokens x d_ff bf16) | partial sums]
    const size_t n_cnt = tile_counter_slots(p);
    const size_t cnt_bytes = align256(n_cnt * sizeof(unsigned));
    const size_t h_bytes = align256((size_t)tokens * d_ff * 2);
    const size_t part_bytes = gemv_workspace_bytes(p, sms);
    if (kStatusBytes + cnt_bytes + h_bytes + part_bytes > kStaticScratchBytes) return TP_MLP_ERR_WORKSPACE;
    int s;
    if ((s = check_dev(x, (size_t)tokens * d_model * 2))) return s;
    if ((s = check_dev(out, (size_t)tokens * d_out * 2))) return s;
    if ((s = check_dev(packed, packed_total_bytes(p)))) return s;

    char *base = static_cast<char *>(scratch);
    int *status = reinterpret_cast<int *>(base);
    unsigned *counters = reinterpret_cast<unsigned *>(base + kStatusBytes);
    void *h = base + kStatusBytes + cnt_bytes;
    float *part = reinterpret_cast<float *>(base + kStatusBytes + cnt_bytes + h_bytes);
    const void *w2p = static_cast<const char *>(packed) + packed_part2_offset(p);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(counters, 0, n_cnt * sizeof(unsigned), st) != cudaSuccess) return TP_MLP_ERR_CUDA;
    Marks none;
    none.n = 0;
    int launches = 0;
    if (launch_gemv(p, x, packed, w2p, h, out, part, counters, status, sms, st, none, &launches) != cudaSuccess)
        return TP_MLP_ERR_CUDA;
    return TP_MLP_OK;
}

extern "C" int tp_mlp_decode_static_status(void) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TP_MLP_ERR_CUDA;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        scratch = g_scratch_ptr[dev];
    }
    if (!scratch) return TP_MLP_OK;   // no call has run on this device
    if (cudaDeviceSynchronize() != cudaSuccess) return TP_MLP_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TP_MLP_ERR_CUDA;
    if (v == 0) return TP_MLP_OK;
    const int zero = 0;
    if (cudaMemcpy(scratch, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return TP_MLP_ERR_CUDA;
    return TP_MLP_ERR_TIMEOUT;
}
