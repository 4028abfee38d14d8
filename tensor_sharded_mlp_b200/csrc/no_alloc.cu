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
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace tpmlp {
namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;   // 8 MiB

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

typedef CUresult (*PFN_range)(CUdeviceptr *, size_t *, CUdeviceptr);

// A device pointer inside one allocation that holds `bytes` from it (a wrong
// pointer becomes an error code rather than an out-of-bounds access).
int check_range(const void *p, size_t bytes) {
    static PFN_range fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *q = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &q, 12000, cudaEnableDefault, &r) ==
                cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_range>(q);
    });
    if (!fn) return TP_MLP_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS) return TP_MLP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(p) + bytes > base + size) return TP_MLP_ERR_SHAPE;
    return TP_MLP_OK;
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

    // scratch layout: [split-tile counters | status word | H (tokens x d_ff bf16) | partial sums]
    const size_t n_cnt = tile_counter_slots(p);
    const size_t cnt_bytes = align256((n_cnt + 1) * sizeof(unsigned));
    const size_t h_bytes = align256((size_t)tokens * d_ff * 2);
    const size_t part_bytes = gemv_workspace_bytes(p, sms);
    if (cnt_bytes + h_bytes + part_bytes > kStaticScratchBytes) return TP_MLP_ERR_WORKSPACE;
    int s;
    if ((s = check_range(x, (size_t)tokens * d_model * 2))) return s;
    if ((s = check_range(out, (size_t)tokens * d_out * 2))) return s;
    if ((s = check_range(packed, packed_total_bytes(p)))) return s;

    char *base = static_cast<char *>(scratch);
    unsigned *counters = reinterpret_cast<unsigned *>(base);
    void *h = base + cnt_bytes;
    float *part = reinterpret_cast<float *>(base + cnt_bytes + h_bytes);
    const void *w2p = static_cast<const char *>(packed) + packed_part2_offset(p);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(counters, 0, cnt_bytes, st) != cudaSuccess) return TP_MLP_ERR_CUDA;
    Marks none;
    none.n = 0;
    int launches = 0;
    int *status = reinterpret_cast<int *>(counters + n_cnt);
    if (launch_gemv(p, x, packed, w2p, h, out, part, counters, status, sms, st, none, &launches) != cudaSuccess)
        return TP_MLP_ERR_CUDA;
    return TP_MLP_OK;
}
