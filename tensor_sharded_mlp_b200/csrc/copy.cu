// copy.cu -- a step's host<->device copies as a kernel.
//
// A decode step moves a few kilobytes in and out ("7.4 推理侧并行" §7.4.1: one
// token's activations against gigabytes of weights), so its copies cost their
// fixed overhead, not their bytes.  A copy-engine transfer in a CUDA graph
// costs several microseconds of setup on each side of the step's kernels;
// a kernel that loads from (or stores to) page-locked host memory mapped
// into the device's address space does the same move over the bus directly,
// and under programmatic dependent launch the step's first kernel is already
// resident when it finishes.
//
// The copy is 16-byte words, grid-strided, with the last bytes % 16 bytes
// done by the first threads of block 0.
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace tpmlp {
namespace {

constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads)
    copy_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, long long n16, int tail) {
    pdl_allow_dependents();
    pdl_wait_previous();   // the source may come from the previous kernel
    const long long stride = (long long)gridDim.x * kCopyThreads;
    long long i = (long long)blockIdx.x * kCopyThreads + threadIdx.x;
    // four words in flight per thread: the bus round trip, not the issue rate, is the cost
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = src[i], b = src[i + stride], c = src[i + 2 * stride], d = src[i + 3 * stride];
        dst[i] = a;
        dst[i + stride] = b;
        dst[i + 2 * stride] = c;
        dst[i + 3 * stride] = d;
    }
    for (; i < n16; i += stride) dst[i] = src[i];
    if (blockIdx.x == 0 && (int)threadIdx.x < tail) {
        const uint8_t *s = reinterpret_cast<const uint8_t *>(src + n16);
        uint8_t *t = reinterpret_cast<uint8_t *>(dst + n16);
        t[threadIdx.x] = s[threadIdx.x];
    }
}

}  // namespace

cudaError_t launch_copy(void *dst, const void *src, size_t bytes, int num_sms, cudaStream_t st) {
    if (bytes == 0) return cudaSuccess;
    const long long n16 = (long long)(bytes / 16);
    const int tail = (int)(bytes % 16);
    long long blocks = (n16 + kCopyThreads - 1) / kCopyThreads;
    if (blocks < 1) blocks = 1;
    if (blocks > 2LL * num_sms) blocks = 2LL * num_sms;
    return launch_pdl(copy_kernel, dim3((unsigned)blocks), dim3(kCopyThreads), 0, st,
                      static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), n16, tail);
}

}  // namespace tpmlp
