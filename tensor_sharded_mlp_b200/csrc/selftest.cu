// selftest.cu -- exercises the bounded wait that every pipelined kernel here uses.
//
// One CTA initialises an mbarrier that nothing will ever arrive on and waits
// for it through mbar_wait with a short limit.  The wait gives up, raises the
// abort flag, and the kernel records the timeout in the handle's status word
// and returns -- the same path a production kernel takes if a copy or an MMA
// never completes.  Nothing traps and the context stays usable.
#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace tpmlp {
namespace {

__global__ void bounded_wait_selftest(int *status, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(tc::smem_u32(&bar), 1);
        abort_flag = 0;
        tc::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = tc::mbar_wait(tc::smem_u32(&bar), 0, &abort_flag, limit_ns);
        if (!ok) atomicExch(status, 1);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int *status, unsigned wait_us, cudaStream_t st) {
    bounded_wait_selftest<<<1, 32, 0, st>>>(status, (unsigned long long)wait_us * 1000ull);
    return cudaGetLastError();
}

}  // namespace tpmlp
