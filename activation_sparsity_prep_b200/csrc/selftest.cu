// selftest.cu -- failure-path self-test of the bounded device waits.
//
// Every spin in the library's kernels (grid barriers, mbarrier waits) gives
// up after a time limit, records a timeout bit in a device status word and
// returns.  These kernels run the library's own wait helpers (grid_barrier
// and mbar_wait from common.cuh, the ones the prepare and linear kernels
// use) on purpose into that limit, without faulting or hanging anything:
// a grid barrier that one block never arrives at, and an mbarrier phase
// that nothing completes.  The prepare's own barriers are exercised through
// sharq_selftest_prepare_timeout (a real prepare launch with one block that
// skips its arrivals).
#include "common.cuh"
#include "sharq_internal.h"

namespace sharq {

unsigned take_status_selftest() { return take_tu_status(); }

namespace {

// Mode 0: every block runs grid_barrier, the last one without arriving, so
// every wait (the last block's too) runs out after limit_ns.  Mode 1: one
// thread waits on a freshly initialised mbarrier whose first phase nothing
// completes.
__global__ void __launch_bounds__(32) wait_selftest_kernel(uint32_t* counter,
                                                            unsigned long long limit_ns, int mode) {
    if (mode == 0) {
        grid_barrier(counter, gridDim.x, limit_ns, blockIdx.x == gridDim.x - 1);
        return;
    }
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, limit_ns);
}

}  // namespace

cudaError_t launch_wait_selftest(uint32_t* counter, unsigned long long limit_ns, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    wait_selftest_kernel<<<4, 32, 0, s>>>(counter, limit_ns, 0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wait_selftest_kernel<<<1, 32, 0, s>>>(counter, limit_ns, 1);
    return cudaGetLastError();
}

}  // namespace sharq
