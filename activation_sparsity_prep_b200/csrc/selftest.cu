// selftest.cu -- failure-path self-test of the bounded device waits.
//
// Every spin in the library's kernels (grid barriers, mbarrier waits) gives
// up after a time limit, records a timeout bit in a device status word and
// returns.  This kernel exercises that path on purpose without faulting or
// hanging anything: a grid wait that one block never joins.
#include "common.cuh"
#include "sharq_internal.h"

namespace sharq {

unsigned take_status_selftest() { return take_tu_status(); }

namespace {

// Every block but the last arrives on *counter and waits for all gridDim.x
// arrivals.  The last block never arrives, so each wait runs out after
// limit_ns, records the timeout bit and returns -- the path a real grid
// barrier takes when a block is lost.
__global__ void __launch_bounds__(32) wait_selftest_kernel(uint32_t* counter,
                                                            unsigned long long limit_ns) {
    if (blockIdx.x == gridDim.x - 1 || threadIdx.x != 0) return;
    atomicAdd(counter, 1u);
    const unsigned long long t0 = globaltimer();
    while (ld_acquire_gpu(counter) < gridDim.x) {
        if (globaltimer() - t0 > limit_ns) {
            record_status(kStatusGridTimeout);
            break;
        }
        __nanosleep(256);
    }
}

}  // namespace

cudaError_t launch_wait_selftest(uint32_t* counter, unsigned long long limit_ns, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    wait_selftest_kernel<<<4, 32, 0, s>>>(counter, limit_ns);
    return cudaGetLastError();
}

}  // namespace sharq
