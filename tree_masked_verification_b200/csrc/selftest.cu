// selftest.cu -- failure detection exercised on the GPU without a fault.
//
// Every wait of the verification kernels is bounded (mbar_wait gives up
// after kWaitLimitCycles of the SM cycle counter) and a wait that gives up
// records kStatusPipelineTimeout in the workspace status word, which the
// host reads with longspec_hta_get_status.  This kernel runs that path on
// purpose: one thread waits on an mbarrier that nothing arrives on, the
// bound expires (about 2 s at B200 clocks), the status bit is set and the
// kernel returns normally, leaving the context usable.  No fault, trap or
// unbounded loop is involved.
#include "hta_kernels.h"

namespace hta {

namespace {

__global__ void wait_timeout_kernel(uint32_t *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    // phase 0 of `bar` never completes: no thread arrives on it
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0)) raise_status(status, kStatusPipelineTimeout);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint32_t *status, cudaStream_t stream) {
    wait_timeout_kernel<<<1, 32, 0, stream>>>(status);
    return cudaGetLastError();
}

}  // namespace hta
