// selftest.cu -- the failure path of the bounded waits, run without a fault.
//
// Every persistent decode kernel waits on mbarriers (pages landed, scores
// ready, buffers free) through mbar_wait, which gives up after a time limit on
// %globaltimer, records DCP_ERR_TIMEOUT in the sticky status word and raises
// the CTA's abort flag, so that a lost copy or a stuck partner ends the kernel
// with a status instead of a hang.  In a correct run that branch never
// executes.  This kernel executes it on purpose: one thread waits on a barrier
// that nothing ever arrives on, and reports what the wait returned.
#include "common.cuh"

namespace dcp {

namespace {

__global__ void __launch_bounds__(32) bounded_wait_kernel(int* status, int64_t* result) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none is ever made
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = global_timer_ns();
        const bool completed = mbar_wait(&bar, 0, &abort_flag, status);
        const uint64_t t1 = global_timer_ns();
        result[0] = completed ? 1 : 0;
        result[1] = abort_flag;
        result[2] = (int64_t)(t1 - t0);
    }
}

}  // namespace

cudaError_t launch_selftest_bounded_wait(int* status, int64_t* result, cudaStream_t s) {
    bounded_wait_kernel<<<1, 32, 0, s>>>(status, result);
    return cudaGetLastError();
}

}  // namespace dcp
