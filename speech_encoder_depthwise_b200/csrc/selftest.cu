// Self-test of the bounded waits: every kernel that waits on an mbarrier for its own copies gives
// up after kSpinLimit polls, records an error word and returns, so a copy that never arrives
// cannot hang the GPU.  This launch runs the same wait (with a limit 256 times shorter) on a
// barrier that nothing will ever complete, so the wait must run out; the host then reads DW_ERR_TIMEOUT from dw_device_error() and the context
// stays usable.  No fault is raised and nothing is left in flight.
#include "dw_internal.h"

namespace dwk {
namespace {

__global__ void wait_timeout_kernel(int *done, uint32_t limit) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none will come
        fence_barrier_init();
    }
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0, limit);  // bounded: gives up and sets the error word
    if (threadIdx.x == 0) *done = ok ? 1 : 2;
}

}  // namespace

cudaError_t selftest_wait_timeout_launch(int *done, cudaStream_t s) {
    // the production waits poll kSpinLimit times; the self-test runs the same wait with a
    // shorter limit so that it ends quickly
    wait_timeout_kernel<<<1, 32, 0, s>>>(done, kSpinLimit >> 8);
    return cudaGetLastError();
}

unsigned int selftest_take_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, dw_device_error_flag, sizeof(v)) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(dw_device_error_flag, &zero, sizeof(zero));
    return v;
}

}  // namespace dwk
