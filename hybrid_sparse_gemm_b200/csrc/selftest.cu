// Self-test of the failure path every kernel shares: a bounded mbarrier wait
// that nothing completes gives up after its limit, records a timeout in the
// device status word and returns, leaving the context usable.
#include "kernels.cuh"

namespace patch {

namespace {

__global__ void selftest_wait_kernel(int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait(&bar, 0, &abort_flag)) atomicCAS(status, 0, kStatusTimeout);
        mbar_arrive(&bar);  // complete the phase so the barrier is left consistent
    }
}

}  // namespace

cudaError_t launch_selftest_wait(int* status, cudaStream_t st) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(status);
    return cudaGetLastError();
}

}  // namespace patch
