// Failure-detection plumbing of the workspace header: the runtime limit of the
// bounded device waits, and a diagnostic kernel whose only wait can never
// complete, so that the timeout path (status word = MSA_ERR_TIMEOUT, context
// still usable) can be exercised without faulting or hanging the GPU.
#include "msa_device.cuh"

namespace msa {

namespace {

__global__ void set_wait_limit_kernel(int *ws, unsigned long long limit_ns) {
    *reinterpret_cast<unsigned long long *>(ws + kWaitLimitWord) = limit_ns;
}

// One thread waits, bounded by the workspace's wait limit, for phase 0 of an
// mbarrier that expects one arrival and gets none.
__global__ void wait_never_kernel(int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0, status);
    }
}

}  // namespace

cudaError_t launch_set_wait_limit(int *ws, unsigned long long limit_ns, cudaStream_t s) {
    set_wait_limit_kernel<<<1, 1, 0, s>>>(ws, limit_ns);
    return cudaGetLastError();
}

cudaError_t launch_wait_never(int *ws, cudaStream_t s) {
    wait_never_kernel<<<1, 32, 0, s>>>(ws);
    return cudaGetLastError();
}

}  // namespace msa
