// Device-side check of the bounded waits every kernel relies on: a wait on
// an mbarrier that nothing will complete must give up after its time limit,
// report HISA_DEV_TIMEOUT in the status word and let the kernel return, so
// that the context stays usable.
#include "hisa_kernels.cuh"

namespace hisa {

namespace {

__global__ void __launch_bounds__(32) wait_probe_kernel(uint32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);          // one arrival expected; none ever comes
        fence_barrier_init();
        if (!mbar_wait(&bar, 0, nullptr)) set_status(status, HISA_DEV_TIMEOUT);
    }
    __syncwarp();
}

}  // namespace

cudaError_t launch_wait_probe(uint32_t* status, cudaStream_t s) {
    wait_probe_kernel<<<1, 32, 0, s>>>(status);
    return cudaGetLastError();
}

}  // namespace hisa
