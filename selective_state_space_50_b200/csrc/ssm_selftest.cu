// Self-test of the failure path of the bounded waits: a kernel waits on an
// mbarrier that nothing will complete, with a budget of about a millisecond;
// the wait gives up, sets the device error word and the kernel returns.  No
// fault, trap or hang is involved: this is the same bounded wait the TMA
// kernels use, made to run out on purpose.

#include "ssm_internal.h"
#include "ssm_tma.cuh"

namespace ssm {
namespace {

__global__ void wait_timeout_kernel(int *err, long long budget) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);       // one arrival expected; none comes
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, err, budget);
}

}  // namespace
}  // namespace ssm

extern "C" ssm_status_t ssm_selftest_wait_timeout(void *stream) {
    int *err = ssm::device_error_word();
    if (!err) return ssm::set_last_error(SSM_ERR_CUDA, "ssm_selftest_wait_timeout: no device error word");
    // about 1 ms at 2 GHz
    ssm::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, 1LL << 21);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return ssm::set_last_error(SSM_ERR_CUDA, cudaGetErrorString(e));
    return ssm::set_last_error(SSM_OK, "");
}
