// Failure-detection self-test: the bounded mbarrier wait of the kernels, run
// against a barrier that nothing completes, must give up after its limit,
// record ATFLASH_ERR_TIMEOUT in the device status word and let the kernel exit.
#include "internal.h"
#include "ptx.cuh"

namespace atf {
namespace {

__global__ void selftest_wait_kernel(int *status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival that never comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    WaitCtl wc{&abort_flag, status, limit_ns, 99};
    const bool ok = mbar_wait_warp(&bar, 0, wc);
    (void)ok;  // the timeout is recorded by the wait itself
}

}  // namespace

cudaError_t launch_selftest_wait(int *status, uint64_t limit_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace atf
