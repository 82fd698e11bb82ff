// selftest.cu -- a kernel that exercises the bounded mbarrier wait's give-up
// path: it waits on a barrier that nothing ever arrives at, so the wait must
// run out, set the abort flag and OR PKV_STATUS_WAIT_TIMEOUT into the status
// word, and the kernel must return. Used by the tests of the failure path.
#include "device_utils.cuh"
#include "launch.h"

namespace pkv {
namespace {

__global__ void bounded_wait_selftest_kernel(int32_t *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 never completes: no thread arrives on `bar`
        const bool ok = mbar_wait_bounded(&bar, 0u, &abort_flag, status);
        if (ok || !abort_flag) atomicOr(status, 0x40000000);  // the wait must not succeed
    }
}

}  // namespace

cudaError_t selftest_bounded_wait_launch(int32_t *status, cudaStream_t stream) {
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status);
    return cudaGetLastError();
}

}  // namespace pkv
