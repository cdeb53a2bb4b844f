// Failure-detection self-test: a wait that nothing satisfies.  The kernel's one
// thread waits on a fresh mbarrier with the library's bounded wait; when the wait
// limit passes it records MXFP4_ERR_TIMEOUT in the device status word and returns,
// which is how every kernel of the library reports a stalled pipeline.  Nothing
// faults, traps or hangs, so the context stays usable afterwards.
#include "common.cuh"
#include "internal.h"

namespace mx {

namespace {

__global__ void selftest_wait_timeout_kernel(unsigned* status) {
    __shared__ uint64_t bar;
    __shared__ int never;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);     // expects one arrival; none is ever made
    never = 0;
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, &never)) record_status(status, MXFP4_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_selftest_wait_timeout(unsigned* status, cudaStream_t stream) {
    selftest_wait_timeout_kernel<<<1, 32, 0, stream>>>(status);
    return cudaGetLastError();
}

}  // namespace mx
