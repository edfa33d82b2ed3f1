// Failure-path self-test: a bounded wait that is made to run out.
//
// One warp waits, through the same mbar_wait every pipeline uses, on an
// mbarrier that nothing will ever complete, with a short limit.  The wait
// gives up, records MLXQ_STATUS_TIMEOUT in the library's device status word
// and the kernel returns normally: nothing faults, traps or hangs, and the
// context stays usable.  The host reads the status with mlxq_device_status.
#include "device_common.cuh"
#include "kernels.h"

namespace mlxq {
namespace {

__global__ void __launch_bounds__(32, 1) k_wait_never_completes(unsigned int* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);  // one arrival expected; none is ever made
        mbar_fence_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, status, limit_ns);
    __syncwarp();
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, cudaStream_t stream) {
    k_wait_never_completes<<<1, 32, 0, stream>>>(device_status_ptr(), limit_ns);
    return cudaGetLastError();
}

}  // namespace mlxq
