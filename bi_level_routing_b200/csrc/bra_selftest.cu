// bra_selftest.cu -- a check of the bounded wait every pipelined kernel of the library relies on:
// a kernel that waits on an mbarrier nothing will ever complete, through the same mbar_wait, with a
// short limit. The wait gives up, sets kErrTimeout in the device error word and the kernel returns;
// nothing (no TMA load, no MMA, no other thread) is in flight when it does, and the context stays
// usable. bra_check_device_error then reports BRA_ERR_TIMEOUT. Nothing of the BRA computation runs.
#include "bra_device.cuh"
#include "bra_launch.h"

namespace bra {

__global__ void __launch_bounds__(32) wait_timeout_kernel(unsigned *err, unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);  // one arrival expected; none will come
    mbar_fence_init();
    mbar_wait(&bar, 0, err, limit_ns);  // gives up after limit_ns and sets kErrTimeout in *err
}

cudaError_t launch_wait_timeout(unsigned *err, unsigned long long limit_ns, cudaStream_t stream)
{
    wait_timeout_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace bra
