// Self-test of the bounded-wait error path that every kernel with
// asynchronous copies relies on: one thread waits, with a short limit, on a
// shared-memory mbarrier that nothing arrives on.  The wait must give up
// after the limit and set the timeout bit of the device error word, with the
// CUDA context left usable.  No fault, trap or unbounded loop is involved.
#include "dcn_device.h"
#include "dcn_launch.h"
#include "dcn_tma.cuh"

namespace dcnb {
namespace {

__global__ void bounded_wait_selftest(unsigned long long limit_ns, unsigned int *err) {
    __shared__ __align__(8) unsigned long long bar;
    const uint32_t a = smem_u32(&bar);
    mbar_init(a, 1);
    fence_mbar_init();
    if (!mbar_wait_bounded(a, 0, limit_ns)) atomicOr(err, kDevErrTmaTimeout);
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(long long limit_ns, cudaStream_t stream) {
    const DeviceInfo *dev = device_info();
    if (!dev) return cudaErrorNotSupported;
    bounded_wait_selftest<<<1, 1, 0, stream>>>((unsigned long long)limit_ns, dev->err);
    return cudaGetLastError();
}

}  // namespace dcnb
