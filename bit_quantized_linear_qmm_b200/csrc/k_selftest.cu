// k_selftest.cu -- a self-test of the library's bounded-wait path.
//
// Every pipeline in this library waits on mbarriers with a time limit; when a
// limit runs out the kernel sets the timeout bit of the device status word
// and returns, so that qlin_get_device_status() reports QLIN_ERR_TIMEOUT and
// the context stays usable.  This kernel makes such a wait run out on purpose:
// it waits on an mbarrier that nothing ever arrives on, for `limit_ns` of
// %globaltimer, then records the timeout and returns.  Nothing faults and
// nothing is left in flight.
#include "qlin_common.cuh"

namespace qlin {
namespace {

__global__ void wait_timeout_kernel(unsigned* status, unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0)
        return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    // phase 0 of `bar` never completes: no thread arrives on it
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(&bar, 0)) {
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(status, kStatusTimeout);
            break;
        }
    }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, cudaStream_t st, const DeviceInfo& dev)
{
    wait_timeout_kernel<<<1, 32, 0, st>>>(dev.status, limit_ns);
    return cudaGetLastError();
}

}  // namespace qlin
