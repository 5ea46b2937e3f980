// selftest.cu -- exercises the failure path of the bounded device-side waits
// without a fault: one thread waits on an mbarrier that nothing ever arrives
// at, gives up after the given limit exactly as the tensor-core kernels do, and
// records the timeout in the device status word.
#include "kernels.h"
#include "sm100.cuh"

namespace sas {
namespace {

__global__ void selftest_wait_kernel(int* status, unsigned long long limit_ns) {
    __shared__ __align__(8) unsigned long long bar;
    const uint32_t b = sm100::smem_u32(&bar);
    sm100::mbar_init(b, 1);
    sm100::fence_barrier_init();
    const unsigned long long t0 = sm100::globaltimer();
    while (!sm100::mbar_try_wait(b, 0)) {  // no thread ever arrives
        if (sm100::globaltimer() - t0 > limit_ns) {
            atomicExch(status, sm100::kStatusTimeout);
            break;
        }
    }
}

}  // namespace

cudaError_t launch_selftest_wait(int* status, unsigned long long limit_ns, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 1, 0, stream>>>(status, limit_ns);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace sas
