// selftest.cu -- runs the failure path of the tensor-core kernels without a
// fault.  The roles and calls are those of the attention kernels: one warp
// allocates tensor memory; one thread issues a tcgen05 MMA, commits it, and then
// waits through sm100::mbar_wait on an mbarrier that nothing ever arrives at; a
// second warp waits through sm100::warp_wait on another such barrier.  The
// first wait gives up after the given limit, sets the CTA's abort flag and the
// caller's status word; the second wait sees the flag and leaves; the issuing
// thread drains its MMAs through sm100::mbar_wait_drain; the tensor memory is
// freed.  Each phase reached is recorded in `trace`.
#include "kernels.h"
#include "sm100.cuh"

namespace sas {
namespace {

using namespace sm100;

constexpr int kThreads = 96;
constexpr uint32_t kA = 128 * 128;  // A tile: 128 rows x 128 B (64 bf16), 128-byte swizzle
constexpr uint32_t kB = 64 * 128;   // B tile: 64 rows x 128 B

__device__ __forceinline__ void mark(int* trace, int phase) {
    if (trace) trace[phase] = 1;
}

__global__ void __launch_bounds__(kThreads, 1) selftest_wait_kernel(int* status, int* trace,
                                                                    unsigned long long limit_ns) {
    __shared__ __align__(1024) uint8_t tiles[kA + kB];
    __shared__ __align__(8) unsigned long long bars[4];  // never_a, never_b, mma_done, drain
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_word;
    volatile int* abort_flag = &abort_word;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t never_a = smem_u32(&bars[0]), never_b = smem_u32(&bars[1]);
    const uint32_t mma_done = smem_u32(&bars[2]), drain = smem_u32(&bars[3]);

    for (int i = threadIdx.x; i < (int)((kA + kB) / 16); i += kThreads)
        reinterpret_cast<uint4*>(tiles)[i] = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // zeros visible to the tensor core
    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bars[i]), 1);
        abort_word = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&tmem_slot), 64);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp == 1) {
        if (lane == 0) {
            // the MMA issuer: one MMA in flight, then the wait that never completes
            const uint32_t sa = smem_u32(tiles), sb = sa + kA;
            mma_ss(tmem, sdesc_sw128(sa, 16, 1024), sdesc_sw128(sb, 16, 1024), idesc_bf16_f32(128, 64, false, false),
                   0u);
            mma_commit(mma_done);
            const bool ok = mbar_wait(never_a, 0, abort_flag, status, limit_ns);
            if (!ok && *abort_flag) mark(trace, 0);
            // all issued MMAs complete before the tensor memory is released
            mma_commit(drain);
            if (mbar_wait_drain(drain, 0, status, limit_ns)) mark(trace, 2);
        }
        __syncwarp();  // the warp reaches the CTA barrier converged
    } else if (warp == 2) {
        // another role waiting on its own barrier, with a longer limit: it must
        // leave on the abort flag, before its own limit runs out
        const unsigned long long t0 = globaltimer();
        const bool ok = warp_wait(never_b, 0, abort_flag, status, 4 * limit_ns);
        if (!ok && lane == 0 && globaltimer() - t0 < 4 * limit_ns) mark(trace, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
        if (lane == 0) mark(trace, 3);
    }
}

__global__ void trace_clear_kernel(int* trace) {
    if (threadIdx.x < 4) trace[threadIdx.x] = 0;
}

}  // namespace

cudaError_t launch_selftest_wait(int* status, int* trace, unsigned long long limit_ns, cudaStream_t stream) {
    // trace is optional: without it the phases are not recorded
    if (trace) {
        trace_clear_kernel<<<1, 32, 0, stream>>>(trace);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
        count_launch();
    }
    selftest_wait_kernel<<<1, kThreads, 0, stream>>>(status, trace, limit_ns);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace sas
