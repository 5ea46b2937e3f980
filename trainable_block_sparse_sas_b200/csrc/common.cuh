// common.cuh -- small device helpers shared by the libsas kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sas {

// Index checks of the debug-bounds build (compiled with -DSAS_DEBUG_BOUNDS): a
// global-memory index the kernel computed is compared with the extent the
// problem shape gives its buffer; an index outside it records
// SAS_ERR_DEVICE_BOUNDS (6) and the source line (bits 8 and up) in the caller's
// device status word -- the first failure wins -- and the access is skipped.
// Nothing traps.  Release builds compile every check to `true`.
constexpr int kStatusBounds = 6;
#ifdef SAS_DEBUG_BOUNDS
__device__ __noinline__ inline bool bounds_fail(int* status, int line) {
    if (status) atomicCAS(status, 0, kStatusBounds | (line << 8));
    return false;
}
#define SAS_IN_BOUNDS(i, n, status) \
    (((long long)(i) >= 0 && (long long)(i) < (long long)(n)) || ::sas::bounds_fail((status), __LINE__))
#else
#define SAS_IN_BOUNDS(i, n, status) ((void)(i), (void)(n), (void)(status), true)
#endif

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Block-wide reductions for blockDim.x a multiple of 32 (<= 1024).  `red` is
// shared scratch of >= 33 floats.  Every thread gets the result.
__device__ __forceinline__ float block_sum(float v, float* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    if (wid == 0) {
        float x = lane < nw ? red[lane] : 0.f;
        x = warp_sum(x);
        if (lane == 0) red[32] = x;
    }
    __syncthreads();
    return red[32];
}

__device__ __forceinline__ float block_max(float v, float* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_max(v);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    if (wid == 0) {
        float x = lane < nw ? red[lane] : -INFINITY;
        x = warp_max(x);
        if (lane == 0) red[32] = x;
    }
    __syncthreads();
    return red[32];
}

// Exclusive prefix sum over the block of one int per thread; returns the
// thread's exclusive prefix and writes the block total to *total.
// `scan` is shared scratch of >= 33 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scan, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) scan[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int w = lane < nw ? scan[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < nw) scan[lane] = w;  // inclusive warp totals
        if (lane == 31) scan[32] = w;
    }
    __syncthreads();
    int warp_off = wid > 0 ? scan[wid - 1] : 0;
    *total = scan[32];
    return warp_off + x - v;
}

// Order-preserving map of a finite float onto uint32 (larger float -> larger
// key).  -0.0 is folded onto +0.0 first so that the two compare equal.
__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace sas
