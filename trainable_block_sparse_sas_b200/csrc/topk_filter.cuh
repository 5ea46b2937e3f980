// topk_filter.cuh -- warp-level pieces of the threshold-filter Top-K shared by
// the standalone selection (select.cu) and the fused decode (decode_sm100.cu):
// the two largest of a stream of 32-bit order keys, the p-th largest of 64 keys
// held two per lane, and the rank of a unique 64-bit key among candidates.
// A lower bound tau of a row's K-th largest score is the K-th largest of any K
// distinct scores of the row; every score at or above it is a candidate, and the
// candidates ranked on (order key << 32 | (2^32 - 1 - index)) give the exact
// Top-K with ties to the lower index (jaehun.me review of SAS, Background Eq. 3;
// walkthrough Step 3).
#pragma once

#include <stdint.h>

namespace sas {

__device__ __forceinline__ void top2_insert(uint32_t k, uint32_t& k1, uint32_t& k2) {
    const uint32_t lo = min(k, k1);
    k1 = max(k, k1);
    k2 = max(k2, lo);
}

// 64 keys, two per lane (position lane and 32 + lane), sorted descending by a
// bitonic network; every lane gets the key at sorted position p.
__device__ __forceinline__ uint32_t warp_kth_of_64(uint32_t x0, uint32_t x1, int p) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 32) {  // partners in the same lane (k = 64: the whole sequence descends)
                const uint32_t hi = max(x0, x1), lo = min(x0, x1);
                x0 = hi;
                x1 = lo;
            } else {
                const uint32_t y0 = __shfl_xor_sync(0xffffffffu, x0, j);
                const uint32_t y1 = __shfl_xor_sync(0xffffffffu, x1, j);
                const bool lower = (lane & j) == 0;
                const bool desc0 = (lane & k) == 0, desc1 = ((lane + 32) & k) == 0;
                x0 = (lower == desc0) ? max(x0, y0) : min(x0, y0);
                x1 = (lower == desc1) ? max(x1, y1) : min(x1, y1);
            }
        }
    }
    const uint32_t v0 = __shfl_sync(0xffffffffu, x0, p & 31), v1 = __shfl_sync(0xffffffffu, x1, p & 31);
    return p < 32 ? v0 : v1;
}

// rank of k among the first C candidates: how many are larger (four independent sums)
__device__ __forceinline__ int count_larger(const unsigned long long* cand, int C, unsigned long long k) {
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0, j = 0;
    for (; j + 4 <= C; j += 4) {
        r0 += cand[j] > k ? 1 : 0;
        r1 += cand[j + 1] > k ? 1 : 0;
        r2 += cand[j + 2] > k ? 1 : 0;
        r3 += cand[j + 3] > k ? 1 : 0;
    }
    for (; j < C; ++j) r0 += cand[j] > k ? 1 : 0;
    return r0 + r1 + r2 + r3;
}

}  // namespace sas
