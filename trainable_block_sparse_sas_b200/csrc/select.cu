// select.cu -- score-row LSE and exact hard Top-K (one CTA per score row).
//
// Gate normaliser: log g_m = s_m - LSE(s) over the row's history blocks
// (jaehun.me review of SAS, section 4.2.2, "Gate activation").  Selection: the K
// largest scores (jaehun.me review, Background Eq. 3; walkthrough Step 3), found
// without sorting by locating the K-th largest value as a threshold (the
// sort-free "gate threshold" Top-K of the shibing624 review, method section, last
// paragraph).  The threshold comes from an MSB-first radix select over
// order-preserving 32-bit keys (4 passes of 8 bits, shared-memory histograms);
// entries equal to the threshold are taken lowest index first, which is the tie
// rule, and the chosen blocks are compacted in index order (contiguous segments
// per thread, one block scan), so the list comes out ascending.
#include "common.cuh"
#include "kernels.h"
#include "topk_filter.cuh"

namespace sas {
namespace {

constexpr int kThreads = 256;

// history blocks of score row `row`: ctx_len gives the decode rows' length, else
// training row r (query block r) has r history blocks; at most row_len
__device__ __forceinline__ int history_len(long row, int n_kv_heads, int n_rows, int row_len,
                                           const int32_t* ctx_len, int block_size) {
    const int r = (int)(row % n_rows);
    int c;
    if (ctx_len) {
        const int b = (int)(row / n_rows) / n_kv_heads;
        const int T = ctx_len[b];
        c = T >= 1 ? (T - 1) / block_size : 0;
    } else {
        c = r;
    }
    return min(c, row_len);
}

// the row's score LSE (whole CTA)
__device__ void row_lse(const float* srow, int c, float* dst, float* red) {
    const int tid = threadIdx.x, nt = blockDim.x;
    float mx = -INFINITY;
    for (int m = tid; m < c; m += nt) mx = fmaxf(mx, srow[m]);
    mx = block_max(mx, red);
    float acc = 0.f;
    for (int m = tid; m < c; m += nt) acc += expf(srow[m] - mx);
    acc = block_sum(acc, red);
    if (tid == 0) *dst = c > 0 ? mx + logf(acc) : -INFINITY;
}


// Radix select of the K (< c) largest of srow[0 .. c) (global or shared memory),
// written to out[0 .. K) in ascending index order.  Called by every thread of a
// kThreads CTA.
__device__ void radix_select_row(const float* srow, int c, int top_k, int32_t* out, int* hist, int* scan,
                                 int* sh_bin_above) {
    const int tid = threadIdx.x, nt = blockDim.x;
    // Radix select of the K-th largest key.  `remaining` counts how many of the
    // keys that match the prefix found so far still have to be taken.
    uint32_t prefix = 0u, pmask = 0u;
    int remaining = top_k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < 256; i += nt) hist[i] = 0;
        __syncthreads();
        for (int m0 = 0; m0 < c; m0 += nt) {
            // one shared-memory atomic per distinct bin in the warp (scores crowd into
            // few top-byte bins, so per-lane atomics would serialise)
            const int m = m0 + tid;
            int bin = -1;
            if (m < c) {
                const uint32_t key = order_key(srow[m]);
                if ((key & pmask) == prefix) bin = (int)((key >> shift) & 255u);
            }
            const unsigned same = __match_any_sync(0xffffffffu, bin);
            if (bin >= 0 && (tid & 31) == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
        }
        __syncthreads();
        if (tid < 32) {
            // lane l scans bins 255-8l down to 248-8l (descending key order)
            int cnt[8], sum = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                cnt[q] = hist[255 - (tid * 8 + q)];
                sum += cnt[q];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += y;
            }
            const int excl = incl - sum;
            if (excl < remaining && remaining <= incl) {
                int acc = excl;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if (acc + cnt[q] >= remaining) {
                        sh_bin_above[0] = 255 - (tid * 8 + q);
                        sh_bin_above[1] = acc;
                        break;
                    }
                    acc += cnt[q];
                }
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sh_bin_above[0] << shift;
        pmask |= 0xFFu << shift;
        remaining -= sh_bin_above[1];
        __syncthreads();
    }
    // `prefix` is now the K-th largest key: every key above it is taken, and the
    // `remaining` lowest-index keys equal to it.  Compact in index order: thread
    // tid owns the contiguous segment [tid seg, (tid + 1) seg) of the row, counts
    // its keys above and equal to the threshold, and a block scan of those counts
    // (one scan of above << 16 | equal when both fit in 16 bits: fewer than K < 2^15
    // keys are above) gives every segment its output offset and the number of
    // equal keys before it.
    const int seg = (c + nt - 1) / nt;
    const int m_lo = min(c, tid * seg), m_hi = min(c, m_lo + seg);
    int gt = 0, eq = 0;
    for (int m = m_lo; m < m_hi; ++m) {
        const uint32_t key = order_key(srow[m]);
        gt += key > prefix ? 1 : 0;
        eq += key == prefix ? 1 : 0;
    }
    int tot, gt_before, eq_before;
    if (c < 65536 && top_k < 32768) {
        const int before = block_exclusive_scan((gt << 16) | eq, scan, &tot);
        gt_before = before >> 16;
        eq_before = before & 0xFFFF;
    } else {
        gt_before = block_exclusive_scan(gt, scan, &tot);
        eq_before = block_exclusive_scan(eq, scan, &tot);
    }
    int pos = gt_before + min(eq_before, remaining);
    int eq_seen = eq_before;
    for (int m = m_lo; m < m_hi && pos < top_k; ++m) {
        const uint32_t key = order_key(srow[m]);
        const bool is_eq = key == prefix;
        if (key > prefix || (is_eq && eq_seen < remaining)) out[pos++] = m;
        eq_seen += is_eq ? 1 : 0;
    }
}


__global__ void __launch_bounds__(kThreads)
    topk_select_kernel(const float* __restrict__ s, int n_kv_heads, int n_rows, int row_len,
                       const int32_t* __restrict__ ctx_len, int block_size, int top_k, int32_t* __restrict__ idx,
                       float* __restrict__ lse_s) {
    __shared__ int hist[256];
    __shared__ float red[33];
    __shared__ int scan[33];
    __shared__ int sh_bin_above[2];
    const long row = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int c = history_len(row, n_kv_heads, n_rows, row_len, ctx_len, block_size);
    const float* srow = s + row * (long)row_len;
    if (lse_s) row_lse(srow, c, lse_s + row, red);
    if (!idx || top_k == 0) return;
    int32_t* out = idx + row * (long)top_k;
    if (top_k >= c) {  // the budget covers the whole history
        for (int m = tid; m < top_k; m += nt) out[m] = m < c ? m : -1;
        return;
    }
    radix_select_row(srow, c, top_k, out, hist, scan, sh_bin_above);
}

// Rows of kFilterMin .. kFilterMax blocks with K <= 64: the row is staged in
// shared memory once and selected by a threshold filter instead of four radix
// passes.  Every thread keeps the two largest keys of its scores (m = tid + 256 u);
// warp 0 takes, per lane, the two largest of the eight warps' values for that
// lane, sorts the 64 (each a distinct score) and reads off the K-th largest, a
// lower bound tau of the K-th largest score; the scores at or above tau (K to a
// few more on random rows) are ranked exactly.  Over kCandCap candidates (rows
// with many equal scores) the radix select runs on the staged row.
constexpr int kFilterMin = 1024, kFilterMax = 16384;  // 16384 / 256 = 64 scores per thread: a 64-bit mask
constexpr int kCandCap = 512;

__global__ void __launch_bounds__(kThreads)
    topk_filter_kernel(const float* __restrict__ s, int n_kv_heads, int n_rows, int row_len,
                       const int32_t* __restrict__ ctx_len, int block_size, int top_k, int32_t* __restrict__ idx,
                       float* __restrict__ lse_s) {
    extern __shared__ float srow[];  // the row's first c scores
    __shared__ int hist[256];
    __shared__ float red[33];
    __shared__ int scan[33];
    __shared__ int sh_bin_above[2];
    __shared__ uint32_t tops[kThreads / 32][64];
    __shared__ unsigned long long cand[kCandCap];
    __shared__ unsigned long long chosen[64];
    __shared__ int misc[2];  // candidates, tau
    const long row = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int c = history_len(row, n_kv_heads, n_rows, row_len, ctx_len, block_size);
    const float* g = s + row * (long)row_len;
    for (int m = tid; m < c; m += nt) srow[m] = g[m];
    if (tid == 0) misc[0] = 0;
    __syncthreads();
    if (lse_s) row_lse(srow, c, lse_s + row, red);
    if (!idx || top_k == 0) return;
    int32_t* out = idx + row * (long)top_k;
    if (top_k >= c) {  // the budget covers the whole history
        for (int m = tid; m < top_k; m += nt) out[m] = m < c ? m : -1;
        return;
    }
    const int K = top_k;
    // the two largest keys of this thread's scores (two chains for overlap)
    uint32_t k1 = 0u, k2 = 0u, k1b = 0u, k2b = 0u;
    int m = tid;
    for (; m + nt < c; m += 2 * nt) {
        top2_insert(order_key(srow[m]), k1, k2);
        top2_insert(order_key(srow[m + nt]), k1b, k2b);
    }
    if (m < c) top2_insert(order_key(srow[m]), k1, k2);
    top2_insert(k1b, k1, k2);
    top2_insert(k2b, k1, k2);
    tops[warp][lane] = k1;
    tops[warp][32 + lane] = k2;
    __syncthreads();
    if (warp == 0) {
        uint32_t c1 = 0u, c2 = 0u;
#pragma unroll
        for (int w2 = 0; w2 < kThreads / 32; ++w2) {
            top2_insert(tops[w2][lane], c1, c2);
            top2_insert(tops[w2][32 + lane], c1, c2);
        }
        const uint32_t tau = warp_kth_of_64(c1, c2, K - 1);
        if (lane == 0) misc[1] = (int)tau;
    }
    __syncthreads();
    const uint32_t tau = (uint32_t)misc[1];
    // candidates: bit u of the mask for score tid + 256 u
    unsigned long long mask = 0ull;
    for (int u = 0, mm = tid; mm < c; ++u, mm += nt) mask |= order_key(srow[mm]) >= tau ? (1ull << u) : 0ull;
    const int cnt = __popcll(mask);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    int wbase = 0;
    if (lane == 31 && incl > 0) wbase = atomicAdd(&misc[0], incl);
    int pos = __shfl_sync(0xffffffffu, wbase, 31) + incl - cnt;
    while (mask) {
        const int u = __ffsll((long long)mask) - 1;
        mask &= mask - 1;
        const int mm = tid + u * nt;
        if (pos < kCandCap)
            cand[pos] = ((unsigned long long)order_key(srow[mm]) << 32) | (0xFFFFFFFFu - (uint32_t)mm);
        ++pos;
    }
    __syncthreads();
    const int C = misc[0];
    if (C > kCandCap) {  // many equal scores: the radix select on the staged row
        radix_select_row(srow, c, top_k, out, hist, scan, sh_bin_above);
        return;
    }
    const unsigned long long* pick = cand;  // exactly K candidates: all are chosen
    if (C > K) {
        for (int j = tid; j < C; j += nt) {
            const unsigned long long k = cand[j];
            const int rk = count_larger(cand, C, k);
            if (rk < K) chosen[rk] = k;
        }
        __syncthreads();
        pick = chosen;
    }
    for (int j = tid; j < K; j += nt) {  // ascending block order
        const uint32_t mj = 0xFFFFFFFFu - (uint32_t)(pick[j] & 0xFFFFFFFFull);
        int p = 0;
        for (int j2 = 0; j2 < K; ++j2) p += (0xFFFFFFFFu - (uint32_t)(pick[j2] & 0xFFFFFFFFull)) < mj ? 1 : 0;
        out[p] = (int32_t)mj;
    }
}

}  // namespace

cudaError_t launch_topk_select(const float* s, int batch, int n_kv_heads, int n_rows, int row_len,
                               const int32_t* ctx_len, int block_size, int top_k, int32_t* idx, float* lse_s,
                               cudaStream_t stream) {
    const long rows = (long)batch * n_kv_heads * n_rows;
    if (rows == 0) return cudaSuccess;
    if (rows > 0x7fffffffL) return cudaErrorInvalidValue;
    if (row_len >= kFilterMin && row_len <= kFilterMax && top_k <= 64) {
        const size_t smem = 4 * (size_t)row_len;
        static size_t smem_set[64] = {};  // per device: raise the limit once, not on the steady path
        int dev = 0;
        cudaError_t err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        if (dev < 0 || dev >= 64 || smem > smem_set[dev]) {
            err = cudaFuncSetAttribute(topk_filter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (err != cudaSuccess) return err;
            if (dev >= 0 && dev < 64) smem_set[dev] = smem;
        }
        topk_filter_kernel<<<(unsigned)rows, kThreads, smem, stream>>>(s, n_kv_heads, n_rows, row_len, ctx_len,
                                                                        block_size, top_k, idx, lse_s);
    } else {
        topk_select_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(s, n_kv_heads, n_rows, row_len, ctx_len,
                                                                    block_size, top_k, idx, lse_s);
    }
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace sas
