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
// rule, and the chosen blocks are compacted in index order, so the list comes
// out ascending.
#include "common.cuh"
#include "kernels.h"

namespace sas {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    topk_select_kernel(const float* __restrict__ s, int n_kv_heads, int n_rows, int row_len,
                       const int32_t* __restrict__ ctx_len, int block_size, int top_k, int32_t* __restrict__ idx,
                       float* __restrict__ lse_s) {
    __shared__ int hist[256];
    __shared__ float red[33];
    __shared__ int scan[33];
    __shared__ int sh_bin, sh_above;

    const long row = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int r = (int)(row % n_rows);
    const int b = (int)(row / n_rows) / n_kv_heads;
    int c;
    if (ctx_len) {
        const int T = ctx_len[b];
        c = T >= 1 ? (T - 1) / block_size : 0;
    } else {
        c = r;
    }
    c = min(c, row_len);
    const float* srow = s + row * (long)row_len;

    if (lse_s) {
        float mx = -INFINITY;
        for (int m = tid; m < c; m += nt) mx = fmaxf(mx, srow[m]);
        mx = block_max(mx, red);
        float acc = 0.f;
        for (int m = tid; m < c; m += nt) acc += expf(srow[m] - mx);
        acc = block_sum(acc, red);
        if (tid == 0) lse_s[row] = c > 0 ? mx + logf(acc) : -INFINITY;
    }
    if (!idx || top_k == 0) return;
    int32_t* out = idx + row * (long)top_k;
    if (top_k >= c) {  // the budget covers the whole history
        for (int m = tid; m < top_k; m += nt) out[m] = m < c ? m : -1;
        return;
    }

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
                        sh_bin = 255 - (tid * 8 + q);
                        sh_above = acc;
                        break;
                    }
                    acc += cnt[q];
                }
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sh_bin << shift;
        pmask |= 0xFFu << shift;
        remaining -= sh_above;
        __syncthreads();
    }
    // `prefix` is now the K-th largest key: every key above it is taken, and the
    // `remaining` lowest-index keys equal to it.  Compact in index order.
    int base_out = 0, eq_seen = 0;
    for (int m0 = 0; m0 < c; m0 += nt) {
        const int m = m0 + tid;
        const uint32_t key = m < c ? order_key(srow[m]) : 0u;
        const int is_eq = (m < c && key == prefix) ? 1 : 0;
        int tot_eq;
        const int eq_rank = block_exclusive_scan(is_eq, scan, &tot_eq) + eq_seen;
        const int take = (m < c && (key > prefix || (is_eq && eq_rank < remaining))) ? 1 : 0;
        int tot_take;
        const int pos = block_exclusive_scan(take, scan, &tot_take) + base_out;
        if (take && pos < top_k) out[pos] = m;
        eq_seen += tot_eq;
        base_out += tot_take;
    }
}

}  // namespace

cudaError_t launch_topk_select(const float* s, int batch, int n_kv_heads, int n_rows, int row_len,
                               const int32_t* ctx_len, int block_size, int top_k, int32_t* idx, float* lse_s,
                               cudaStream_t stream) {
    const long rows = (long)batch * n_kv_heads * n_rows;
    if (rows == 0) return cudaSuccess;
    if (rows > 0x7fffffffL) return cudaErrorInvalidValue;
    topk_select_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(s, n_kv_heads, n_rows, row_len, ctx_len, block_size,
                                                                top_k, idx, lse_s);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace sas
