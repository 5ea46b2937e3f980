// scorer.cu -- the parameter-free pooled-key selector scorer.
//
// SAS's selector scores a query against per-block key summaries built by
// pooling (jaehun.me review, walkthrough Step 1; Limitations: pooling-based block
// summaries); its trained weights are not given, so this is the weight-free form:
// mean pooling on both sides.
//
// Training shape (one score row per kv head and query block):
//   qbar[b,h,c] = mean of q over the b tokens of block c and the G query heads
//                 of group h;  kbar[b,h,m] = mean of k over block m's tokens;
//   s[b,h,c,m]  = sigma qbar[b,h,c] . kbar[b,h,m] for m < c, 0 for m >= c.
//   pool_train_kernel: one CTA per (b, block, kv head), 16-byte loads over the
//     block's rows, fp32 sums: a single pass over q and k, bound by HBM.
//   pool_scores_kernel: 64 x 64 tiles of the strictly lower triangle in fp32 on
//     the CUDA cores, 4 x 4 outputs per thread (Cq^2 d / 2 FMAs per head: small
//     next to the pooling pass).
//
// Decode shape:
//   pool_keys_kernel: ksum[b,h,m] = mean of the cache's block m (full blocks in
//     [m0, m1)), stored in the cache's dtype, for a summary cache kept next to
//     the KV cache and extended as blocks fill.
//   decode_scores_kernel: s[b,h,m] = sigma qbar[b,h] . ksum[b,h,m] for the full
//     history blocks m < (ctx_len - 1) / b, 0 up to s_cols; qbar = mean over the
//     group's heads.  One warp per block summary, lanes across d (coalesced rows),
//     four summaries in flight per warp: bound by reading the summaries.

#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace sas {
namespace {

constexpr int kPoolThreads = 128;

// 16-byte vector of T
template <typename T>
struct Vec {
    static constexpr int N = 16 / sizeof(T);
};

template <typename T>
__device__ __forceinline__ void add_vec(float* acc, const uint4 x);
template <>
__device__ __forceinline__ void add_vec<__nv_bfloat16>(float* acc, const uint4 x) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
    }
}
template <>
__device__ __forceinline__ void add_vec<float>(float* acc, const uint4 x) {
    acc[0] += __uint_as_float(x.x);
    acc[1] += __uint_as_float(x.y);
    acc[2] += __uint_as_float(x.z);
    acc[3] += __uint_as_float(x.w);
}

// Sum of `rows` rows of `span` elements (row r at base + r * stride, 16-byte
// aligned), folded over `fold` equal parts of the span (the G heads of a query
// row): out[e] = sum_r sum_f row_r[f * (span / fold) + e], e < span / fold.
// All NT threads of the CTA take part; red is shared scratch of NT * 8 floats;
// the result is written by threads e < span / fold.
template <typename T, int NT = kPoolThreads>
__device__ __forceinline__ void pool_rows(const T* base, long stride, int rows, int span, int fold, float* red,
                                          float scale, float* out) {
    constexpr int V = Vec<T>::N;
    const int nv = span / V;                    // vectors per row
    const int rg = NT / nv;                     // rows in flight; threads from rg * nv on idle
    const int tid = threadIdx.x;
    const int r0 = tid / nv, v = tid % nv;
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    if (r0 < rg) {
#pragma unroll 4
        for (int r = r0; r < rows; r += rg) {
            const uint4 x = *reinterpret_cast<const uint4*>(base + r * stride + v * V);
            add_vec<T>(acc, x);
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < V; ++i) red[tid * V + i] = acc[i];
    __syncthreads();
    const int part = span / fold;
    for (int e = tid; e < part; e += NT) {
        float s = 0.f;
        for (int f = 0; f < fold; ++f) {
            const int el = f * part + e;  // element of the span
            const int vv = el / V, ii = el % V;
            for (int g = 0; g < rg; ++g) s += red[(g * nv + vv) * V + ii];
        }
        out[e] = s * scale;
    }
    __syncthreads();
}

// NT threads per (b, block, kv head): 64 when a query row's G heads fit in 64
// 16-byte vectors, so that every CTA of a training problem is resident at once
template <typename T, int NT>
__global__ void __launch_bounds__(NT) pool_train_kernel(const T* __restrict__ q, const T* __restrict__ k, int n, int Hq,
                                                        int Hkv, int d, int bs, int Cq, float* __restrict__ qbar,
                                                        float* __restrict__ kbar) {
    __shared__ float red[NT * 8];
    const int h = (int)(blockIdx.x % Hkv);
    const int c = (int)((blockIdx.x / Hkv) % Cq);
    const int b = (int)(blockIdx.x / ((long)Hkv * Cq));
    const int G = Hq / Hkv;
    const long row0 = (long)b * n + (long)c * bs;
    const long u = ((long)b * Hkv + h) * Cq + c;
    pool_rows<T, NT>(q + (row0 * Hq + (long)h * G) * d, (long)Hq * d, bs, G * d, G, red, 1.f / (float)(bs * G),
                     qbar + u * d);
    pool_rows<T, NT>(k + (row0 * Hkv + h) * d, (long)Hkv * d, bs, d, 1, red, 1.f / (float)bs, kbar + u * d);
}

constexpr int kTile = 64;   // output tile (query blocks x key blocks)
constexpr int kTileE = 32;  // head-dim chunk staged in shared memory

// s[b,h,c,m] for one 64 x 64 tile; 256 threads, a 4 x 4 register tile each
// (rows ty + 16 i, columns tx + 16 j), so a thread reads 8 shared values per 16 FMAs
__global__ void __launch_bounds__(256) pool_scores_kernel(const float* __restrict__ qbar,
                                                          const float* __restrict__ kbar, int Cq, int d, float sigma,
                                                          float* __restrict__ s) {
    __shared__ float qs[kTile][kTileE + 1], ks[kTile][kTileE + 1];
    const int tiles = (Cq + kTile - 1) / kTile;
    const int tc = (int)(blockIdx.x % tiles), tm = (int)((blockIdx.x / tiles) % tiles);
    const long bh = blockIdx.x / ((long)tiles * tiles);
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    const int c0 = tc * kTile, m0 = tm * kTile;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    if (m0 < c0 + kTile - 1) {  // the tile holds some m < c
        const float* qb = qbar + bh * Cq * d;
        const float* kb = kbar + bh * Cq * d;
        for (int e0 = 0; e0 < d; e0 += kTileE) {
            // 64 rows x 32 columns of each side: 8 elements per thread, coalesced rows
            for (int idx = tid; idx < kTile * kTileE; idx += 256) {
                const int r = idx / kTileE, e = e0 + idx % kTileE;
                qs[r][idx % kTileE] = (c0 + r < Cq && e < d) ? qb[(long)(c0 + r) * d + e] : 0.f;
                ks[r][idx % kTileE] = (m0 + r < Cq && e < d) ? kb[(long)(m0 + r) * d + e] : 0.f;
            }
            __syncthreads();
#pragma unroll 8
            for (int e = 0; e < kTileE; ++e) {
                float qv[4], kv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) qv[i] = qs[ty + 16 * i][e];
#pragma unroll
                for (int j = 0; j < 4; ++j) kv[j] = ks[tx + 16 * j][e];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
            }
            __syncthreads();
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + ty + 16 * i, m = m0 + tx + 16 * j;
            if (c < Cq && m < Cq) s[(bh * Cq + c) * Cq + m] = m < c ? sigma * acc[i][j] : 0.f;
        }
}

// ksum[b,h,m] = mean of the cache block m, m in [m0, m1); one CTA per (b, h, m)
template <typename T>
__global__ void __launch_bounds__(kPoolThreads) pool_keys_kernel(const T* __restrict__ kc, int Hkv, int Tmax, int d,
                                                                 int bs, int m0, int nblk, int nsum,
                                                                 T* __restrict__ ksum) {
    __shared__ float red[kPoolThreads * 8];
    __shared__ float mean[256];
    const long bh = blockIdx.x / nblk;
    const int m = m0 + (int)(blockIdx.x % nblk);
    pool_rows<T>(kc + (bh * Tmax + (long)m * bs) * d, d, bs, d, 1, red, 1.f / (float)bs, mean);
    // pool_rows ends with a barrier: the means are visible to every thread
    for (int e = threadIdx.x; e < d; e += kPoolThreads) ksum[(bh * nsum + m) * d + e] = from_f32<T>(mean[e]);
}

// The same over a paged pool [num_pages, b, Hkv, d]: block m of sequence b is the
// page page_table[b * pps + m]; a page id outside the pool gives a zero summary
template <typename T>
__global__ void __launch_bounds__(kPoolThreads) pool_keys_paged_kernel(const T* __restrict__ kp,
                                                                       const int32_t* __restrict__ table, int pps,
                                                                       int num_pages, int Hkv, int d, int bs, int m0,
                                                                       int nblk, int nsum, T* __restrict__ ksum) {
    __shared__ float red[kPoolThreads * 8];
    __shared__ float mean[256];
    const long bh = blockIdx.x / nblk;
    const int m = m0 + (int)(blockIdx.x % nblk);
    const int b = (int)(bh / Hkv), h = (int)(bh % Hkv);
    const int page = table[(long)b * pps + m];
    if (page < 0 || page >= num_pages) {
        for (int e = threadIdx.x; e < d; e += kPoolThreads) ksum[(bh * nsum + m) * d + e] = from_f32<T>(0.f);
        return;
    }
    pool_rows<T>(kp + ((long)page * bs * Hkv + h) * d, (long)Hkv * d, bs, d, 1, red, 1.f / (float)bs, mean);
    for (int e = threadIdx.x; e < d; e += kPoolThreads) ksum[(bh * nsum + m) * d + e] = from_f32<T>(mean[e]);
}

// EPL consecutive elements (2 or 4) as floats, one vector load
template <typename T, int EPL>
__device__ __forceinline__ void load_lane(const T* p, float* x) {
    if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(p);
        if constexpr (EPL == 4) {
            const uint2 u = *reinterpret_cast<const uint2*>(p);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
            x[0] = a.x;
            x[1] = a.y;
            x[2] = b.x;
            x[3] = b.y;
        } else {
            const float2 a = __bfloat1622float2(*h);
            x[0] = a.x;
            x[1] = a.y;
        }
    } else {
        if constexpr (EPL == 4) {
            const float4 u = *reinterpret_cast<const float4*>(p);
            x[0] = u.x;
            x[1] = u.y;
            x[2] = u.z;
            x[3] = u.w;
        } else {
            const float2 u = *reinterpret_cast<const float2*>(p);
            x[0] = u.x;
            x[1] = u.y;
        }
    }
}

constexpr int kScoreThreads = 256;
constexpr int kScoreChunk = 256;  // blocks per CTA

// s[b,h,m] for one chunk of blocks; D = 64 or 128 (lane = D / 32 elements)
template <typename T, int D>
__global__ void __launch_bounds__(kScoreThreads) decode_scores_kernel(const T* __restrict__ q,
                                                                      const T* __restrict__ ksum,
                                                                      const int32_t* __restrict__ ctx_len, int Hq,
                                                                      int Hkv, int bs, int nsum, int s_cols,
                                                                      float sigma, float* __restrict__ s) {
    constexpr int EPL = D / 32;
    __shared__ float qb[D];
    const int chunks = (s_cols + kScoreChunk - 1) / kScoreChunk;
    const long bh = blockIdx.x / chunks;
    const int m_begin = (int)(blockIdx.x % chunks) * kScoreChunk;
    const int b = (int)(bh / Hkv), h = (int)(bh % Hkv);
    const int G = Hq / Hkv;
    const int T_ = ctx_len[b];
    const int Cb = min(T_ > 0 ? (T_ - 1) / bs : 0, min(nsum, s_cols));
    for (int e = threadIdx.x; e < D; e += kScoreThreads) {
        float a = 0.f;
        for (int g = 0; g < G; ++g) a += to_f32<T>(q[((long)b * Hq + h * G + g) * D + e]);
        qb[e] = a * (sigma / (float)G);
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float ql[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) ql[i] = qb[EPL * lane + i];
    const int m_end = min(m_begin + kScoreChunk, s_cols);
    constexpr int kW = kScoreThreads / 32;
    for (int m = m_begin + warp; m < m_end; m += 4 * kW) {
        float part[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int mm = m + j * kW;
            part[j] = 0.f;
            if (mm < Cb) {
                float x[EPL];
                load_lane<T, EPL>(ksum + (bh * nsum + mm) * D + EPL * lane, x);
#pragma unroll
                for (int i = 0; i < EPL; ++i) part[j] = fmaf(ql[i], x[i], part[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float v = warp_sum(part[j]);
            const int mm = m + j * kW;
            if (lane == 0 && mm < m_end) s[bh * s_cols + mm] = mm < Cb ? v : 0.f;
        }
    }
}

template <typename T>
cudaError_t pooled_scores_t(const TrainParams& p, float* qbar, float* kbar, float* s, cudaStream_t stream) {
    const long units = (long)p.B * p.Hkv * p.Cq;
    if (units <= 0) return cudaSuccess;
    if (p.Hq / p.Hkv * p.d / Vec<T>::N <= 64)
        pool_train_kernel<T, 64><<<(unsigned)units, 64, 0, stream>>>(
            static_cast<const T*>(p.q), static_cast<const T*>(p.k), p.n, p.Hq, p.Hkv, p.d, p.bs, p.Cq, qbar, kbar);
    else
        pool_train_kernel<T, kPoolThreads><<<(unsigned)units, kPoolThreads, 0, stream>>>(
            static_cast<const T*>(p.q), static_cast<const T*>(p.k), p.n, p.Hq, p.Hkv, p.d, p.bs, p.Cq, qbar, kbar);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    count_launch();
    const long tiles = (p.Cq + kTile - 1) / kTile;
    const long grid = tiles * tiles * p.B * p.Hkv;
    if (grid > 0x7fffffffL) return cudaErrorInvalidValue;
    pool_scores_kernel<<<(unsigned)grid, 256, 0, stream>>>(qbar, kbar, p.Cq, p.d, p.scale, s);
    err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace

// the pooling pass takes each row span as whole 16-byte vectors, one per thread:
// d * sizeof(T) a multiple of 16 and G * d * sizeof(T) at most 2 KB
bool pool_shape_ok(int d, int G, int elem_bytes) {
    const int V = 16 / elem_bytes;
    return d % V == 0 && d <= 256 && G * d / V <= kPoolThreads;
}

size_t pooled_scores_workspace(const TrainParams& p) {
    return 2 * sizeof(float) * (size_t)p.B * p.Hkv * p.Cq * p.d;
}

// p.q, p.k the inputs, s the scores [B, Hkv, Cq, Cq]; ws the workspace
cudaError_t launch_pooled_scores(const TrainParams& p, float* s, void* ws, cudaStream_t stream) {
    float* qbar = static_cast<float*>(ws);
    float* kbar = qbar + (size_t)p.B * p.Hkv * p.Cq * p.d;
    return p.is_bf16 ? pooled_scores_t<__nv_bfloat16>(p, qbar, kbar, s, stream)
                     : pooled_scores_t<float>(p, qbar, kbar, s, stream);
}

cudaError_t launch_pool_keys(const DecodeParams& p, int m0, int m1, void* ksum, int nsum, cudaStream_t stream) {
    const long grid = (long)p.B * p.Hkv * (m1 - m0);
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffffL) return cudaErrorInvalidValue;
    if (p.is_bf16)
        pool_keys_kernel<__nv_bfloat16><<<(unsigned)grid, kPoolThreads, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(p.k), p.Hkv, p.Tmax, p.d, p.bs, m0, m1 - m0, nsum,
            static_cast<__nv_bfloat16*>(ksum));
    else
        pool_keys_kernel<float><<<(unsigned)grid, kPoolThreads, 0, stream>>>(
            static_cast<const float*>(p.k), p.Hkv, p.Tmax, p.d, p.bs, m0, m1 - m0, nsum, static_cast<float*>(ksum));
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

cudaError_t launch_pool_keys_paged(const DecodeParams& p, int m0, int m1, void* ksum, int nsum, cudaStream_t stream) {
    const long grid = (long)p.B * p.Hkv * (m1 - m0);
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffffL) return cudaErrorInvalidValue;
    if (p.is_bf16)
        pool_keys_paged_kernel<__nv_bfloat16><<<(unsigned)grid, kPoolThreads, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(p.k), p.page_table, p.pages_per_seq, p.num_pages, p.Hkv, p.d, p.bs, m0,
            m1 - m0, nsum, static_cast<__nv_bfloat16*>(ksum));
    else
        pool_keys_paged_kernel<float><<<(unsigned)grid, kPoolThreads, 0, stream>>>(
            static_cast<const float*>(p.k), p.page_table, p.pages_per_seq, p.num_pages, p.Hkv, p.d, p.bs, m0, m1 - m0,
            nsum, static_cast<float*>(ksum));
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

cudaError_t launch_decode_scores(const DecodeParams& p, const void* ksum, int nsum, float* s, int s_cols,
                                 cudaStream_t stream) {
    const long chunks = (s_cols + kScoreChunk - 1) / kScoreChunk;
    const long grid = (long)p.B * p.Hkv * chunks;
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffffL) return cudaErrorInvalidValue;
    const unsigned g = (unsigned)grid;
    if (p.is_bf16) {
        const auto* qq = static_cast<const __nv_bfloat16*>(p.q);
        const auto* kk = static_cast<const __nv_bfloat16*>(ksum);
        if (p.d == 128)
            decode_scores_kernel<__nv_bfloat16, 128>
                <<<g, kScoreThreads, 0, stream>>>(qq, kk, p.ctx_len, p.Hq, p.Hkv, p.bs, nsum, s_cols, p.scale, s);
        else
            decode_scores_kernel<__nv_bfloat16, 64>
                <<<g, kScoreThreads, 0, stream>>>(qq, kk, p.ctx_len, p.Hq, p.Hkv, p.bs, nsum, s_cols, p.scale, s);
    } else {
        const auto* qq = static_cast<const float*>(p.q);
        const auto* kk = static_cast<const float*>(ksum);
        if (p.d == 128)
            decode_scores_kernel<float, 128>
                <<<g, kScoreThreads, 0, stream>>>(qq, kk, p.ctx_len, p.Hq, p.Hkv, p.bs, nsum, s_cols, p.scale, s);
        else
            decode_scores_kernel<float, 64>
                <<<g, kScoreThreads, 0, stream>>>(qq, kk, p.ctx_len, p.Hq, p.Hkv, p.bs, nsum, s_cols, p.scale, s);
    }
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace sas
