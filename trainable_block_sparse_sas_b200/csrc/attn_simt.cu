// attn_simt.cu -- CUDA-core (FFMA) gated block-sparse attention, forward and
// backward, for fp32 problems (where tensor cores cannot meet fp32 accuracy) and
// for any shape the tensor-core kernels do not cover.
//
// Forward (jaehun.me review of SAS, Eq. 9 and the Kernel implementation
// paragraph): one CTA per (batch, query head, query block c) streams the
// attended key blocks -- the selected history blocks of c, ascending, each with
// the log-gate bias log g_m = s[c,m] - lse_s[c], then the current block c with
// bias 0 and a causal mask -- through shared memory with an online softmax.
//
// Backward, without atomics and therefore deterministic:
//   bwd_dq       one CTA per (batch, kv head, query block c), looping over the
//                group's query heads: recomputes P from the saved lse, dS =
//                P (dP - D), dq = sigma dS K, and the block-wise log-gate gradient
//                dlogg[c,m] = sum of dS over the tile (jaehun.me review, Kernel
//                implementation paragraph), then ds[c,:] = dlogg - g sum(dlogg).
//                D_i = dO_i . o_i is taken from the exact output, not from the
//                rounded o the forward stored: a first pass over the attended
//                blocks sums D_i = sum_j P_ij w_j dP_ij (the identity o_i =
//                sum_j P_ij w_j v_j; w = 1 except for the outer gate's g), and
//                the row's D goes to the workspace for the dk/dv kernel.  With
//                the sigmoid and raw-logit gates one history block can hold most
//                of a row's mass, and dlogg of that block then sums the rounding
//                error of the stored o over every row of the query block.
//
// Gate variants: the sigmoid and raw-logit gates change the bias and ds; the
// outer gate weights V by g (dS = P (g dP - D), dv from g P, dlogg = g sum P dP);
// the hard STE gate has bias 0, and its dq kernel also walks the dropped history
// blocks (flagged negative in the block list) for their straight-through
// gradient, giving dq nothing from them.
//   bwd_dkdv     one CTA per (batch, kv head, key block m), looping over the query
//                blocks that attend m (m itself, and every c > m whose selection
//                holds m) and the group's heads: dv = P^T dO, dk = sigma dS^T Q.
#include "common.cuh"
#include "kernels.h"

namespace sas {
namespace {

constexpr int kThreads = 256;

template <int D, int BS>
struct Cfg {
    static constexpr int RG = BS / 4;         // 4-row groups of an S tile
    static constexpr int NT_S = RG * RG;      // 4x4 micro-tiles of an S tile
    static constexpr int CG = kThreads / RG;  // column groups of an O-like tile
    static constexpr int COLS = D / CG;       // columns per thread of an O-like tile
    static constexpr int LD = D + 1;          // padded row stride of [BS][D] tiles
    static constexpr int LDS = BS + 1;        // padded row stride of [BS][BS] tiles
    static_assert(BS % 4 == 0 && kThreads % RG == 0 && D % CG == 0, "tile mapping");
};

template <typename T>
__device__ __forceinline__ float ldg(const void* p, long i) {
    return to_f32<T>(static_cast<const T*>(p)[i]);
}

template <typename T>
__device__ __forceinline__ void stg(void* p, long i, float v) {
    static_cast<T*>(p)[i] = from_f32<T>(v);
}

// a store of element i of a tensor of n elements (checked in the debug-bounds build)
template <typename T>
__device__ __forceinline__ void stg_chk(void* p, long i, long n, float v, int* status) {
    if (SAS_IN_BOUNDS(i, n, status)) static_cast<T*>(p)[i] = from_f32<T>(v);
}

// rows [BS] of head `head` (of `H` heads) starting at token t0 -> smem [BS][LD]
// (the debug-bounds build checks each index against the tensor's B n H D elements)
template <typename T, int D, int BS>
__device__ __forceinline__ void load_rows(float* dst, const void* src, int b, int n, int H, int head, int t0,
                                          const TrainParams& p) {
    using C = Cfg<D, BS>;
    for (int i = threadIdx.x; i < BS * D; i += kThreads) {
        const int r = i / D, e = i % D;
        const long gi = (((long)b * n + t0 + r) * H + head) * D + e;
        dst[r * C::LD + e] = SAS_IN_BOUNDS(gi, (long)p.B * n * H * D, p.status) ? ldg<T>(src, gi) : 0.f;
    }
}

// The attended history blocks of query block c, ascending, into blocks[]; the
// current block is appended at blocks[count].  Entries of idx outside [0, c) are
// dropped so that a malformed list cannot send a load out of range.
__device__ __forceinline__ int build_list(const TrainParams& p, long unit, int c, int* blocks) {
    __shared__ int cnt_sh;
    if (p.full_scope) {
        for (int i = threadIdx.x; i < c; i += kThreads) blocks[i] = i;
        if (threadIdx.x == 0) {
            blocks[c] = c;
            cnt_sh = c;
        }
    } else if (threadIdx.x == 0) {
        const int kk = min(p.top_k, c);
        const int32_t* row = p.idx + unit * p.top_k;
        int cnt = 0;
        const long n_idx = (long)p.B * p.Hkv * p.Cq * p.top_k;
        for (int i = 0; i < kk; ++i) {
            const int v = SAS_IN_BOUNDS(unit * p.top_k + i, n_idx, p.status) ? row[i] : -1;
            if (v >= 0 && v < c) blocks[cnt++] = v;
        }
        blocks[cnt] = c;
        cnt_sh = cnt;
    }
    __syncthreads();
    return cnt_sh;
}

// Every history block of query block c in order, for the hard STE gate's
// backward: blocks[m] = m when the selection holds m, -(m + 1) when it dropped m;
// the current block at blocks[c].  Returns c.
__device__ __forceinline__ int build_list_all(const TrainParams& p, long unit, int c, int* blocks) {
    for (int i = threadIdx.x; i < c; i += kThreads) blocks[i] = p.full_scope ? i : -(i + 1);
    if (threadIdx.x == 0) blocks[c] = c;
    __syncthreads();
    if (!p.full_scope && threadIdx.x == 0) {
        const int kk = min(p.top_k, c);
        const int32_t* row = p.idx + unit * p.top_k;
        const long n_idx = (long)p.B * p.Hkv * p.Cq * p.top_k;
        for (int i = 0; i < kk; ++i) {
            const int v = SAS_IN_BOUNDS(unit * p.top_k + i, n_idx, p.status) ? row[i] : -1;
            if (v >= 0 && v < c) blocks[v] = v;
        }
    }
    __syncthreads();
    return c;
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads) fwd_simt_kernel(TrainParams p) {
    using C = Cfg<D, BS>;
    extern __shared__ float smem[];
    float* Qs = smem;
    float* Ks = Qs + BS * C::LD;
    float* Vs = Ks + BS * C::LD;
    float* Ss = Vs + BS * C::LD;
    float* row_m = Ss + BS * C::LDS;
    float* row_l = row_m + BS;
    float* row_a = row_l + BS;
    int* blocks = reinterpret_cast<int*>(row_a + BS);

    const int tid = threadIdx.x;
    const int c = p.Cq - 1 - (int)(blockIdx.x % p.Cq);  // late (long) query blocks first
    const int hq = (int)((blockIdx.x / p.Cq) % p.Hq);
    const int b = (int)(blockIdx.x / ((long)p.Cq * p.Hq));
    const int G = p.Hq / p.Hkv, h = hq / G;
    const long unit = ((long)b * p.Hkv + h) * p.Cq + c;
    const int nsel = build_list(p, unit, c, blocks);
    const float* srow = p.s + unit * p.Cq;
    const float lse_c = gate_softmax_family(p.gate) ? p.lse_s[unit] : 0.f;

    load_rows<T, D, BS>(Qs, p.q, b, p.n, p.Hq, hq, c * BS, p);
    if (tid < BS) {
        row_m[tid] = -INFINITY;
        row_l[tid] = 0.f;
    }
    const int tr = tid / C::CG, tc = tid % C::CG;
    float acc[4][C::COLS];
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int ee = 0; ee < C::COLS; ++ee) acc[ii][ee] = 0.f;

    for (int t = 0; t <= nsel; ++t) {
        const int blk = blocks[t];
        const bool cur = (t == nsel);
        const float lg = cur ? 0.f : gate_log(srow[blk], lse_c, p.gate);
        const float bias = gate_in_logits(p.gate) ? lg : 0.f;
        const float w = (p.gate == kGateOuter && !cur) ? expf(lg) : 1.f;  // outer gate: g weights V
        __syncthreads();
        load_rows<T, D, BS>(Ks, p.k, b, p.n, p.Hkv, h, blk * BS, p);
        load_rows<T, D, BS>(Vs, p.v, b, p.n, p.Hkv, h, blk * BS, p);
        __syncthreads();
        for (int tile = tid; tile < C::NT_S; tile += kThreads) {
            const int ttr = tile / C::RG, ttc = tile % C::RG;
            float sacc[4][4] = {};
            for (int e = 0; e < D; ++e) {
                float qv[4], kv[4];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) qv[ii] = Qs[(ttr + C::RG * ii) * C::LD + e];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) kv[jj] = Ks[(ttc + C::RG * jj) * C::LD + e];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) sacc[ii][jj] = fmaf(qv[ii], kv[jj], sacc[ii][jj]);
            }
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int r = ttr + C::RG * ii, j = ttc + C::RG * jj;
                    float z = fmaf(p.scale, sacc[ii][jj], bias);
                    if (cur && j > r) z = -INFINITY;
                    Ss[r * C::LDS + j] = z;
                }
        }
        __syncthreads();
        if (tid < BS) {
            float* srow_s = Ss + tid * C::LDS;
            float mx = row_m[tid];
            for (int j = 0; j < BS; ++j) mx = fmaxf(mx, srow_s[j]);
            const float alpha = expf(row_m[tid] - mx);
            float sum = 0.f;
            for (int j = 0; j < BS; ++j) {
                const float pv = expf(srow_s[j] - mx);
                srow_s[j] = pv;
                sum += pv;
            }
            row_l[tid] = row_l[tid] * alpha + sum;
            row_m[tid] = mx;
            row_a[tid] = alpha;
        }
        __syncthreads();
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const float a = row_a[tr + C::RG * ii];
#pragma unroll
            for (int ee = 0; ee < C::COLS; ++ee) acc[ii][ee] *= a;
        }
        for (int j = 0; j < BS; ++j) {
            float pv[4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) pv[ii] = Ss[(tr + C::RG * ii) * C::LDS + j] * w;
#pragma unroll
            for (int ee = 0; ee < C::COLS; ++ee) {
                const float vv = Vs[j * C::LD + tc + C::CG * ee];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) acc[ii][ee] = fmaf(pv[ii], vv, acc[ii][ee]);
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
        const int r = tr + C::RG * ii;
        const float inv = 1.f / row_l[r];
        const long base = (((long)b * p.n + c * BS + r) * p.Hq + hq) * D;
#pragma unroll
        for (int ee = 0; ee < C::COLS; ++ee)
            stg_chk<T>(p.o, base + tc + C::CG * ee, (long)p.B * p.n * p.Hq * D, acc[ii][ee] * inv, p.status);
    }
    const long li = ((long)b * p.Hq + hq) * p.n + c * BS + tid;
    if (tid < BS && SAS_IN_BOUNDS(li, (long)p.B * p.Hq * p.n, p.status)) p.lse[li] = row_m[tid] + logf(row_l[tid]);
}

// One 4x4 micro-tile of S = Q K^T (unscaled) and dP = dO V^T: rows ttr + RG*ii
// of the [BS][D] query-side tiles against rows ttc + RG*jj of the key-side tiles.
template <int D, int BS>
__device__ __forceinline__ void tile_s_dp(const float* Qs, const float* dOs, const float* Ks, const float* Vs,
                                          int ttr, int ttc, float (&sacc)[4][4], float (&pacc)[4][4]) {
    using C = Cfg<D, BS>;
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) sacc[ii][jj] = pacc[ii][jj] = 0.f;
    for (int e = 0; e < D; ++e) {
        float qv[4], gv[4], kv[4], vv[4];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            qv[ii] = Qs[(ttr + C::RG * ii) * C::LD + e];
            gv[ii] = dOs[(ttr + C::RG * ii) * C::LD + e];
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            kv[jj] = Ks[(ttc + C::RG * jj) * C::LD + e];
            vv[jj] = Vs[(ttc + C::RG * jj) * C::LD + e];
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                sacc[ii][jj] = fmaf(qv[ii], kv[jj], sacc[ii][jj]);
                pacc[ii][jj] = fmaf(gv[ii], vv[jj], pacc[ii][jj]);
            }
    }
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads) bwd_dq_kernel(TrainParams p) {
    using C = Cfg<D, BS>;
    extern __shared__ float smem[];
    float* Qs = smem;
    float* dOs = Qs + BS * C::LD;
    float* Ks = dOs + BS * C::LD;
    float* Vs = Ks + BS * C::LD;
    float* Ss = Vs + BS * C::LD;  // dS tile
    float* rowL = Ss + BS * C::LDS;
    float* rowD = rowL + BS;
    float* red = rowD + BS;  // 33
    float* dlg = red + 33;   // [Cq]
    int* blocks = reinterpret_cast<int*>(dlg + p.Cq);

    const int tid = threadIdx.x;
    const int c = p.Cq - 1 - (int)(blockIdx.x % p.Cq);
    const int h = (int)((blockIdx.x / p.Cq) % p.Hkv);
    const int b = (int)(blockIdx.x / ((long)p.Cq * p.Hkv));
    const int G = p.Hq / p.Hkv;
    const long unit = ((long)b * p.Hkv + h) * p.Cq + c;
    const bool ste = p.gate == kGateSte;
    const int nsel = ste ? build_list_all(p, unit, c, blocks) : build_list(p, unit, c, blocks);
    const float* srow = p.s + unit * p.Cq;
    const float lse_c = gate_softmax_family(p.gate) ? p.lse_s[unit] : 0.f;
    for (int i = tid; i < nsel; i += kThreads) dlg[i] = 0.f;
    const int tr = tid / C::CG, tc = tid % C::CG;

    for (int g = 0; g < G; ++g) {
        const int hq = h * G + g;
        __syncthreads();
        load_rows<T, D, BS>(Qs, p.q, b, p.n, p.Hq, hq, c * BS, p);
        load_rows<T, D, BS>(dOs, p.dO, b, p.n, p.Hq, hq, c * BS, p);
        const long ri = ((long)b * p.Hq + hq) * p.n + c * BS + tid;
        const bool ri_ok = tid < BS && SAS_IN_BOUNDS(ri, (long)p.B * p.Hq * p.n, p.status);
        if (tid < BS) {
            rowL[tid] = ri_ok ? p.lse_in[ri] : 0.f;
            rowD[tid] = 0.f;
        }
        // pass 1: D_i = sum_j P_ij w_j dP_ij over the blocks the forward attended
        for (int t = 0; t <= nsel; ++t) {
            const int code = blocks[t];
            if (code < 0) continue;  // STE: a block the selection dropped is not part of o
            const bool cur = (t == nsel);
            const float lg = cur ? 0.f : gate_log(srow[code], lse_c, p.gate);
            const float bias = gate_in_logits(p.gate) ? lg : 0.f;
            const float w = (p.gate == kGateOuter && !cur) ? expf(lg) : 1.f;
            __syncthreads();
            load_rows<T, D, BS>(Ks, p.k, b, p.n, p.Hkv, h, code * BS, p);
            load_rows<T, D, BS>(Vs, p.v, b, p.n, p.Hkv, h, code * BS, p);
            __syncthreads();
            for (int tile = tid; tile < C::NT_S; tile += kThreads) {
                const int ttr = tile / C::RG, ttc = tile % C::RG;
                float sacc[4][4], pacc[4][4];
                tile_s_dp<D, BS>(Qs, dOs, Ks, Vs, ttr, ttc, sacc, pacc);
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int r = ttr + C::RG * ii, j = ttc + C::RG * jj;
                        const float z = fmaf(p.scale, sacc[ii][jj], bias);
                        const float pr = (cur && j > r) ? 0.f : expf(z - rowL[r]);
                        Ss[r * C::LDS + j] = pr * w * pacc[ii][jj];
                    }
            }
            __syncthreads();
            if (tid < BS) {
                float a = 0.f;
                for (int j = 0; j < BS; ++j) a += Ss[tid * C::LDS + j];
                rowD[tid] += a;
            }
        }
        __syncthreads();
        if (ri_ok) p.Dbuf[ri] = rowD[tid];  // for dk / dv
        float acc[4][C::COLS];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int ee = 0; ee < C::COLS; ++ee) acc[ii][ee] = 0.f;

        // pass 2: dS, dq and the blocks' log-gate gradients
        for (int t = 0; t <= nsel; ++t) {
            const int code = blocks[t];
            const bool dropped = code < 0;  // STE: a block the selection dropped
            const int blk = dropped ? -code - 1 : code;
            const bool cur = (t == nsel);
            const float lg = cur ? 0.f : gate_log(srow[blk], lse_c, p.gate);
            const float bias = gate_in_logits(p.gate) ? lg : 0.f;
            const float w = (p.gate == kGateOuter && !cur) ? expf(lg) : 1.f;
            __syncthreads();
            load_rows<T, D, BS>(Ks, p.k, b, p.n, p.Hkv, h, blk * BS, p);
            load_rows<T, D, BS>(Vs, p.v, b, p.n, p.Hkv, h, blk * BS, p);
            __syncthreads();
            float local = 0.f;
            for (int tile = tid; tile < C::NT_S; tile += kThreads) {
                const int ttr = tile / C::RG, ttc = tile % C::RG;
                float sacc[4][4], pacc[4][4];
                tile_s_dp<D, BS>(Qs, dOs, Ks, Vs, ttr, ttc, sacc, pacc);
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int r = ttr + C::RG * ii, j = ttc + C::RG * jj;
                        const float z = fmaf(p.scale, sacc[ii][jj], bias);
                        const float pr = (cur && j > r) ? 0.f : expf(z - rowL[r]);
                        const float dS = pr * (w * pacc[ii][jj] - rowD[r]);
                        Ss[r * C::LDS + j] = dS;
                        // the block's log-gate gradient: sum dS (the outer gate: g sum P dP)
                        local += p.gate == kGateOuter ? w * pr * pacc[ii][jj] : dS;
                    }
            }
            if (!cur) {
                const float tot = block_sum(local, red);
                if (tid == 0) dlg[t] += tot;
            }
            __syncthreads();
            if (dropped) continue;  // its dS reaches dlogg only
            for (int j = 0; j < BS; ++j) {
                float sv[4];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) sv[ii] = Ss[(tr + C::RG * ii) * C::LDS + j];
#pragma unroll
                for (int ee = 0; ee < C::COLS; ++ee) {
                    const float kv = Ks[j * C::LD + tc + C::CG * ee];
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) acc[ii][ee] = fmaf(sv[ii], kv, acc[ii][ee]);
                }
            }
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const int r = tr + C::RG * ii;
            const long base = (((long)b * p.n + c * BS + r) * p.Hq + hq) * D;
#pragma unroll
            for (int ee = 0; ee < C::COLS; ++ee)
                stg_chk<T>(p.dq, base + tc + C::CG * ee, (long)p.B * p.n * p.Hq * D, p.scale * acc[ii][ee], p.status);
        }
    }
    __syncthreads();
    // STE: dlg holds the straight-through dL/dg; as a log-gate gradient, g dL/dg
    if (ste)
        for (int i = tid; i < nsel; i += kThreads) dlg[i] *= expf(srow[i] - lse_c);
    __syncthreads();
    // ds[c, m] from dlogg (0 for blocks the row does not attend, and for m >= c):
    // g = softmax(s): dlogg_m - g_m * sum(dlogg); sigmoid dlogg_m (1 - g_m); raw dlogg_m
    float part = 0.f;
    for (int i = tid; i < nsel; i += kThreads) part += dlg[i];
    const float tot = block_sum(part, red);
    float* dsrow = p.ds + unit * p.Cq;
    if (!SAS_IN_BOUNDS((unit + 1) * p.Cq - 1, (long)p.B * p.Hkv * p.Cq * p.Cq, p.status)) return;
    for (int m = tid; m < p.Cq; m += kThreads)
        dsrow[m] = (m < c && gate_softmax_family(p.gate)) ? -expf(srow[m] - lse_c) * tot : 0.f;
    __syncthreads();
    for (int i = tid; i < nsel; i += kThreads) {
        const int m = blocks[i] < 0 ? -blocks[i] - 1 : blocks[i];
        dsrow[m] = gate_ds(dlg[i], gate_log(srow[m], lse_c, p.gate), tot, p.gate);
    }
}

// is history block m in the (ascending) selection of query block c?
__device__ __forceinline__ bool selected(const TrainParams& p, long unit_c, int c, int m) {
    if (p.full_scope) return m < c;
    int lo = 0, hi = min(p.top_k, c) - 1;
    if (!SAS_IN_BOUNDS(unit_c * p.top_k + hi, (long)p.B * p.Hkv * p.Cq * p.top_k, p.status)) return false;
    const int32_t* row = p.idx + unit_c * p.top_k;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int v = row[mid];
        if (v == m) return true;
        if (v >= 0 && v < m) lo = mid + 1;
        else hi = mid - 1;
    }
    return false;
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads) bwd_dkdv_kernel(TrainParams p) {
    using C = Cfg<D, BS>;
    extern __shared__ float smem[];
    float* Ks = smem;
    float* Vs = Ks + BS * C::LD;
    float* Qs = Vs + BS * C::LD;
    float* dOs = Qs + BS * C::LD;
    float* Ps = dOs + BS * C::LD;
    float* dSs = Ps + BS * C::LDS;
    float* rowL = dSs + BS * C::LDS;
    float* rowD = rowL + BS;
    int* clist = reinterpret_cast<int*>(rowD + BS);  // [kThreads]
    int* scan = clist + kThreads;                    // [33]

    const int tid = threadIdx.x;
    const int m = (int)(blockIdx.x % p.Cq);  // early (heavily selected) key blocks first
    const int h = (int)((blockIdx.x / p.Cq) % p.Hkv);
    const int b = (int)(blockIdx.x / ((long)p.Cq * p.Hkv));
    const int G = p.Hq / p.Hkv;
    const long ubase = ((long)b * p.Hkv + h) * p.Cq;
    load_rows<T, D, BS>(Ks, p.k, b, p.n, p.Hkv, h, m * BS, p);
    load_rows<T, D, BS>(Vs, p.v, b, p.n, p.Hkv, h, m * BS, p);
    const int tr = tid / C::CG, tc = tid % C::CG;  // rows here are keys j
    float dk[4][C::COLS], dv[4][C::COLS];
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int ee = 0; ee < C::COLS; ++ee) dk[ii][ee] = dv[ii][ee] = 0.f;

    for (int c0 = m; c0 < p.Cq; c0 += kThreads) {
        const int cc = c0 + tid;
        const int att = (cc < p.Cq && (cc == m || selected(p, ubase + cc, cc, m))) ? 1 : 0;
        int cnt;
        const int pos = block_exclusive_scan(att, scan, &cnt);
        if (att) clist[pos] = cc;
        __syncthreads();
        for (int li = 0; li < cnt; ++li) {
            const int c = clist[li];
            const bool diag = (c == m);
            const float lg =
                diag ? 0.f
                     : gate_log(p.s[(ubase + c) * p.Cq + m], gate_softmax_family(p.gate) ? p.lse_s[ubase + c] : 0.f,
                                p.gate);
            const float bias = gate_in_logits(p.gate) ? lg : 0.f;
            const float w = (p.gate == kGateOuter && !diag) ? expf(lg) : 1.f;  // outer gate: g weights V
            for (int g = 0; g < G; ++g) {
                const int hq = h * G + g;
                __syncthreads();
                load_rows<T, D, BS>(Qs, p.q, b, p.n, p.Hq, hq, c * BS, p);
                load_rows<T, D, BS>(dOs, p.dO, b, p.n, p.Hq, hq, c * BS, p);
                if (tid < BS) {
                    const long ri = ((long)b * p.Hq + hq) * p.n + c * BS + tid;
                    const bool ok = SAS_IN_BOUNDS(ri, (long)p.B * p.Hq * p.n, p.status);
                    rowL[tid] = ok ? p.lse_in[ri] : 0.f;
                    rowD[tid] = ok ? p.Dbuf[ri] : 0.f;
                }
                __syncthreads();
                for (int tile = tid; tile < C::NT_S; tile += kThreads) {
                    const int ttr = tile / C::RG, ttc = tile % C::RG;  // query rows, keys
                    float sacc[4][4], pacc[4][4];
                    tile_s_dp<D, BS>(Qs, dOs, Ks, Vs, ttr, ttc, sacc, pacc);
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            const int r = ttr + C::RG * ii, j = ttc + C::RG * jj;
                            const float z = fmaf(p.scale, sacc[ii][jj], bias);
                            const float pr = (diag && j > r) ? 0.f : expf(z - rowL[r]);
                            Ps[r * C::LDS + j] = pr * w;
                            dSs[r * C::LDS + j] = pr * (w * pacc[ii][jj] - rowD[r]);
                        }
                }
                __syncthreads();
                for (int r = 0; r < BS; ++r) {
                    float pv[4], sv[4];
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
                        pv[ii] = Ps[r * C::LDS + tr + C::RG * ii];
                        sv[ii] = dSs[r * C::LDS + tr + C::RG * ii];
                    }
#pragma unroll
                    for (int ee = 0; ee < C::COLS; ++ee) {
                        const float gv = dOs[r * C::LD + tc + C::CG * ee];
                        const float qv = Qs[r * C::LD + tc + C::CG * ee];
#pragma unroll
                        for (int ii = 0; ii < 4; ++ii) {
                            dv[ii][ee] = fmaf(pv[ii], gv, dv[ii][ee]);
                            dk[ii][ee] = fmaf(sv[ii], qv, dk[ii][ee]);
                        }
                    }
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
        const int j = tr + C::RG * ii;
        const long base = (((long)b * p.n + m * BS + j) * p.Hkv + h) * D;
#pragma unroll
        for (int ee = 0; ee < C::COLS; ++ee) {
            const long n_kv = (long)p.B * p.n * p.Hkv * D;
            stg_chk<T>(p.dk, base + tc + C::CG * ee, n_kv, p.scale * dk[ii][ee], p.status);
            stg_chk<T>(p.dv, base + tc + C::CG * ee, n_kv, dv[ii][ee], p.status);
        }
    }
}

size_t fwd_smem(int D, int BS, int Cq) {
    return sizeof(float) * (3 * BS * (D + 1) + BS * (BS + 1) + 3 * BS) + sizeof(int) * (Cq + 1);
}
size_t dq_smem(int D, int BS, int Cq) {
    return sizeof(float) * (4 * BS * (D + 1) + BS * (BS + 1) + 2 * BS + 33 + Cq) + sizeof(int) * (Cq + 1);
}
size_t dkdv_smem(int D, int BS) {
    return sizeof(float) * (4 * BS * (D + 1) + 2 * BS * (BS + 1) + 2 * BS) + sizeof(int) * (kThreads + 33);
}

template <typename Kern>
cudaError_t launch(Kern kern, long grid, size_t smem, const TrainParams& p, cudaStream_t stream) {
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffffL) return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(p);
    err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

#define SAS_DISPATCH_SIMT(KERNEL, GRID, SMEM)                                                         \
    do {                                                                                              \
        if (p.is_bf16) {                                                                              \
            if (p.d == 128) {                                                                         \
                switch (p.bs) {                                                                       \
                    case 16: return launch(KERNEL<__nv_bfloat16, 128, 16>, GRID, SMEM, p, stream);    \
                    case 32: return launch(KERNEL<__nv_bfloat16, 128, 32>, GRID, SMEM, p, stream);    \
                    case 64: return launch(KERNEL<__nv_bfloat16, 128, 64>, GRID, SMEM, p, stream);    \
                }                                                                                     \
            } else if (p.d == 64) {                                                                   \
                switch (p.bs) {                                                                       \
                    case 16: return launch(KERNEL<__nv_bfloat16, 64, 16>, GRID, SMEM, p, stream);     \
                    case 32: return launch(KERNEL<__nv_bfloat16, 64, 32>, GRID, SMEM, p, stream);     \
                    case 64: return launch(KERNEL<__nv_bfloat16, 64, 64>, GRID, SMEM, p, stream);     \
                }                                                                                     \
            }                                                                                         \
        } else {                                                                                      \
            if (p.d == 128) {                                                                         \
                switch (p.bs) {                                                                       \
                    case 16: return launch(KERNEL<float, 128, 16>, GRID, SMEM, p, stream);            \
                    case 32: return launch(KERNEL<float, 128, 32>, GRID, SMEM, p, stream);            \
                    case 64: return launch(KERNEL<float, 128, 64>, GRID, SMEM, p, stream);            \
                }                                                                                     \
            } else if (p.d == 64) {                                                                   \
                switch (p.bs) {                                                                       \
                    case 16: return launch(KERNEL<float, 64, 16>, GRID, SMEM, p, stream);             \
                    case 32: return launch(KERNEL<float, 64, 32>, GRID, SMEM, p, stream);             \
                    case 64: return launch(KERNEL<float, 64, 64>, GRID, SMEM, p, stream);             \
                }                                                                                     \
            }                                                                                         \
        }                                                                                             \
        return cudaErrorNotSupported;                                                                 \
    } while (0)

cudaError_t launch_fwd_impl(const TrainParams& p, cudaStream_t stream) {
    const long grid = (long)p.B * p.Hq * p.Cq;
    const size_t smem = fwd_smem(p.d, p.bs, p.Cq);
    SAS_DISPATCH_SIMT(fwd_simt_kernel, grid, smem);
}

cudaError_t launch_dq_impl(const TrainParams& p, cudaStream_t stream) {
    const long grid = (long)p.B * p.Hkv * p.Cq;
    const size_t smem = dq_smem(p.d, p.bs, p.Cq);
    SAS_DISPATCH_SIMT(bwd_dq_kernel, grid, smem);
}

cudaError_t launch_dkdv_impl(const TrainParams& p, cudaStream_t stream) {
    const long grid = (long)p.B * p.Hkv * p.Cq;
    const size_t smem = dkdv_smem(p.d, p.bs);
    SAS_DISPATCH_SIMT(bwd_dkdv_kernel, grid, smem);
}

}  // namespace

size_t simt_max_smem(int D, int BS, int Cq) {
    size_t a = fwd_smem(D, BS, Cq), b = dq_smem(D, BS, Cq), c = dkdv_smem(D, BS);
    return a > b ? (a > c ? a : c) : (b > c ? b : c);
}

cudaError_t launch_fwd_simt(const TrainParams& p, cudaStream_t stream) { return launch_fwd_impl(p, stream); }

size_t bwd_simt_workspace(const TrainParams& p) {
    return sizeof(float) * (size_t)p.B * p.Hq * p.n;  // D rows, written by the dq kernel
}

cudaError_t launch_bwd_simt(const TrainParams& p, cudaStream_t stream) {
    cudaError_t err = launch_dq_impl(p, stream);
    if (err != cudaSuccess) return err;
    if (p.phase_event && (err = cudaEventRecord(static_cast<cudaEvent_t>(p.phase_event), stream)) != cudaSuccess)
        return err;
    return launch_dkdv_impl(p, stream);
}

}  // namespace sas
