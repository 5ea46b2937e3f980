// decode.cu -- gate-free hard-Top-K decode attention (jaehun.me review of SAS,
// walkthrough Step 6: at inference the gate is dropped and only the Top-K blocks
// plus the current block are attended), and the dense full-context comparator.
//
// Split-K over the attended blocks: CTA (bh, split) handles a contiguous run of
// the (b, kv head)'s attended block list -- the selected blocks ascending, then
// the current partial block [C*b, t] -- for all query heads of the group, and
// writes an unnormalised partial (o, running max, running sum) per head.  A
// second kernel merges the partials of each (b, kv head).
#include "common.cuh"
#include "kernels.h"

namespace sas {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxG = 16;

// attended block `li` of (b, h): selected entries first (valid ones only), then
// the current block at position nsel.  Returns -1 past the end.
struct DecodeList {
    int nsel, cur_blk, t;
};

__device__ __forceinline__ DecodeList decode_list(const DecodeParams& p, int b, int h) {
    DecodeList L;
    int T = p.ctx_len[b];
    T = max(1, min(T, p.Tmax));
    L.t = T - 1;
    L.cur_blk = L.t / p.bs;
    if (p.idx == nullptr) {
        L.nsel = L.cur_blk;  // dense: every history block
    } else {
        const int32_t* row = p.idx + ((long)b * p.Hkv + h) * p.top_k;
        int cnt = 0;
        const long n_idx = (long)p.B * p.Hkv * p.top_k;
        while (cnt < p.top_k && SAS_IN_BOUNDS(((long)b * p.Hkv + h) * p.top_k + cnt, n_idx, p.status) &&
               row[cnt] >= 0 && row[cnt] < L.cur_blk)
            ++cnt;
        L.nsel = cnt;
    }
    return L;
}

__device__ __forceinline__ int list_block(const DecodeParams& p, const DecodeList& L, int b, int h, int li) {
    if (li == L.nsel) return L.cur_blk;
    if (p.idx == nullptr) return li;
    return p.idx[((long)b * p.Hkv + h) * p.top_k + li];
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) decode_partial_kernel(DecodeParams p) {
    extern __shared__ float smem[];
    const int G = p.Hq / p.Hkv;
    float* qs = smem;                 // [G][D]
    float* sc = qs + G * D;           // [G][per_split * bs]
    const int ntok_max = p.per_split * p.bs;
    __shared__ float red_m[kMaxG], red_l[kMaxG];

    const int bh = blockIdx.y, split = blockIdx.x;
    const int b = bh / p.Hkv, h = bh % p.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const DecodeList L = decode_list(p, b, h);
    const int li0 = split * p.per_split, li1 = min(L.nsel + 1, li0 + p.per_split);
    float* part = p.part + ((long)bh * p.nsplit + split) * G * (D + 2);
    // the partials of this CTA, within the workspace (or the built-in scratch)
    const long n_part = (long)p.B * p.Hkv * p.nsplit * G * (D + 2);
    if (!SAS_IN_BOUNDS(((long)bh * p.nsplit + split + 1) * G * (D + 2) - 1, n_part, p.status)) return;

    for (int i = tid; i < G * D; i += kThreads) {
        const int g = i / D, e = i % D;
        const long qi = ((long)b * p.Hq + h * G + g) * D + e;
        qs[i] = SAS_IN_BOUNDS(qi, (long)p.B * p.Hq * D, p.status)
                    ? to_f32<T>(static_cast<const T*>(p.q)[qi]) * p.scale
                    : 0.f;
    }
    __syncthreads();
    const T* kc = static_cast<const T*>(p.k) + (long)bh * p.Tmax * D;
    const T* vc = static_cast<const T*>(p.v) + (long)bh * p.Tmax * D;

    // scores: one warp per token, lanes split d
    int ntok = 0;
    for (int li = li0; li < li1; ++li) {
        const int blk = list_block(p, L, b, h, li);
        const int j0 = blk * p.bs, j1 = min(j0 + p.bs, L.t + 1);
        for (int j = j0 + warp; j < j1; j += kThreads / 32) {
            float kv[D / 32];
#pragma unroll
            for (int u = 0; u < D / 32; ++u)
                kv[u] = SAS_IN_BOUNDS(((long)bh * p.Tmax + j) * D + lane + 32 * u, (long)p.B * p.Hkv * p.Tmax * D,
                                      p.status)
                            ? to_f32<T>(kc[(long)j * D + lane + 32 * u])
                            : 0.f;
            for (int g = 0; g < G; ++g) {
                float a = 0.f;
#pragma unroll
                for (int u = 0; u < D / 32; ++u) a = fmaf(qs[g * D + lane + 32 * u], kv[u], a);
                a = warp_sum(a);
                if (lane == 0) sc[g * ntok_max + ntok + (j - j0)] = a;
            }
        }
        ntok += j1 - j0;
    }
    __syncthreads();
    // per-head max and sum (warp g handles head g, strided)
    for (int g = warp; g < G; g += kThreads / 32) {
        float mx = -INFINITY;
        for (int j = lane; j < ntok; j += 32) mx = fmaxf(mx, sc[g * ntok_max + j]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int j = lane; j < ntok; j += 32) {
            const float pv = ntok > 0 ? expf(sc[g * ntok_max + j] - mx) : 0.f;
            sc[g * ntok_max + j] = pv;
            sum += pv;
        }
        sum = warp_sum(sum);
        if (lane == 0) {
            red_m[g] = mx;
            red_l[g] = sum;
        }
    }
    __syncthreads();
    // o_g[e] = sum_j p_gj v_j[e]: thread per e (strided), all heads
    for (int e = tid; e < D; e += kThreads) {
        float acc[kMaxG];
#pragma unroll
        for (int g = 0; g < kMaxG; ++g) acc[g] = 0.f;
        int jt = 0;
        for (int li = li0; li < li1; ++li) {
            const int blk = list_block(p, L, b, h, li);
            const int j0 = blk * p.bs, j1 = min(j0 + p.bs, L.t + 1);
            for (int j = j0; j < j1; ++j, ++jt) {
                const float vv =
                    SAS_IN_BOUNDS(((long)bh * p.Tmax + j) * D + e, (long)p.B * p.Hkv * p.Tmax * D, p.status)
                        ? to_f32<T>(vc[(long)j * D + e])
                        : 0.f;
#pragma unroll
                for (int g = 0; g < kMaxG; ++g)
                    if (g < G) acc[g] = fmaf(sc[g * ntok_max + jt], vv, acc[g]);
            }
        }
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
            if (g < G) part[g * (D + 2) + e] = acc[g];
    }
    if (tid < G) {
        part[tid * (D + 2) + D] = red_m[tid];
        part[tid * (D + 2) + D + 1] = red_l[tid];
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) decode_combine_kernel(DecodeParams p) {
    const int G = p.Hq / p.Hkv;
    const int bh = blockIdx.x;
    const int b = bh / p.Hkv, h = bh % p.Hkv;
    const float* part = p.part + (long)bh * p.nsplit * G * (D + 2);
    if (!SAS_IN_BOUNDS((long)(bh + 1) * p.nsplit * G * (D + 2) - 1, (long)p.B * p.Hkv * p.nsplit * G * (D + 2),
                       p.status))
        return;
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
        for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, part[(s * G + g) * (D + 2) + D]);
        float Lsum = 0.f;
        for (int s = 0; s < p.nsplit; ++s) {
            const float* ps = part + (s * G + g) * (D + 2);
            if (ps[D + 1] > 0.f) Lsum += ps[D + 1] * expf(ps[D] - M);
        }
        const float inv = 1.f / Lsum;
        for (int e = threadIdx.x; e < D; e += kThreads) {
            float acc = 0.f;
            for (int s = 0; s < p.nsplit; ++s) {
                const float* ps = part + (s * G + g) * (D + 2);
                if (ps[D + 1] > 0.f) acc += ps[e] * expf(ps[D] - M);
            }
            const long oi = ((long)b * p.Hq + h * G + g) * D + e;
            if (SAS_IN_BOUNDS(oi, (long)p.B * p.Hq * D, p.status)) static_cast<T*>(p.o)[oi] = from_f32<T>(acc * inv);
        }
    }
}

template <typename T, int D>
cudaError_t launch_typed(const DecodeParams& p, cudaStream_t stream) {
    const int G = p.Hq / p.Hkv;
    const size_t smem = sizeof(float) * ((size_t)G * D + (size_t)G * p.per_split * p.bs);
    cudaError_t err =
        cudaFuncSetAttribute(decode_partial_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid(p.nsplit, p.B * p.Hkv);
    decode_partial_kernel<T, D><<<grid, kThreads, smem, stream>>>(p);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    count_launch();
    decode_combine_kernel<T, D><<<p.B * p.Hkv, kThreads, 0, stream>>>(p);
    err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace

// Split plan: a function of the problem only (not of the device), so that the
// workspace query needs no device.  About 4 CTAs per SM of a 148-SM B200.
void decode_plan(DecodeParams& p) {
    // attended list length: Top-K blocks + current (sparse) or every block (dense)
    p.list_max = p.idx ? p.top_k + 1 : (p.Tmax + p.bs - 1) / p.bs;
    const long rows = (long)p.B * p.Hkv;
    const int per_cap = 1024 / p.bs > 0 ? 1024 / p.bs : 1;
    const long target_ctas = 4L * 148;
    long per = (p.list_max * rows + target_ctas - 1) / target_ctas;
    if (per < 1) per = 1;
    if (per > per_cap) per = per_cap;
    p.per_split = (int)per;
    p.nsplit = (p.list_max + p.per_split - 1) / p.per_split;
}

size_t decode_workspace(const DecodeParams& p) {
    const int G = p.Hq / p.Hkv;
    return sizeof(float) * (size_t)p.B * p.Hkv * p.nsplit * G * (p.d + 2);
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream) {
    if (p.Hq / p.Hkv > kMaxG) return cudaErrorNotSupported;
    if (p.is_bf16) {
        if (p.d == 128) return launch_typed<__nv_bfloat16, 128>(p, stream);
        if (p.d == 64) return launch_typed<__nv_bfloat16, 64>(p, stream);
    } else {
        if (p.d == 128) return launch_typed<float, 128>(p, stream);
        if (p.d == 64) return launch_typed<float, 64>(p, stream);
    }
    return cudaErrorNotSupported;
}

}  // namespace sas
