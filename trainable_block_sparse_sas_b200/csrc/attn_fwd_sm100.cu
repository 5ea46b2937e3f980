// attn_fwd_sm100.cu -- tensor-core (tcgen05 / TMEM / TMA) forward of SAS gated
// block-sparse attention for bf16, head_dim 128, block size 64, and 2 or 4
// query heads per KV head.
//
// o = softmax(sigma q K_S^T + log g_S) V_S (jaehun.me review of SAS, Eq. 9 and the
// Kernel implementation paragraph): for query block c the attended key blocks
// are its selected history blocks, each adding log g_m = s[c,m] - lse_s[c] to
// its logits, then the current block c with bias 0 and a causal mask.
//
// One CTA per (batch, kv head, query block).  The G query heads of the group
// share the selection, so their 64 rows each are stacked into G*64 query rows
// (row r = token * G + head, exactly the order of a TMA box over [token, head,
// d]) and processed as G/2 M-tiles of 128 rows.  Attended key blocks go two at a
// time (N = 128 keys) through a 2-stage shared-memory ring.
//   warp 0      TMA producer: Q once, then K and V blocks by block index
//   warp 1      TMEM allocation and the single MMA-issuing thread:
//                 S_i = Q_i K^T        (SS MMA, S in TMEM, 128 lanes x N columns)
//                 O_i += P_i V         (TS MMA, P read from TMEM where S was)
//   warps 2..9  softmax, one warpgroup per M-tile, one thread per row: scale,
//               add the block's log-gate bias (log2 units), mask the current
//               block causally, online max with lazy rescale of O (only when the
//               max grows by more than 2^8), exponentiate, write P as bf16 into
//               TMEM, and finally normalise O and store o and lse.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
// Every wait is time-bounded; on a timeout the kernel records the device status
// word, drains its MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <cstring>

#include "kernels.h"
#include "sm100.cuh"

namespace sas {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kBS = 64;
constexpr int kStages = 2;
constexpr int kThreads = 320;
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kKvHalf = 128 * 128;     // 2 blocks x 64 rows x 128 B (one 64-wide d slab)
constexpr uint32_t kKvStage = 2 * kKvHalf;  // both d slabs
constexpr uint32_t kBlockSlab = 64 * 128;   // one block, one d slab

struct FwdArgs {
    CUtensorMap tq, tk, tv;
    const float* s;
    const float* lse_s;
    const int32_t* idx;
    __nv_bfloat16* o;
    float* lse;
    int* status;
    int B, Hq, Hkv, n, Cq, top_k, full_scope;
    float scale_log2;
};

template <int MT>
struct FwdLayout {
    static constexpr int G = 2 * MT;
    static constexpr uint32_t kQHalf = MT * 128 * 128;  // all query rows, one d slab
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + 2 * kQHalf;
    static constexpr uint32_t kV = kK + kStages * kKvStage;
    static constexpr uint32_t kBars = kV + kStages * kKvStage;
    // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_ready[2], o_done[2], drain
    static constexpr int kNumBars = 1 + 2 * kStages + 6 + 1;
    static constexpr uint32_t kMisc = kBars + 8 * kNumBars;  // tmem base, abort flag, list count
    static constexpr uint32_t kList = kMisc + 16;  // [Cq + 1] ints, then [Cq + 1] biases
    static size_t bytes(int Cq) { return 1024 + kList + 8 * (size_t)(Cq + 1); }
};

__device__ __forceinline__ void tmem_ld32_sync(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld32(taddr, r);
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) fwd_sm100_kernel(const __grid_constant__ FwdArgs a) {
    using L = FwdLayout<MT>;
    constexpr int G = L::G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(base);
    const uint32_t sQ = sbase + L::kQ, sK = sbase + L::kK, sV = sbase + L::kV;
    const uint32_t bar0 = sbase + L::kBars;
    auto q_full = [&]() { return bar0; };
    auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto kv_empty = [&](int s) { return bar0 + 8u * (1 + kStages + s); };
    auto s_full = [&](int i) { return bar0 + 8u * (1 + 2 * kStages + i); };
    auto p_ready = [&](int i) { return bar0 + 8u * (3 + 2 * kStages + i); };
    auto o_done = [&](int i) { return bar0 + 8u * (5 + 2 * kStages + i); };
    const uint32_t drain = bar0 + 8u * (7 + 2 * kStages);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L::kMisc + 4);
    int* list_count = reinterpret_cast<int*>(base + L::kMisc + 8);
    int* list = reinterpret_cast<int*>(base + L::kList);
    float* bias2 = reinterpret_cast<float*>(base + L::kList + 4 * (a.Cq + 1));  // log-gate, log2 units

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // head-major order: concurrent CTAs share one KV head's K/V in L2; within a
    // head, long (late) query blocks first
    const int c = a.Cq - 1 - (int)(blockIdx.x % a.Cq);
    const int bh = (int)(blockIdx.x / a.Cq);
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const long unit = (long)bh * a.Cq + c;

    if (threadIdx.x == 0) {
        mbar_init(q_full(), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full(i), 1);
            mbar_init(p_ready(i), 128);
            mbar_init(o_done(i), 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&a.tq);
        prefetch_tmap(&a.tk);
        prefetch_tmap(&a.tv);
    }
    if (warp == 0) {
        // attended history blocks (ascending) with their log-gate biases, then the
        // current block (bias 0); lanes read the selection in parallel
        const float* srow = a.s + unit * a.Cq;
        const float lse_c = a.lse_s[unit];
        int cnt = 0;
        const int kk = a.full_scope ? c : min(a.top_k, c);
        const int32_t* row = a.idx + unit * a.top_k;
        for (int base_i = 0; base_i < kk; base_i += 32) {
            const int i = base_i + lane;
            const int v = i < kk ? (a.full_scope ? i : row[i]) : -1;
            const bool ok = v >= 0 && v < c;
            const unsigned bal = __ballot_sync(0xffffffffu, ok);
            if (ok) {
                const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
                list[pos] = v;
                bias2[pos] = (srow[v] - lse_c) * kLog2e;
            }
            cnt += __popc(bal);
        }
        if (lane == 0) {
            list[cnt] = c;
            bias2[cnt] = 0.f;
            *list_count = cnt + 1;
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nlist = *list_count;
    const int nsteps = (nlist + 1) / 2;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int q_row = b * a.n + c * kBS;
            mbar_arrive_expect_tx(q_full(), 2 * L::kQHalf);
            tma_load_3d(sQ, &a.tq, q_full(), 0, h * G, q_row);
            tma_load_3d(sQ + L::kQHalf, &a.tq, q_full(), 64, h * G, q_row);
            for (int t = 0; t < nsteps; ++t) {
                const int s = t % kStages, use = t / kStages;
                if (t >= kStages && !mbar_wait(kv_empty(s), (use - 1) & 1, abort_flag, a.status)) break;
                const int nb = min(2, nlist - 2 * t);
                mbar_arrive_expect_tx(kv_full(s), (uint32_t)nb * 4u * kBlockSlab);
                for (int bi = 0; bi < nb; ++bi) {
                    const int row0 = b * a.n + list[2 * t + bi] * kBS;
                    for (int kh = 0; kh < 2; ++kh) {
                        const uint32_t off = s * kKvStage + kh * kKvHalf + bi * kBlockSlab;
                        tma_load_3d(sK + off, &a.tk, kv_full(s), kh * 64, h, row0);
                        tma_load_3d(sV + off, &a.tv, kv_full(s), kh * 64, h, row0);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s64 = idesc_bf16_f32(128, 64, false, false);
            constexpr uint32_t idesc_s128 = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
            // per-tile interleaving: S_i(t+1) is issued right after PV_i(t), so tile 0's
            // next softmax overlaps tile 1's current one
            auto issue_s = [&](int t, int i) {
                const int s = t % kStages;
                const int nb = min(2, nlist - 2 * t);
                const uint32_t idesc_s = nb == 2 ? idesc_s128 : idesc_s64;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const int kh = ks >> 2, kk = ks & 3;
                    const uint64_t ad = sdesc_sw128(sQ + kh * L::kQHalf + i * 128 * 128 + kk * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(sK + s * kKvStage + kh * kKvHalf + kk * 32, 16, 1024);
                    mma_ss(tmem + i * 128, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
                }
                mma_commit(s_full(i));
            };
            bool ok = mbar_wait(q_full(), 0, abort_flag, a.status) && mbar_wait(kv_full(0), 0, abort_flag, a.status);
            if (ok) {
                tc_fence_after();
                for (int i = 0; i < MT; ++i) issue_s(0, i);
            }
            for (int t = 0; ok && t < nsteps; ++t) {
                const int s = t % kStages;
                const int nb = min(2, nlist - 2 * t);
                bool next_ready = false;
                for (int i = 0; i < MT; ++i) {
                    if (!mbar_wait(p_ready(i), t & 1, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int ks = 0; ks < 4 * nb; ++ks) {
                        const uint64_t bd = sdesc_sw128(sV + s * kKvStage + ks * 2048, kKvHalf, 1024);
                        mma_ts(tmem + 256 + i * 128, tmem + i * 128 + ks * 8, bd, idesc_pv,
                               (t > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(o_done(i));
                    if (i == MT - 1 && t + kStages < nsteps) mma_commit(kv_empty(s));
                    if (t + 1 < nsteps) {
                        if (!next_ready) {
                            if (!mbar_wait(kv_full((t + 1) % kStages), ((t + 1) / kStages) & 1, abort_flag, a.status)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            next_ready = true;
                        }
                        issue_s(t + 1, i);
                    }
                }
            }
            // all issued MMAs complete before TMEM is released
            mma_commit(drain);
            mbar_wait_drain(drain, 0, a.status);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int grp = (warp - 2) >> 2;
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        if (grp < MT) {
            const int row = 32 * quad + lane;
            const int r_unit = 128 * grp + row;
            const int tok = r_unit / G, g = r_unit % G;
            const uint32_t tS = tmem + ((uint32_t)(32 * quad) << 16) + grp * 128;
            const uint32_t tO = tmem + ((uint32_t)(32 * quad) << 16) + 256 + grp * 128;
            float m_used = -INFINITY, l = 0.f;
            bool ok = true;
            for (int t = 0; t < nsteps; ++t) {
                if (!warp_wait(s_full(grp), t & 1, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nb = min(2, nlist - 2 * t);
                // pass 1: row max over the raw logits (sigma > 0), causal mask on the
                // current block only
                float mb[2];
#pragma unroll
                for (int bi = 0; bi < 2; ++bi) {
                    mb[bi] = -INFINITY;
                    if (bi < nb) {
                        const bool cur = (2 * t + bi == nlist - 1);
                        uint32_t r0[32], r1[32];
                        tmem_ld64_sync(tS + bi * 64, r0, r1);
                        float m0 = -INFINITY, m1 = -INFINITY;
                        if (!cur) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                m0 = fmaxf(m0, __uint_as_float(r0[j]));
                                m1 = fmaxf(m1, __uint_as_float(r1[j]));
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                if (j <= tok) m0 = fmaxf(m0, __uint_as_float(r0[j]));
                                if (32 + j <= tok) m1 = fmaxf(m1, __uint_as_float(r1[j]));
                            }
                        }
                        mb[bi] = fmaf(fmaxf(m0, m1), a.scale_log2, bias2[2 * t + bi]);
                    }
                }
                const float mx = fmaxf(mb[0], mb[1]);
                const float m_new = fmaxf(m_used, mx);
                const bool need = m_new > m_used + kRescaleLog2;
                if (__any_sync(0xffffffffu, need)) {
                    const float alpha = need ? ex2(m_used - m_new) : 1.f;
                    if (t > 0) {  // PV of step t-1 completed before S of step t did
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            uint32_t r[32];
                            tmem_ld32_sync(tO + ch * 32, r);
#pragma unroll
                            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
                            tmem_st32(tO + ch * 32, r);
                        }
                        tmem_wait_st();
                    }
                    l *= alpha;
                    if (need) m_used = m_new;
                }
                // pass 2: p = 2^(S sigma log2e + bias - m) with packed fp32 pairs, written
                // as bf16 pairs over the columns already read
                uint64_t rs2 = 0ull;
#pragma unroll
                for (int bi = 0; bi < 2; ++bi) {
                    if (bi < nb) {
                        const bool cur = (2 * t + bi == nlist - 1);
                        const float off = bias2[2 * t + bi] - m_used;
                        const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), off2 = f2_pack(off, off);
                        uint32_t r0[32], r1[32];
                        tmem_ld64_sync(tS + bi * 64, r0, r1);
                        uint32_t pk[32];
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const uint32_t* rr = jj < 16 ? r0 : r1;
                            const int jl = (jj & 15) * 2;
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(rr[jl]), __uint_as_float(rr[jl + 1])), sc2, off2),
                                      x0, x1);
                            float p0 = ex2(x0), p1 = ex2(x1);
                            if (cur) {
                                if (2 * jj > tok) p0 = 0.f;
                                if (2 * jj + 1 > tok) p1 = 0.f;
                            }
                            rs2 = f2_add(rs2, f2_pack(p0, p1));
                            pk[jj] = pack_bf16x2(p0, p1);
                        }
                        tmem_st32(tS + bi * 32, pk);
                    }
                }
                float rsa, rsb;
                f2_unpack(rs2, rsa, rsb);
                const float rs = rsa + rsb;
                tmem_wait_st();
                l += rs;
                tc_fence_before();
                mbar_arrive(p_ready(grp));
            }
            if (ok && warp_wait(o_done(grp), (nsteps - 1) & 1, abort_flag, a.status)) {
                tc_fence_after();
                const float inv_l = 1.f / l;
                const int hq = h * G + g;
                __nv_bfloat16* orow = a.o + (((long)b * a.n + c * kBS + tok) * a.Hq + hq) * kD;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t r[32];
                    tmem_ld32_sync(tO + ch * 32, r);
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * inv_l, __uint_as_float(r[2 * j + 1]) * inv_l);
                    uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
                }
                a.lse[((long)b * a.Hq + hq) * a.n + c * kBS + tok] = m_used * kLn2 + logf(l);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();  // lane 0 ran the MMA loop alone: reconverge before the .aligned dealloc
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [rows, heads, 128] bf16 viewed as a 3-D tensor {d, heads, rows};
// box {64, box_heads, box_rows} with 128-byte swizzle
bool encode_tma_rows(CUtensorMap* map, const void* ptr, int heads, long rows, int box_heads, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)128, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)128 * 2, (cuuint64_t)heads * 128 * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int MT>
cudaError_t launch_mt(const TrainParams& p, cudaStream_t stream) {
    FwdArgs a;
    memset(&a, 0, sizeof(a));
    const long rows = (long)p.B * p.n;
    if (!encode_tma_rows(&a.tq, p.q, p.Hq, rows, 2 * MT, kBS) || !encode_tma_rows(&a.tk, p.k, p.Hkv, rows, 1, kBS) ||
        !encode_tma_rows(&a.tv, p.v, p.Hkv, rows, 1, kBS))
        return cudaErrorInvalidValue;
    a.s = p.s;
    a.lse_s = p.lse_s;
    a.idx = p.idx;
    a.o = static_cast<__nv_bfloat16*>(p.o);
    a.lse = p.lse;
    a.status = p.status;
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.n = p.n;
    a.Cq = p.Cq;
    a.top_k = p.top_k;
    a.full_scope = p.full_scope;
    a.scale_log2 = p.scale * kLog2e;
    const size_t smem = FwdLayout<MT>::bytes(p.Cq);
    cudaError_t err = cudaFuncSetAttribute(fwd_sm100_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const long grid = (long)p.B * p.Hkv * p.Cq;
    fwd_sm100_kernel<MT><<<(unsigned)grid, kThreads, smem, stream>>>(a);
    err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace

bool fwd_sm100_supported(const TrainParams& p) {
    if (!p.is_bf16 || p.d != kD || p.bs != kBS) return false;
    const int G = p.Hq / p.Hkv;
    if (G != 2 && G != 4) return false;
    if ((reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.k) | reinterpret_cast<uintptr_t>(p.v) |
         reinterpret_cast<uintptr_t>(p.o)) & 15u)
        return false;
    if ((long)p.B * p.n > 0x7fffffffL || (long)p.B * p.Hkv * p.Cq > 0x7fffffffL) return false;
    return FwdLayout<2>::bytes(p.Cq) <= 227 * 1024;
}

cudaError_t launch_fwd_sm100(const TrainParams& p, cudaStream_t stream) {
    const int G = p.Hq / p.Hkv;
    return G == 4 ? launch_mt<2>(p, stream) : launch_mt<1>(p, stream);
}

}  // namespace sas
