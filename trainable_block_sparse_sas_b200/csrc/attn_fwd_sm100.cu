// attn_fwd_sm100.cu -- tensor-core (tcgen05 / TMEM / TMA) forward of SAS gated
// block-sparse attention for bf16, head_dim 128, block size 64, and 2, 4 or 8
// query heads per KV head (8: two CTAs per query block, four heads each, adjacent
// in the grid so that they share the block's K and V in L2).
//
// o = softmax(sigma q K_S^T + log g_S) V_S (jaehun.me review of SAS, Eq. 9 and the
// Kernel implementation paragraph): for query block c the attended key blocks
// are the current block c with bias 0 and a causal mask (processed first, so its
// K and V are requested before the list is built) and its selected history
// blocks, each adding log g_m = s[c,m] - lse_s[c] to its logits.
//
// One CTA per (batch, kv head, query block).  The G query heads of the group
// share the selection, so their 64 rows each are stacked into G*64 query rows
// (row r = token * G + head, exactly the order of a TMA box over [token, head,
// d]) and processed as G/2 M-tiles of 128 rows.  Attended key blocks go one at a
// time (N = 64 keys) through a 4-stage shared-memory ring of K and V.
//   warp 0      TMA producer: K and V blocks of the list after the first (Q and the
//               current block's K and V are requested at the start)
//   warps 1..4  MMA issuers, two per M-tile (separate threads, so that the PV
//               chain waiting for P does not hold up the next S):
//                 S_i = Q_i K^T   (SS MMA into TMEM buffer t mod 2 of tile i)
//                 O_i += P_i V    (TS MMA, P read from the buffer it was written to)
//               With two S buffers per tile, S of block t+1 is computed while the
//               softmax of block t runs; S of block t+2 waits for PV of block t.
//   warps 5..12 softmax, one warpgroup per M-tile, one thread per row: scale,
//               add the block's log-gate bias (log2 units), mask the current
//               block causally, online max with lazy rescale of O (only when the
//               max grows by more than 2^8), exponentiate, write P as bf16 into
//               TMEM, and finally normalise O and store o and lse.
// TMEM columns: tile i's S buffers [128 i, 128 i + 64) and [128 i + 64, 128 i + 128)
// (P in the first 32 columns of its buffer), O_i [256 + 128 i, 384 + 128 i).
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
constexpr int kStages = 4;                 // K/V ring, one attended block per stage
// warp 0 TMA; warps 1..4 MMA issuers (S and PV per M-tile); warps 5..12 softmax
constexpr int kThreads = 416;
constexpr int kSoftmaxWarp0 = 5;
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kSlab = 64 * 128;        // one block (64 rows x 128 B), one 64-wide d slab
constexpr uint32_t kStage = 4 * kSlab;      // K (2 slabs) then V (2 slabs)

struct FwdArgs {
    CUtensorMap tq, tk, tv;
    const float* s;
    const float* lse_s;
    const int32_t* idx;
    __nv_bfloat16* o;
    float* lse;
    int* status;
    int B, Hq, Hkv, n, Cq, top_k, full_scope, gate;
    int hsplit;  // CTAs per query block, each taking G = 2 MT of the group's query heads
    float scale_log2;
};

template <int MT>
struct FwdLayout {
    static constexpr int G = 2 * MT;
    static constexpr uint32_t kQHalf = MT * 128 * 128;  // all query rows, one d slab
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kKV = kQ + 2 * kQHalf;     // [stage] { K: 2 slabs, V: 2 slabs }
    static constexpr uint32_t kBars = kKV + kStages * kStage;
    // q_full, kv_full[S], kv_empty[S], s_full[tile][buf], p_ready[tile][buf], pv_done[tile][buf],
    // drain, stagger.  Per-buffer barriers: a buffer's next phase needs this block's
    // PV, so no waiter can fall two phases behind.
    static constexpr int kNumBars = 1 + 2 * kStages + 4 + 4 + 4 + 1 + 1;
    static constexpr uint32_t kMisc = kBars + 8 * kNumBars;  // tmem base, abort flag, list count
    static constexpr uint32_t kList = kMisc + 16;  // [Cq + 1] ints, [Cq + 1] biases, [Cq + 1] value weights
    static size_t bytes(int Cq) { return 1024 + kList + 12 * (size_t)(Cq + 1); }
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

// kOuter: the outer gate, g scaling each history block's P before P.V (the row
// sum l stays that of the gate-free P)
template <int MT, bool kOuter>
__global__ void __launch_bounds__(kThreads, 1) fwd_sm100_kernel(const __grid_constant__ FwdArgs a) {
    using L = FwdLayout<MT>;
    constexpr int G = L::G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_align1024(smem_raw);
    const uint32_t sbase = smem_u32(base);
    const uint32_t sQ = sbase + L::kQ, sKV = sbase + L::kKV;
    const uint32_t bar0 = sbase + L::kBars;
    const uint32_t q_full = bar0;
    auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto kv_empty = [&](int s) { return bar0 + 8u * (1 + kStages + s); };
    auto s_full = [&](int i, int bf) { return bar0 + 8u * (1 + 2 * kStages + 2 * i + bf); };
    auto p_ready = [&](int i, int bf) { return bar0 + 8u * (5 + 2 * kStages + 2 * i + bf); };
    auto pv_done = [&](int i, int bf) { return bar0 + 8u * (9 + 2 * kStages + 2 * i + bf); };
    const uint32_t drain = bar0 + 8u * (13 + 2 * kStages);
    // single phase: tile 0's softmax has begun; tile 1 starts then, so that the two
    // tiles' softmax phases (exponentials) and latency-bound phases interleave
    const uint32_t stagger = bar0 + 8u * (14 + 2 * kStages);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L::kMisc + 4);
    int* list_count = reinterpret_cast<int*>(base + L::kMisc + 8);
    int* list = reinterpret_cast<int*>(base + L::kList);
    float* bias2 = reinterpret_cast<float*>(base + L::kList + 4 * (a.Cq + 1));  // log-gate, log2 units
    float* wgt = reinterpret_cast<float*>(base + L::kList + 8 * (a.Cq + 1));    // outer gate: g

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // head-major order: concurrent CTAs share one KV head's K/V in L2; within a
    // head, long (late) query blocks first; a query block's head splits adjacent
    const int hs = (int)(blockIdx.x % a.hsplit);
    const int c = a.Cq - 1 - (int)((blockIdx.x / a.hsplit) % a.Cq);
    const int bh = (int)(blockIdx.x / ((long)a.hsplit * a.Cq));
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const long unit = (long)bh * a.Cq + c;
    const int hq0 = (h * a.hsplit + hs) * G;  // first query head of this CTA

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), MT);  // each tile's PV issuer, after its PV of the block
        }
        for (int i = 0; i < 2; ++i) {
            for (int bf = 0; bf < 2; ++bf) {
                mbar_init(s_full(i, bf), 1);
                mbar_init(p_ready(i, bf), 128);
                mbar_init(pv_done(i, bf), 1);
            }
        }
        mbar_init(drain, 2 * MT);
        mbar_init(stagger, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&a.tk);
        prefetch_tmap(&a.tv);
        // Q of the query block does not depend on the selection: request it now
        const int q_row = b * a.n + c * kBS;
        mbar_arrive_expect_tx(q_full, 2 * L::kQHalf);
        tma_load_3d(sQ, &a.tq, q_full, 0, hq0, q_row);
        tma_load_3d(sQ + L::kQHalf, &a.tq, q_full, 64, hq0, q_row);
        // the current block is the list's first entry: its K and V go out now too
        mbar_arrive_expect_tx(kv_full(0), kStage);
        for (int kh = 0; kh < 2; ++kh) {
            tma_load_3d(sKV + kh * kSlab, &a.tk, kv_full(0), kh * 64, h, q_row);
            tma_load_3d(sKV + 2 * kSlab + kh * kSlab, &a.tv, kv_full(0), kh * 64, h, q_row);
        }
    }
    if (warp == 0) {
        // the current block (bias 0), then the attended history blocks (ascending)
        // with their log-gate biases; lanes read the selection in parallel
        const float* srow = a.s + unit * a.Cq;
        const long n_units = (long)a.B * a.Hkv * a.Cq;
        const float lse_c =
            gate_softmax_family(a.gate) && SAS_IN_BOUNDS(unit, n_units, a.status) ? a.lse_s[unit] : 0.f;
        int cnt = 0;
        const int kk = a.full_scope ? c : min(a.top_k, c);
        const int32_t* row = a.idx + unit * a.top_k;
        for (int base_i = 0; base_i < kk; base_i += 32) {
            const int i = base_i + lane;
            const int v = i < kk ? (a.full_scope ? i
                                    : SAS_IN_BOUNDS(unit * a.top_k + i, n_units * a.top_k, a.status) ? row[i] : -1)
                                 : -1;
            const bool ok = v >= 0 && v < c && SAS_IN_BOUNDS(unit * a.Cq + v, n_units * a.Cq, a.status);
            const unsigned bal = __ballot_sync(0xffffffffu, ok);
            if (ok) {
                const int pos = 1 + cnt + __popc(bal & ((1u << lane) - 1u));
                const float lg = gate_log(srow[v], lse_c, a.gate);
                list[pos] = v;
                bias2[pos] = gate_in_logits(a.gate) ? lg * kLog2e : 0.f;
                if (kOuter) wgt[pos] = expf(lg);
            }
            cnt += __popc(bal);
        }
        if (lane == 0) {
            list[0] = c;
            bias2[0] = 0.f;
            if (kOuter) wgt[0] = 1.f;
            *list_count = cnt + 1;
        }
        __syncwarp();  // the warp reaches the CTA barrier converged
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nlist = *list_count;  // one step per attended block

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int t = 1; t < nlist; ++t) {  // block 0 (the current block) was requested at start
                const int s = t % kStages;
                if (t >= kStages && !mbar_wait(kv_empty(s), (t / kStages - 1) & 1, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(kv_full(s), kStage);
                const int row0 = b * a.n + list[t] * kBS;
                const uint32_t st = sKV + s * kStage;
                for (int kh = 0; kh < 2; ++kh) {
                    tma_load_3d(st + kh * kSlab, &a.tk, kv_full(s), kh * 64, h, row0);
                    tma_load_3d(st + 2 * kSlab + kh * kSlab, &a.tv, kv_full(s), kh * 64, h, row0);
                }
            }
        }
        // every warp reaches the CTA barrier below converged: a barrier reached by a
        // warp in diverged pieces can release it before the other warps arrive
        __syncwarp();
    } else if (warp <= 4) {
        // ------------------------------------------------------------ MMA issuers
        // warps 1, 3: S_i = Q_i K^T for tile i = (warp - 1) / 2; warps 2, 4: O_i += P_i V
        const int i = (warp - 1) >> 1;
        const bool pv_chain = ((warp - 1) & 1) != 0;
        if (lane == 0 && i < MT) {
            bool ok = mbar_wait(q_full, 0, abort_flag, a.status);
            if (!pv_chain) {
                constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
                for (int t = 0; ok && t < nlist; ++t) {
                    const int s = t % kStages, bf = t & 1;
                    if (!mbar_wait(kv_full(s), (t / kStages) & 1, abort_flag, a.status)) break;
                    // buffer bf holds P of block t-2 until its PV has run
                    if (t >= 2 && !mbar_wait(pv_done(i, bf), ((t >> 1) - 1) & 1, abort_flag, a.status)) break;
                    if (i == 1 && t == 0 && !mbar_wait(stagger, 0, abort_flag, a.status)) break;
                    tc_fence_after();
                    const uint32_t kst = sKV + s * kStage;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const int kh = ks >> 2, kk = ks & 3;
                        mma_ss(tmem + i * 128 + bf * 64, sdesc_sw128(sQ + kh * L::kQHalf + i * 128 * 128 + kk * 32, 16, 1024),
                               sdesc_sw128(kst + kh * kSlab + kk * 32, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(s_full(i, bf));
                }
            } else {
                constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
                for (int t = 0; ok && t < nlist; ++t) {
                    const int s = t % kStages, bf = t & 1;
                    if (!mbar_wait(kv_full(s), (t / kStages) & 1, abort_flag, a.status)) break;
                    if (!mbar_wait(p_ready(i, bf), (t >> 1) & 1, abort_flag, a.status)) break;
                    tc_fence_after();
                    const uint32_t vst = sKV + s * kStage + 2 * kSlab;
#pragma unroll
                    for (int ks = 0; ks < kBS / 16; ++ks) {
                        mma_ts(tmem + 256 + i * 128, tmem + i * 128 + bf * 64 + ks * 8,
                               sdesc_sw128(vst + ks * 2048, kSlab, 1024), idesc_pv, (t > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(pv_done(i, bf));
                    if (t + kStages < nlist) mma_commit(kv_empty(s));
                }
            }
            // all issued MMAs complete before TMEM is released
            mma_commit(drain);
            mbar_wait_drain(drain, 0, a.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int grp = (warp - kSoftmaxWarp0) >> 2;
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        if (grp < MT) {
            const int row = 32 * quad + lane;
            const int r_unit = 128 * grp + row;
            const int tok = r_unit / G, g = r_unit % G;
            const uint32_t tS = tmem + ((uint32_t)(32 * quad) << 16) + grp * 128;
            const uint32_t tO = tmem + ((uint32_t)(32 * quad) << 16) + 256 + grp * 128;
            float m_used = -INFINITY, l = 0.f;
            bool ok = true;
            for (int t = 0; t < nlist; ++t) {
                const int bf = t & 1;
                if (!warp_wait(s_full(grp, bf), (t >> 1) & 1, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                if (t == 0 && grp == 0 && quad == 0 && lane == 0) mbar_arrive(stagger);
                tc_fence_after();
                const bool cur = (t == 0);
                uint32_t r0[32], r1[32];
                tmem_ld64_sync(tS + bf * 64, r0, r1);
                // row max over the raw logits (sigma > 0), causal mask on the current block
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
                const float mx = fmaf(fmaxf(m0, m1), a.scale_log2, bias2[t]);
                const float m_new = fmaxf(m_used, mx);
                const bool need = m_new > m_used + kRescaleLog2;
                if (__any_sync(0xffffffffu, need)) {
                    const float alpha = need ? ex2(m_used - m_new) : 1.f;
                    if (t > 0) {
                        // O is final for block t-1 once that block's PV has completed
                        if (!warp_wait(pv_done(grp, (t - 1) & 1), ((t - 1) >> 1) & 1, abort_flag, a.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll 1
                        for (int ch = 0; ch < 4; ++ch) {
                            uint32_t ro[32];
                            tmem_ld32_sync(tO + ch * 32, ro);
#pragma unroll
                            for (int j = 0; j < 32; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * alpha);
                            tmem_st32(tO + ch * 32, ro);
                        }
                        tmem_wait_st();
                    }
                    l *= alpha;
                    if (need) m_used = m_new;
                }
                // p = 2^(S sigma log2e + bias - m) with packed fp32 pairs, written as bf16
                // pairs over the first 32 columns of this buffer
                const float off = bias2[t] - m_used;
                const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), off2 = f2_pack(off, off);
                const float w = kOuter ? wgt[t] : 1.f;
                uint64_t rs2 = 0ull;
                uint32_t pk[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const uint32_t* rr = jj < 16 ? r0 : r1;
                    const int jl = (jj & 15) * 2;
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(rr[jl]), __uint_as_float(rr[jl + 1])), sc2, off2), x0, x1);
                    float p0 = ex2(x0), p1 = ex2(x1);
                    if (cur) {
                        if (2 * jj > tok) p0 = 0.f;
                        if (2 * jj + 1 > tok) p1 = 0.f;
                    }
                    rs2 = f2_add(rs2, f2_pack(p0, p1));
                    pk[jj] = kOuter ? pack_bf16x2(p0 * w, p1 * w) : pack_bf16x2(p0, p1);
                }
                tmem_st32(tS + bf * 64, pk);
                float rsa, rsb;
                f2_unpack(rs2, rsa, rsb);
                tmem_wait_st();
                l += rsa + rsb;
                tc_fence_before();
                mbar_arrive(p_ready(grp, bf));
            }
            const int tl = nlist - 1;
            // the row's outputs (the checks of the debug-bounds build skip the stores
            // only: the TMEM loads below are whole-warp instructions)
            const long orow_i = (((long)b * a.n + c * kBS + tok) * a.Hq + hq0 + g) * kD;
            const long lse_i = ((long)b * a.Hq + hq0 + g) * a.n + c * kBS + tok;
            const bool inb = SAS_IN_BOUNDS(orow_i + kD - 1, (long)a.B * a.n * a.Hq * kD, a.status) &&
                             SAS_IN_BOUNDS(lse_i, (long)a.B * a.Hq * a.n, a.status);
            if (ok && warp_wait(pv_done(grp, tl & 1), (tl >> 1) & 1, abort_flag, a.status)) {
                tc_fence_after();
                const float inv_l = 1.f / l;
                const int hq = hq0 + g;
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
                    if (inb) {
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
                    }
                }
                if (inb) a.lse[lse_i] = m_used * kLn2 + logf(l);
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
cudaError_t launch_mt(const TrainParams& p, int hsplit, cudaStream_t stream) {
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
    a.gate = p.gate;
    a.scale_log2 = p.scale * kLog2e;
    a.hsplit = hsplit;
    const size_t smem = FwdLayout<MT>::bytes(p.Cq);
    auto kern = p.gate == kGateOuter ? fwd_sm100_kernel<MT, true> : fwd_sm100_kernel<MT, false>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const long grid = (long)p.B * p.Hkv * p.Cq * hsplit;
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(a);
    err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace

bool fwd_sm100_supported(const TrainParams& p) {
    if (!p.is_bf16 || p.d != kD || p.bs != kBS) return false;
    const int G = p.Hq / p.Hkv;
    if (G != 2 && G != 4 && G != 8) return false;
    if ((reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.k) | reinterpret_cast<uintptr_t>(p.v) |
         reinterpret_cast<uintptr_t>(p.o)) & 15u)
        return false;
    if ((long)p.B * p.n > 0x7fffffffL || (long)p.B * p.Hkv * p.Cq * (G == 8 ? 2 : 1) > 0x7fffffffL) return false;
    return FwdLayout<2>::bytes(p.Cq) <= 227 * 1024;
}

cudaError_t launch_fwd_sm100(const TrainParams& p, cudaStream_t stream) {
    const int G = p.Hq / p.Hkv;
    // G = 2: one 128-row tile per CTA; G = 4: two; G = 8: two CTAs of two tiles (4 heads) each
    if (G == 2) return launch_mt<1>(p, 1, stream);
    return launch_mt<2>(p, G / 4, stream);
}

}  // namespace sas
