// attn_bwd_sm100.cu -- tensor-core (tcgen05 / TMEM / TMA) backward of SAS gated
// block-sparse attention for bf16, head_dim 128, block size 64, 2, 4 or 8 query
// heads per KV head.  Two kernels; results are deterministic (with 8 heads per
// KV head the dq kernel runs two CTAs of four heads per query block, which add
// their shares of the ds row -- two addends, so the order does not matter):
//
// bwd_dq_sm100: one CTA per (batch, kv head, query block c), the group's query
//   heads stacked into 128-row M-tiles as in the forward.  For each attended key
//   block (selected history blocks, then the current block):
//     S_i = Q_i K^T and dP_i = dO_i V^T             (SS MMAs into TMEM)
//     softmax warps: P = exp(S sigma + log g_m - lse), dS = P (dP - D),
//       dS written back to TMEM as bf16, and the tile sum of dS kept per warp
//       -- the block-wise log-gate gradient dlogg[c,m] (jaehun.me review of SAS,
//       Kernel implementation paragraph; inner-gate gradient, section 4.2.2)
//     dQ_i += dS_i K                                  (TS MMA, dS read from TMEM)
//   Epilogue: dq = sigma dQ, and ds[c,m] from dlogg per the gate.
//   D enters dS first as dO_i . o_i from the stored (bf16) output; the row's
//   probability-weighted D, sum_j P_ij dP_ij, differs from it by the row sum of
//   that dS, delta_i.  With each block's mass M_it = sum_{j in t} P_ij (kept in
//   the workspace as bf16) the epilogue takes delta_i M_it out of dlogg_t, so
//   dlogg and ds do not carry the rounding of o (summed over G*64 rows, that
//   rounding would otherwise reach several 1e-2 when one block holds a row's mass).
//
// bwd_dkdv_sm100: one CTA per (batch, kv head, key block m).  It walks the query
//   blocks that attend m (m itself with the causal mask, and every later block
//   whose selection holds m), one 128-row M-tile at a time:
//     S = Q K_m^T and dP = dO V_m^T                   (SS MMAs, double-buffered TMEM)
//     softmax warps: P (from S alone) and then dS as above, each written as bf16
//       rows into swizzled smem and published on its own barrier
//     dV^T += dO^T P and dK^T += Q^T dS               (SS MMAs, M = head_dim = 128)
//   Q and dO come through rings of their own (three Q stages where the list of
//   attending blocks leaves room, two dO stages), each stage freed by the MMAs
//   that read it.  Epilogue: dk = sigma dK, dv = dV.  The first items (query
//   block m itself) are requested together with K and V, before the list of
//   attending blocks is built.
//
// D_i is computed by the dq kernel's softmax threads (one row each): dO_i . o_i,
// then corrected by delta_i; the corrected value is written to the workspace for
// the dk/dv kernel, which runs after it.
//
// Gate variants (SAS's ablations of its design choices): sigmoid and raw logit change log g; the
// outer gate scales P by g (dS = P (g dP - D), dV from g P, dlogg = g sum P dP);
// the hard STE gate has bias 0 and its dq kernel also walks the dropped history
// blocks, whose dS feeds dlogg but not dQ.
// Every wait is time-bounded and reports through the device status word.

#include <cstring>

#include "kernels.h"
#include "sm100.cuh"

namespace sas {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kBS = 64;
constexpr int kDoStages = 2;                 // dk/dv dO ring depth (the Q ring takes 3 where it fits)
constexpr size_t kSmemLimit = 227 * 1024;     // dynamic shared memory per CTA
constexpr uint32_t kSlab64 = 64 * 128;    // 64 rows x 128 B: one block, one 64-wide d slab
constexpr uint32_t kSlab128 = 128 * 128;  // 128 rows x 128 B

struct BwdArgs {
    CUtensorMap tq, tdo, tk, tv;
    const float* s;
    const float* lse_s;
    const int32_t* idx;
    const float* lse;
    float* Dbuf;
    __nv_bfloat16* Mbuf;  // [CTA][list slot][row] block masses of the dq kernel
    float* Cbuf;          // [CTA][row] the rows' coefficients of those masses in dlogg
    const __nv_bfloat16* o;
    const __nv_bfloat16* dO;
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* ds;
    int* status;
    int B, Hq, Hkv, n, Cq, top_k, full_scope, gate;
    int hsplit;  // dq kernel: CTAs per query block, each taking 2 MT of the group's heads
    float scale, scale_log2;
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

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// ============================================================================
// dq / ds kernel
// ============================================================================
// warp 0 TMA; per M-tile i, warp 1 + 2i issues the S chain and warp 2 + 2i the
// dQ and dP chain (separate threads, so that a chain waiting for its operands
// does not hold up the other); warps 5..12 softmax, one group per M-tile.  The two tiles
// take turns: tile 1 issues block t once tile 0 has issued it, tile 0 issues
// block t+1 once tile 1 has issued block t, so one tile's MMAs run while the
// other tile's softmax does.
constexpr int kDqThreads = 416;
constexpr int kDqSoftmaxWarp0 = 5;

// ST: depth of the K/V ring (3 where the shared memory allows it: a block's
// K/V is then requested two blocks ahead of its use).
template <int MT, int ST>
struct DqLayout {
    static constexpr int G = 2 * MT;
    static constexpr uint32_t kHalf = MT * kSlab128;  // all query rows, one d slab
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kDO = kQ + 2 * kHalf;
    static constexpr uint32_t kK = kDO + 2 * kHalf;
    static constexpr uint32_t kV = kK + ST * 2 * kSlab64;
    static constexpr uint32_t kBars = kV + ST * 2 * kSlab64;
    // q_full, kv_full[S], kv_empty[S], s_full[2], ds_ready[2], dq_done, drain, issued[2]
    static constexpr int kNumBars = 1 + 2 * ST + 2 + 2 + 1 + 1 + 2;
    static constexpr uint32_t kMisc = kBars + 8 * kNumBars;
    static constexpr uint32_t kList = kMisc + 16;
    // list [nl] ints, biases [nl] floats, value weights [nl] floats, then the
    // per-warp dlogg partials [nl][8]; nl = the longest list (attended history
    // blocks + the current block)
    __host__ __device__ static uint32_t part_off(int nl) { return (kList + 12 * (uint32_t)nl + 15) & ~15u; }
    static size_t bytes(int nl) { return 1024 + part_off(nl) + 32 * (size_t)nl; }
};

// the hard STE gate's dq kernel walks every history block (dropped ones give
// their straight-through gradient only)
__host__ __device__ inline int dq_list_max(int Cq, int top_k, int full_scope, int gate) {
    return (full_scope || gate == kGateSte ? Cq : min(top_k, Cq)) + 1;
}

// kOuter: the outer gate (dS = P (g dP - D)); the other gates keep dS = P (dP - D)
template <int MT, int ST, bool kOuter>
__global__ void __launch_bounds__(kDqThreads, 1) bwd_dq_sm100_kernel(const __grid_constant__ BwdArgs a) {
    using L = DqLayout<MT, ST>;
    constexpr int kStages = ST;
    constexpr int G = L::G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_align1024(smem_raw);
    const uint32_t sbase = smem_u32(base);
    const uint32_t sQ = sbase + L::kQ, sDO = sbase + L::kDO, sK = sbase + L::kK, sV = sbase + L::kV;
    const uint32_t bar0 = sbase + L::kBars;
    const uint32_t q_full = bar0;
    auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto kv_empty = [&](int s) { return bar0 + 8u * (1 + kStages + s); };
    auto s_full = [&](int i) { return bar0 + 8u * (1 + 2 * kStages + i); };
    auto ds_ready = [&](int i) { return bar0 + 8u * (3 + 2 * kStages + i); };
    const uint32_t dq_done = bar0 + 8u * (5 + 2 * kStages);
    const uint32_t drain = bar0 + 8u * (6 + 2 * kStages);
    auto issued = [&](int i) { return bar0 + 8u * (7 + 2 * kStages + i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L::kMisc + 4);
    int* list_count = reinterpret_cast<int*>(base + L::kMisc + 8);
    float* tot_sh = reinterpret_cast<float*>(base + L::kMisc + 12);
    int* list = reinterpret_cast<int*>(base + L::kList);
    const int nl = dq_list_max(a.Cq, a.top_k, a.full_scope, a.gate);
    float* part = reinterpret_cast<float*>(base + L::part_off(nl));  // [slot][8 softmax warps]
    float* bias2 = reinterpret_cast<float*>(base + L::kList + 4 * nl);  // log-gate, log2 units
    // value weight: g for the outer gate; for the hard STE gate 1 on selected and
    // 0 on dropped blocks; else 1
    float* wgt = reinterpret_cast<float*>(base + L::kList + 8 * nl);
    const bool ste = a.gate == kGateSte;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // head-major order (concurrent CTAs share one KV head in L2), long query blocks
    // first, a query block's head splits adjacent
    const int hs = (int)(blockIdx.x % a.hsplit);
    const int c = a.Cq - 1 - (int)((blockIdx.x / a.hsplit) % a.Cq);
    const int bh = (int)(blockIdx.x / ((long)a.hsplit * a.Cq));
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const long unit = (long)bh * a.Cq + c;
    const int hq0 = (h * a.hsplit + hs) * G;  // first query head of this CTA
    // block masses M_t of the CTA's rows: [list slot][128 * MT rows], bf16
    __nv_bfloat16* mbase = a.Mbuf + (long)blockIdx.x * nl * (128 * MT);

    for (int i = threadIdx.x; i < 8 * nl; i += kDqThreads) part[i] = 0.f;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), MT);  // each tile's dQ/dP issuer, after its dQ of the stage
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full(i), 2);  // S chain and dP chain
            mbar_init(ds_ready(i), 128);
            mbar_init(issued(i), 2);  // both issuers of tile i have issued a block
        }
        mbar_init(dq_done, MT);
        mbar_init(drain, 2 * MT);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&a.tk);
        prefetch_tmap(&a.tv);
        // Q and dO of the query block do not depend on the selection: request them now
        const int q_row = b * a.n + c * kBS;
        mbar_arrive_expect_tx(q_full, 4 * L::kHalf);
        for (int kh = 0; kh < 2; ++kh) {
            tma_load_3d(sQ + kh * L::kHalf, &a.tq, q_full, kh * 64, hq0, q_row);
            tma_load_3d(sDO + kh * L::kHalf, &a.tdo, q_full, kh * 64, hq0, q_row);
        }
    }
    // the score row is read again by the ds epilogue: have it in L2 by then
    if (threadIdx.x < (a.Cq * 4 + 127) / 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a.s + unit * a.Cq + threadIdx.x * 32) : "memory");
    if (warp == 0) {
        // attended history blocks (ascending) with their log-gate biases, then the
        // current block (bias 0); lanes read the selection in parallel
        const float* srow = a.s + unit * a.Cq;
        const long n_units = (long)a.B * a.Hkv * a.Cq;
        const float lse_c =
            gate_softmax_family(a.gate) && SAS_IN_BOUNDS(unit, n_units, a.status) ? a.lse_s[unit] : 0.f;
        int cnt = 0;
        const int kk = a.full_scope ? c : min(a.top_k, c);
        const int32_t* row = a.idx + unit * a.top_k;
        if (ste && !a.full_scope) {
            // every history block in order, flagged by the selection
            for (int m = lane; m < c; m += 32) {
                list[m] = m;
                bias2[m] = 0.f;
                wgt[m] = 0.f;
            }
            __syncwarp();
            for (int i = lane; i < kk; i += 32) {
                const int v = SAS_IN_BOUNDS(unit * a.top_k + i, n_units * a.top_k, a.status) ? row[i] : -1;
                if (v >= 0 && v < c) wgt[v] = 1.f;
            }
            __syncwarp();
            cnt = c;
        } else {
            for (int base_i = 0; base_i < kk; base_i += 32) {
                const int i = base_i + lane;
                const int v = i < kk ? (a.full_scope ? i
                                        : SAS_IN_BOUNDS(unit * a.top_k + i, n_units * a.top_k, a.status) ? row[i]
                                                                                                          : -1)
                                     : -1;
                const bool ok = v >= 0 && v < c && SAS_IN_BOUNDS(unit * a.Cq + v, n_units * a.Cq, a.status);
                const unsigned bal = __ballot_sync(0xffffffffu, ok);
                if (ok) {
                    const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
                    const float lg = gate_log(srow[v], lse_c, a.gate);
                    list[pos] = v;
                    bias2[pos] = gate_in_logits(a.gate) ? lg * kLog2e : 0.f;
                    wgt[pos] = a.gate == kGateOuter ? expf(lg) : 1.f;
                }
                cnt += __popc(bal);
            }
        }
        if (lane == 0) {
            list[cnt] = c;
            bias2[cnt] = 0.f;
            wgt[cnt] = 1.f;
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
    const int nlist = *list_count;  // history blocks + the current block

    if (warp == 0) {
        if (lane == 0) {
            for (int t = 0; t < nlist; ++t) {
                const int s = t % kStages;
                if (t >= kStages && !mbar_wait(kv_empty(s), (t / kStages - 1) & 1, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(kv_full(s), 4 * kSlab64);
                const int row0 = b * a.n + list[t] * kBS;
                for (int kh = 0; kh < 2; ++kh) {
                    tma_load_3d(sK + s * 2 * kSlab64 + kh * kSlab64, &a.tk, kv_full(s), kh * 64, h, row0);
                    tma_load_3d(sV + s * 2 * kSlab64 + kh * kSlab64, &a.tv, kv_full(s), kh * 64, h, row0);
                }
            }
        }
        // every warp reaches the CTA barrier below converged: a barrier reached by a
        // warp in diverged pieces can release it before the other warps arrive
        __syncwarp();
    } else if (warp < kDqSoftmaxWarp0) {
        const int i = (warp - 1) >> 1;       // M-tile
        const bool dp_chain = ((warp - 1) & 1) != 0;
        if (lane == 0 && i < MT) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
            constexpr uint32_t idesc_dq = idesc_bf16_f32(128, 128, false, true);
            // S_i = Q_i K^T (columns i*128) or dP_i = dO_i V^T (columns i*128 + 64); the
            // softmax writes dS over dP, so dQ_i(t-1) = dS K precedes dP_i(t) in the
            // dP thread's order
            const uint32_t a_base = (dp_chain ? sDO : sQ) + i * kSlab128;
            const uint32_t b_base = dp_chain ? sV : sK;
            const uint32_t d_col = tmem + i * 128 + (dp_chain ? 64 : 0);
            auto issue_dq = [&](int t) {
                const uint32_t kst = sK + (t % kStages) * 2 * kSlab64;
#pragma unroll
                for (int ks = 0; ks < kBS / 16; ++ks) {
                    const uint64_t bd = sdesc_sw128(kst + ks * 2048, kSlab64, 1024);
                    mma_ts(tmem + 256 + i * 128, tmem + i * 128 + 64 + ks * 8, bd, idesc_dq, (t > 0 || ks > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(q_full, 0, abort_flag, a.status);
            for (int t = 0; ok && t < nlist; ++t) {
                const int s = t % kStages;
                if (!mbar_wait(kv_full(s), (t / kStages) & 1, abort_flag, a.status)) break;
                // block t reuses the tile's S/dP columns once softmax(t-1) is done with them
                if (t > 0 && !mbar_wait(ds_ready(i), (t - 1) & 1, abort_flag, a.status)) break;
                if (MT == 2) {  // turn order between the two tiles
                    if (i == 1 && !mbar_wait(issued(0), t & 1, abort_flag, a.status)) break;
                    if (i == 0 && t > 0 && !mbar_wait(issued(1), (t - 1) & 1, abort_flag, a.status)) break;
                }
                tc_fence_after();
                if (dp_chain && t > 0) {
                    issue_dq(t - 1);
                    if (t - 1 + kStages < nlist) mma_commit(kv_empty((t - 1) % kStages));
                }
                const uint32_t bst = b_base + s * 2 * kSlab64;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const int kh = ks >> 2, kk = ks & 3;
                    mma_ss(d_col, sdesc_sw128(a_base + kh * L::kHalf + kk * 32, 16, 1024),
                           sdesc_sw128(bst + kh * kSlab64 + kk * 32, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                }
                mma_commit(s_full(i));
                if (MT == 2) mbar_arrive(issued(i));
            }
            if (ok && dp_chain && nlist > 0 && mbar_wait(ds_ready(i), (nlist - 1) & 1, abort_flag, a.status)) {
                tc_fence_after();
                issue_dq(nlist - 1);
            }
            if (dp_chain) mma_commit(dq_done);
            mma_commit(drain);
            mbar_wait_drain(drain, 0, a.status);
        }
        __syncwarp();
    } else {
        const int wi = warp - kDqSoftmaxWarp0;  // 0..7
        const int grp = wi >> 2;
        const int quad = warp & 3;
        if (grp < MT) {
            const int row = 32 * quad + lane;
            const int r_unit = 128 * grp + row;
            const int tok = r_unit / G, g = r_unit % G;
            const int hq = hq0 + g;
            const long ri = ((long)b * a.Hq + hq) * a.n + c * kBS + tok;
            const long e0 = (((long)b * a.n + c * kBS + tok) * a.Hq + hq) * kD;
            // debug-bounds build: this row's global indices (o, dO, dq rows; lse, D)
            const bool inb = SAS_IN_BOUNDS(e0 + kD - 1, (long)a.B * a.n * a.Hq * kD, a.status) &&
                             SAS_IN_BOUNDS(ri, (long)a.B * a.Hq * a.n, a.status);
            const float lse2 = inb ? a.lse[ri] * kLog2e : 0.f;
            // D = dO . o of this row (fp32 sum of the bf16 products), kept for the
            // dk/dv kernel as well
            float Drow = 0.f;
            if (inb) {
                const uint4* po = reinterpret_cast<const uint4*>(a.o + e0);
                const uint4* pd = reinterpret_cast<const uint4*>(a.dO + e0);
                uint64_t acc2 = 0ull;
#pragma unroll 4
                for (int v4 = 0; v4 < kD / 8; ++v4) {
                    const uint4 x = po[v4], y = pd[v4];
                    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[u]));
                        const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[u]));
                        acc2 = f2_fma(f2_pack(xf.x, xf.y), f2_pack(yf.x, yf.y), acc2);
                    }
                }
                float da, db;
                f2_unpack(acc2, da, db);
                Drow = da + db;
                a.Dbuf[ri] = Drow;
            }
            const long n_mass = (long)gridDim.x * dq_list_max(a.Cq, a.top_k, a.full_scope, a.gate) * (128 * MT);
            const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
            const uint32_t tS = tmem + lane_off + grp * 128, tP = tS + 64;
            const uint32_t tQ = tmem + lane_off + 256 + grp * 128;
            __nv_bfloat16* mrow = mbase + r_unit;  // stride 128 * MT per slot
            float delta = 0.f;  // sum_j dS_ij of the row (dS taken with the stored-o D)
            bool ok = true;
            for (int t = 0; t < nlist; ++t) {
                if (!warp_wait(s_full(grp), t & 1, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const bool cur = (t == nlist - 1);
                const float off = bias2[t] - lse2;
                const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), off2 = f2_pack(off, off);
                const uint64_t negD2 = f2_pack(-Drow, -Drow);
                // dS = P (w dP - D), w = g for the outer gate; a dropped block of the STE
                // gate (w = 0 in the list) gives dQ nothing
                const float wt = wgt[t];
                const bool dropped = ste && wt == 0.f;
                const uint64_t w2 = f2_pack(wt, wt);
                uint64_t rs2 = 0ull, m2 = 0ull;
                uint32_t pk[32];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {  // 32 keys at a time
                    uint32_t sr[32], dr[32];
                    tmem_ld32x2_sync(tS + 32 * hh, tP + 32 * hh, sr, dr);
#pragma unroll
                    for (int jq = 0; jq < 16; ++jq) {
                        const int jj = 16 * hh + jq;
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * jq]), __uint_as_float(sr[2 * jq + 1])), sc2, off2),
                                  x0, x1);
                        float p0 = ex2(x0), p1 = ex2(x1);
                        if (cur) {
                            if (2 * jj > tok) p0 = 0.f;
                            if (2 * jj + 1 > tok) p1 = 0.f;
                        }
                        const uint64_t p2 = f2_pack(p0, p1);
                        const uint64_t dp2 = f2_pack(__uint_as_float(dr[2 * jq]), __uint_as_float(dr[2 * jq + 1]));
                        const uint64_t ds2 = f2_mul(p2, kOuter ? f2_fma(dp2, w2, negD2) : f2_add(dp2, negD2));
                        rs2 = f2_add(rs2, ds2);
                        m2 = f2_add(m2, p2);
                        float d0, d1;
                        f2_unpack(ds2, d0, d1);
                        pk[jj] = pack_bf16x2(d0, d1);
                    }
                }
                float rsa, rsb;
                f2_unpack(rs2, rsa, rsb);
                float rs = rsa + rsb;
                if (dropped) {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) pk[jj] = 0u;
                }
                tmem_st32(tP, pk);  // dS over dP, for dQ = dS K
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(ds_ready(grp));
                if (!dropped) delta += rs;  // the row's P sum to 1 over the attended keys
                if (!cur) {
                    float ma, mb;
                    f2_unpack(m2, ma, mb);
                    if (SAS_IN_BOUNDS((mrow - a.Mbuf) + (long)t * (128 * MT), n_mass, a.status))
                        mrow[t * (128 * MT)] = __float2bfloat16_rn(ma + mb);
                    rs = warp_sum(rs);
                    if (lane == 0) part[t * 8 + wi] = rs;
                }
            }
            if (inb) a.Dbuf[ri] = Drow + delta;  // D for dk / dv
            // dlogg_t = sum_i (dS-sum_it - coef_i M_it): the exact-D correction, or
            // for the outer gate g_t sum P dP = dS-sum + D M
            a.Cbuf[(long)blockIdx.x * (128 * MT) + r_unit] = kOuter ? -Drow : delta;
            if (ok && warp_wait(dq_done, 0, abort_flag, a.status)) {
                tc_fence_after();
                __nv_bfloat16* drow = a.dq + (((long)b * a.n + c * kBS + tok) * a.Hq + hq) * kD;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t r[32];
                    tmem_ld32_sync(tQ + ch * 32, r);
                    uint32_t o[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        o[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * a.scale, __uint_as_float(r[2 * j + 1]) * a.scale);
                    uint4* dst = reinterpret_cast<uint4*>(drow + ch * 32);
                    if (inb) {
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(o[4 * v4], o[4 * v4 + 1], o[4 * v4 + 2], o[4 * v4 + 3]);
                    }
                }
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
    // dlogg_t: the group's warp partials, less sum_i delta_i M_it; eight threads per
    // slot, each a strip of the rows (2 MT 16-byte loads), summed over the eight
    const int nsel = nlist - 1;
    const int sub = threadIdx.x & 7;
    const unsigned grp_mask = 0xffu << (threadIdx.x & 24);  // the 8 lanes sharing a slot
    for (int t = threadIdx.x >> 3; t < nsel; t += kDqThreads / 8) {
        const uint4* mv = reinterpret_cast<const uint4*>(mbase + (long)t * (128 * MT)) + sub * 2 * MT;
        const float4* dv4 = reinterpret_cast<const float4*>(a.Cbuf + (long)blockIdx.x * (128 * MT)) + sub * 4 * MT;
        float corr = 0.f;
#pragma unroll
        for (int v = 0; v < 2 * MT; ++v) {  // 8 rows per 16-byte load
            const uint4 x = mv[v];
            const float4 d0 = dv4[2 * v], d1 = dv4[2 * v + 1];
            const float2 m01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.x));
            const float2 m23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.y));
            const float2 m45 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.z));
            const float2 m67 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.w));
            corr = fmaf(d0.x, m01.x, corr);
            corr = fmaf(d0.y, m01.y, corr);
            corr = fmaf(d0.z, m23.x, corr);
            corr = fmaf(d0.w, m23.y, corr);
            corr = fmaf(d1.x, m45.x, corr);
            corr = fmaf(d1.y, m45.y, corr);
            corr = fmaf(d1.z, m67.x, corr);
            corr = fmaf(d1.w, m67.y, corr);
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) corr += __shfl_xor_sync(grp_mask, corr, o);
        if (sub != 0) continue;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) acc += part[t * 8 + w];
        float dl = acc - corr;
        // STE: the straight-through dL/dg of the block, as a log-gate gradient g dL/dg
        if (ste) dl *= expf(a.s[unit * a.Cq + list[t]] - a.lse_s[unit]);
        part[t * 8] = dl;
    }
    __syncthreads();
    if (warp == 0) {
        float tot = 0.f;
        for (int t = lane; t < nsel; t += 32) tot += part[t * 8];
        tot = warp_sum(tot);
        if (lane == 0) *tot_sh = tot;
    }
    __syncthreads();
    if (*abort_flag) return;
    if (!SAS_IN_BOUNDS((unit + 1) * a.Cq - 1, (long)a.B * a.Hkv * a.Cq * a.Cq, a.status)) return;
    const float tot = *tot_sh;
    const float* srow = a.s + unit * a.Cq;
    float* dsrow = a.ds + unit * a.Cq;
    // every block: ds of a block the row does not attend (dlogg 0: -g_m * sum(dlogg)
    // for the softmax gate, 0 otherwise; 0 from c on); then the attended ones are
    // overwritten with their ds, log g_m from the bias kept in smem
    const float lse_c = gate_softmax_family(a.gate) ? a.lse_s[unit] : 0.f;
    if (a.hsplit > 1) {
        // the group's heads are split over hsplit CTAs: ds is linear in dlogg, so each
        // CTA adds its share of every entry m < c to the row (zeroed before the
        // launch); two addends per entry keep the sum independent of their order
        float* dlm = reinterpret_cast<float*>(base + L::kQ);  // the freed Q tile: dlogg by block
        for (int m = threadIdx.x; m < c; m += kDqThreads) dlm[m] = 0.f;
        __syncthreads();
        for (int t = threadIdx.x; t < nsel; t += kDqThreads) dlm[list[t]] = part[t * 8];
        __syncthreads();
        for (int m = threadIdx.x; m < c; m += kDqThreads) {
            const float v = gate_ds(dlm[m], gate_log(srow[m], lse_c, a.gate), tot, a.gate);
            if (v != 0.f) atomicAdd(dsrow + m, v);
        }
        return;
    }
    if (gate_softmax_family(a.gate)) {
        for (int m = threadIdx.x; m < a.Cq; m += kDqThreads) dsrow[m] = m < c ? -expf(srow[m] - lse_c) * tot : 0.f;
    } else {
        for (int m = threadIdx.x; m < a.Cq; m += kDqThreads) dsrow[m] = 0.f;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < nsel; t += kDqThreads) {
        const float lg = gate_in_logits(a.gate) ? bias2[t] * kLn2 : gate_log(srow[list[t]], lse_c, a.gate);
        dsrow[list[t]] = gate_ds(part[t * 8], lg, tot, a.gate);
    }
}

// ============================================================================
// dk / dv kernel
// ============================================================================
// warp 0 TMA; warps 1 and 2 issue the S and dP MMA chains, warps 3 and 4 the dV
// and dK chains with lanes 0 and 1 taking the two 64-row halves of each item
// into separate accumulators (separate threads, so that a chain waiting for its
// operands or its P / dS does not hold up another); warps 5..12 two softmax
// groups (key halves)
constexpr int kKvThreads = 416;
constexpr int kKvSoftmaxWarp0 = 5;

template <int QS>
struct DkvLayout {
    static constexpr int DS = kDoStages;
    static constexpr uint32_t kK = 0;                     // 2 slabs x 64 rows
    static constexpr uint32_t kV = kK + 2 * kSlab64;
    static constexpr uint32_t kQ = kV + 2 * kSlab64;      // [stage][slab] 128 rows
    static constexpr uint32_t kDO = kQ + QS * 2 * kSlab128;
    static constexpr uint32_t kP = kDO + DS * 2 * kSlab128;  // 128 rows x 64 keys bf16
    static constexpr uint32_t kDS = kP + kSlab128;
    static constexpr uint32_t kBars = kDS + kSlab128;
    // kv_full, q_full[QS], q_empty[QS], do_full[DS], do_empty[DS], s_full[2], dp_full[2],
    // s_free[2], dp_free[2], p_ready, ds_ready, p_done, ds_done, final, drain
    static constexpr int kNumBars = 1 + 2 * QS + 2 * DS + 14;
    static constexpr uint32_t kMisc = kBars + 8 * kNumBars;
    static constexpr uint32_t kList = kMisc + 16;
    static constexpr uint32_t kScan = kList;  // 40 ints of scan scratch, then the list as int16
    static size_t bytes(int Cq) { return 1024 + kList + 4 * 40 + 2 * (size_t)(Cq + 1); }
};

// is history block m in the ascending selection of query block c (unit uc)?
__device__ __forceinline__ bool holds(const BwdArgs& a, long uc, int c, int m) {
    int lo = 0, hi = min(a.top_k, c) - 1;
    if (!SAS_IN_BOUNDS(uc * a.top_k + hi, (long)a.B * a.Hkv * a.Cq * a.top_k, a.status)) return false;
    const int32_t* row = a.idx + uc * a.top_k;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int v = row[mid];
        if (v == m) return true;
        if (v >= 0 && v < m) lo = mid + 1;
        else hi = mid - 1;
    }
    return false;
}

// kOuter: the outer gate, P and dP scaled by g of the (query block, key block)
// pair: dV += (g P)^T dO, dS = P (g dP - D).
// QS: depth of the Q ring (dO's is kDoStages).  Q of an item is free once S and dK
// of the item have completed, dO once dP and dV have; P is published as soon as S
// lands, so dV and the dO ring do not wait for dP and dS.
template <int MT, bool kOuter, int QS>
__global__ void __launch_bounds__(kKvThreads, 1) bwd_dkdv_sm100_kernel(const __grid_constant__ BwdArgs a) {
    using L = DkvLayout<QS>;
    constexpr int DS = L::DS;
    constexpr int G = 2 * MT;
    constexpr int kRowsTok = 128 / G;  // tokens per 128-row item
    // items of query block m, loaded up front
    constexpr int kPreQ = QS < MT ? QS : MT, kPreDO = DS < MT ? DS : MT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_align1024(smem_raw);
    const uint32_t sbase = smem_u32(base);
    const uint32_t sK = sbase + L::kK, sV = sbase + L::kV, sQ = sbase + L::kQ, sDO = sbase + L::kDO;
    const uint32_t sP = sbase + L::kP, sDS = sbase + L::kDS;
    const uint32_t bar0 = sbase + L::kBars;
    const uint32_t kv_full = bar0;
    auto q_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto q_empty = [&](int s) { return bar0 + 8u * (1 + QS + s); };
    auto do_full = [&](int s) { return bar0 + 8u * (1 + 2 * QS + s); };
    auto do_empty = [&](int s) { return bar0 + 8u * (1 + 2 * QS + DS + s); };
    constexpr int kB = 1 + 2 * QS + 2 * DS;  // first barrier after the rings
    auto s_full = [&](int i) { return bar0 + 8u * (kB + i); };
    auto dp_full = [&](int i) { return bar0 + 8u * (kB + 2 + i); };
    auto s_free = [&](int i) { return bar0 + 8u * (kB + 4 + i); };
    auto dp_free = [&](int i) { return bar0 + 8u * (kB + 6 + i); };
    const uint32_t p_ready = bar0 + 8u * (kB + 8);
    const uint32_t ds_ready = bar0 + 8u * (kB + 9);
    const uint32_t p_done = bar0 + 8u * (kB + 10);
    const uint32_t ds_done = bar0 + 8u * (kB + 11);
    const uint32_t final_bar = bar0 + 8u * (kB + 12);
    const uint32_t drain = bar0 + 8u * (kB + 13);
    static_assert(kB + 14 == L::kNumBars, "barrier count");
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L::kMisc + 4);
    int* scan = reinterpret_cast<int*>(base + L::kScan);  // 33 ints
    int16_t* list = reinterpret_cast<int16_t*>(scan + 40);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // head-major order (concurrent CTAs share one KV head's Q/dO in L2); within a
    // head, early (widely selected) key blocks first
    const int m = (int)(blockIdx.x % a.Cq);
    const int bh = (int)(blockIdx.x / a.Cq);
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const long ubase = (long)bh * a.Cq;

    if (threadIdx.x == 0) {
        // arrival counts: commits of the chains that must all have completed
        mbar_init(kv_full, 1);
        for (int s = 0; s < QS; ++s) {
            mbar_init(q_full(s), 1);
            mbar_init(q_empty(s), 3);  // S chain and the two dK lanes
        }
        for (int s = 0; s < DS; ++s) {
            mbar_init(do_full(s), 1);
            mbar_init(do_empty(s), 3);  // dP chain and the two dV lanes
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full(i), 1);
            mbar_init(dp_full(i), 1);
            mbar_init(s_free(i), 256);  // softmax threads have read the buffer
            mbar_init(dp_free(i), 256);
        }
        mbar_init(p_ready, 256);
        mbar_init(ds_ready, 256);
        mbar_init(p_done, 2);
        mbar_init(ds_done, 2);
        mbar_init(final_bar, 4);
        mbar_init(drain, 6);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&a.tq);
        prefetch_tmap(&a.tdo);
        // K and V of the key block do not depend on the list: requested before it is built
        mbar_arrive_expect_tx(kv_full, 4 * kSlab64);
        const int krow = b * a.n + m * kBS;
        for (int kh = 0; kh < 2; ++kh) {
            tma_load_3d(sK + kh * kSlab64, &a.tk, kv_full, kh * 64, h, krow);
            tma_load_3d(sV + kh * kSlab64, &a.tv, kv_full, kh * 64, h, krow);
        }
        // so are the first items: query block m itself, which always attends m
        for (int j = 0; j < kPreQ; ++j) {
            const int qrow = b * a.n + m * kBS + j * kRowsTok;
            mbar_arrive_expect_tx(q_full(j), 2 * kSlab128);
            for (int kh = 0; kh < 2; ++kh) tma_load_3d(sQ + (j * 2 + kh) * kSlab128, &a.tq, q_full(j), kh * 64, h * G, qrow);
        }
        for (int j = 0; j < kPreDO; ++j) {
            const int qrow = b * a.n + m * kBS + j * kRowsTok;
            mbar_arrive_expect_tx(do_full(j), 2 * kSlab128);
            for (int kh = 0; kh < 2; ++kh)
                tma_load_3d(sDO + (j * 2 + kh) * kSlab128, &a.tdo, do_full(j), kh * 64, h * G, qrow);
        }
    }

    // query blocks attending key block m: m itself, then every c > m holding m
    list[0] = (int16_t)m;
    int nlist = 1;
    for (int c0 = m + 1; c0 < a.Cq; c0 += kKvThreads) {
        const int cc = c0 + (int)threadIdx.x;
        const int att = (cc < a.Cq && (a.full_scope || holds(a, ubase + cc, cc, m))) ? 1 : 0;
        int cnt;
        const int pos = block_exclusive_scan(att, scan, &cnt);
        if (att) list[nlist + pos] = (int16_t)cc;
        nlist += cnt;
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nitems = nlist * MT;
    // TMEM: S/dP buffers at 0 and 128 (S | dP), dV^T halves at 256 and 320, dK^T halves at 384 and 448

    if (warp == 0) {
        // lane 0 refills the Q ring, lane 1 the dO ring, each in item order
        if (lane < 2) {
            const bool is_q = lane == 0;
            const int ns = is_q ? QS : DS;
            const uint32_t ring = is_q ? sQ : sDO;
            const CUtensorMap* tm = is_q ? &a.tq : &a.tdo;
            int st = is_q ? kPreQ % QS : kPreDO % DS;
            for (int j = is_q ? kPreQ : kPreDO; j < nitems; ++j) {
                const uint32_t full = is_q ? q_full(st) : do_full(st), empty = is_q ? q_empty(st) : do_empty(st);
                if (j >= ns && !mbar_wait(empty, (j / ns - 1) & 1, abort_flag, a.status)) break;
                const int c = list[j / MT], i = j % MT;
                const int qrow = b * a.n + c * kBS + i * kRowsTok;
                mbar_arrive_expect_tx(full, 2 * kSlab128);
                for (int kh = 0; kh < 2; ++kh) tma_load_3d(ring + (st * 2 + kh) * kSlab128, tm, full, kh * 64, h * G, qrow);
                st = st + 1 == ns ? 0 : st + 1;
            }
        }
        // every warp reaches the CTA barrier below converged: a barrier reached by a
        // warp in diverged pieces can release it before the other warps arrive
        __syncwarp();
    } else if (warp < kKvSoftmaxWarp0) {
        const int chain = warp - 1;  // 0 S, 1 dP, 2 dV, 3 dK
        if (lane < (chain < 2 ? 1 : 2)) {
            bool ok = true;
            // Q chains (S, dK) walk the Q ring, dO chains (dP, dV) the dO ring
            const bool on_q = chain == 0 || chain == 3;
            const int ns = on_q ? QS : DS;
            if (chain < 2) {
                // S = Q K^T (chain 0) or dP = dO V^T (chain 1) of item j into TMEM buffer j & 1,
                // once the softmax threads have read that buffer's previous item
                constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
                const uint32_t a_base = chain == 0 ? sQ : sDO, b_base = chain == 0 ? sK : sV;
                ok = mbar_wait(kv_full, 0, abort_flag, a.status);
                int st = 0;
                for (int j = 0; ok && j < nitems; ++j) {
                    const int buf = j & 1;
                    if (j >= 2 && !mbar_wait(chain == 0 ? s_free(buf) : dp_free(buf), ((j >> 1) - 1) & 1, abort_flag,
                                             a.status))
                        break;
                    if (!mbar_wait(chain == 0 ? q_full(st) : do_full(st), (j / ns) & 1, abort_flag, a.status)) break;
                    tc_fence_after();
                    const uint32_t at = a_base + st * 2 * kSlab128;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const int kh = ks >> 2, kk = ks & 3;
                        mma_ss(tmem + buf * 128 + chain * 64, sdesc_sw128(at + kh * kSlab128 + kk * 32, 16, 1024),
                               sdesc_sw128(b_base + kh * kSlab64 + kk * 32, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(chain == 0 ? s_full(buf) : dp_full(buf));
                    if (j + ns < nitems) mma_commit(chain == 0 ? q_empty(st) : do_empty(st));
                    st = st + 1 == ns ? 0 : st + 1;
                }
            } else {
                // dV^T += dO^T P (chain 2) or dK^T += Q^T dS (chain 3), accumulated over all
                // items; lane 0 sums rows 0..63 of each item, lane 1 rows 64..127
                constexpr uint32_t idesc_g = idesc_bf16_f32(128, 64, true, true);
                const uint32_t a_base = chain == 2 ? sDO : sQ, b_base = chain == 2 ? sP : sDS;
                const uint32_t acc = tmem + 256 + (chain - 2) * 128 + lane * 64;
                int st = 0;
                for (int j = 0; j < nitems; ++j) {
                    // P (dS) of item j is in shared memory, and so is its dO (Q): dV does not
                    // follow dP, so it waits for dO itself
                    if (!mbar_wait(chain == 2 ? p_ready : ds_ready, j & 1, abort_flag, a.status) ||
                        !mbar_wait(chain == 2 ? do_full(st) : q_full(st), (j / ns) & 1, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t at = a_base + st * 2 * kSlab128 + lane * 4 * 2048;
                    const uint32_t bt = b_base + lane * 4 * 2048;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        mma_ss(acc, sdesc_sw128(at + ks * 2048, kSlab128, 1024), sdesc_sw128(bt + ks * 2048, kSlab128, 1024),
                               idesc_g, (j > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(chain == 2 ? p_done : ds_done);
                    if (j + ns < nitems) mma_commit(chain == 2 ? do_empty(st) : q_empty(st));
                    st = st + 1 == ns ? 0 : st + 1;
                }
                if (ok) mma_commit(final_bar);
            }
            // every chain's MMAs complete before TMEM is released
            mma_commit(drain);
            mbar_wait_drain(drain, 0, a.status);
        }
        __syncwarp();
    } else {
        const int quad = warp & 3;
        const int kw = (warp - kKvSoftmaxWarp0) >> 2;  // key half of the block handled by this group
        const int row = 32 * quad + lane;     // row of the 128-row item
        const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
        bool ok = true;
        // per-item row statistics, fetched one item ahead
        auto fetch = [&](int j, float& off, float& dneg, float& w, int& tok, bool& diag) {
            const int c = list[j / MT], i = j % MT;
            const int r_unit = 128 * i + row;
            tok = r_unit / G;
            const int g = r_unit % G;
            const long ri = ((long)b * a.Hq + h * G + g) * a.n + c * kBS + tok;
            diag = (c == m);
            const long n_units = (long)a.B * a.Hkv * a.Cq;
            const bool inb = SAS_IN_BOUNDS((ubase + c) * a.Cq + m, n_units * a.Cq, a.status) &&
                             SAS_IN_BOUNDS(ri, (long)a.B * a.Hq * a.n, a.status);
            const float lg =
                (diag || !inb) ? 0.f
                               : gate_log(a.s[(ubase + c) * a.Cq + m],
                                          gate_softmax_family(a.gate) ? a.lse_s[ubase + c] : 0.f, a.gate);
            off = (gate_in_logits(a.gate) ? lg * kLog2e : 0.f) - (inb ? a.lse[ri] : 0.f) * kLog2e;
            dneg = inb ? -a.Dbuf[ri] : 0.f;
            w = (kOuter && !diag) ? expf(lg) : 1.f;
        };
        float off = 0.f, dneg = 0.f, w = 1.f;
        int tok = 0;
        bool diag = false;
        if (nitems > 0) fetch(0, off, dneg, w, tok, diag);
        const uint32_t rbase = (uint32_t)row * 128u;
        for (int j = 0; j < nitems; ++j) {
            const int buf = j & 1;
            float n_off = 0.f, n_dneg = 0.f, n_w = 1.f;
            int n_tok = 0;
            bool n_diag = false;
            if (j + 1 < nitems) fetch(j + 1, n_off, n_dneg, n_w, n_tok, n_diag);
            // P from S alone, published before dP is read
            if (!warp_wait(s_full(buf), (j >> 1) & 1, abort_flag, a.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float p[32];
            uint32_t pk[16];
            {
                const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), off2 = f2_pack(off, off);
                uint32_t sr[32];
                tmem_ld32_sync(tmem + lane_off + buf * 128 + 32 * kw, sr);
                tc_fence_before();
                mbar_arrive(s_free(buf));
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * jj]), __uint_as_float(sr[2 * jj + 1])), sc2, off2),
                              x0, x1);
                    float p0 = ex2(x0), p1 = ex2(x1);
                    if (diag) {
                        const int key = 32 * kw + 2 * jj;
                        if (key > tok) p0 = 0.f;
                        if (key + 1 > tok) p1 = 0.f;
                    }
                    p[2 * jj] = p0;
                    p[2 * jj + 1] = p1;
                    pk[jj] = kOuter ? pack_bf16x2(p0 * w, p1 * w) : pack_bf16x2(p0, p1);
                }
            }
            // the P buffer is free once the dV MMAs of item j-1 completed
            if (j > 0 && !warp_wait(p_done, (j - 1) & 1, abort_flag, a.status)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int chunk = 4 * kw + ch;  // 16-byte chunk = 8 keys
                const uint32_t sw = (uint32_t)((chunk ^ (row & 7)) * 16);
                st_shared_v4(sP + rbase + sw, pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(p_ready);
            // dS = P (w dP - D)
            if (!warp_wait(dp_full(buf), (j >> 1) & 1, abort_flag, a.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                const uint64_t dn2 = f2_pack(dneg, dneg), w2 = f2_pack(w, w);
                uint32_t dr[32];
                tmem_ld32_sync(tmem + lane_off + buf * 128 + 64 + 32 * kw, dr);
                tc_fence_before();
                mbar_arrive(dp_free(buf));
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    float d0, d1;
                    f2_unpack(f2_mul(f2_pack(p[2 * jj], p[2 * jj + 1]),
                                     f2_fma(f2_pack(__uint_as_float(dr[2 * jj]), __uint_as_float(dr[2 * jj + 1])), w2, dn2)),
                              d0, d1);
                    pk[jj] = pack_bf16x2(d0, d1);
                }
            }
            off = n_off;
            dneg = n_dneg;
            w = n_w;
            tok = n_tok;
            diag = n_diag;
            // the dS buffer is free once the dK MMAs of item j-1 completed
            if (j > 0 && !warp_wait(ds_done, (j - 1) & 1, abort_flag, a.status)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int chunk = 4 * kw + ch;
                const uint32_t sw = (uint32_t)((chunk ^ (row & 7)) * 16);
                st_shared_v4(sDS + rbase + sw, pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(ds_ready);
        }
        if (ok && warp_wait(final_bar, 0, abort_flag, a.status)) {
            tc_fence_after();
            // group 0 writes dv, group 1 dk, each the sum of its two row-half
            // accumulators; TMEM lane = head-dim index
            const int d = 32 * quad + lane;
            __nv_bfloat16* dst = kw == 0 ? a.dv : a.dk;
            const float mul = kw == 0 ? 1.f : a.scale;
#pragma unroll 1
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t r0[32], r1[32];
                tmem_ld32x2_sync(tmem + lane_off + 256 + kw * 128 + ch * 32, tmem + lane_off + 320 + kw * 128 + ch * 32,
                                 r0, r1);
#pragma unroll
                for (int jx = 0; jx < 32; ++jx) {
                    const int key = ch * 32 + jx;
                    const long di = (((long)b * a.n + m * kBS + key) * a.Hkv + h) * kD + d;
                    if (SAS_IN_BOUNDS(di, (long)a.B * a.n * a.Hkv * kD, a.status))
                        dst[di] = __float2bfloat16_rn((__uint_as_float(r0[jx]) + __uint_as_float(r1[jx])) * mul);
                }
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

template <typename Kern>
cudaError_t launch_kernel(Kern kern, long grid, int threads, size_t smem, const BwdArgs& a, cudaStream_t stream) {
    if (grid <= 0) return cudaSuccess;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    kern<<<(unsigned)grid, threads, smem, stream>>>(a);
    err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

// bf16 block masses: every query row once per list slot (256-byte multiple)
static size_t bwd_sm100_mass_bytes(const TrainParams& p) {
    const size_t b = sizeof(__nv_bfloat16) * (size_t)p.B * p.Hq * p.n * dq_list_max(p.Cq, p.top_k, p.full_scope, p.gate);
    return (b + 255) & ~(size_t)255;
}

// MT: 128-row tiles per CTA of the dq kernel (2 MT query heads, hsplit CTAs per
// query block); MK: 128-row items per query block of the dk/dv kernel (G = 2 MK).
template <int MT, int MK>
cudaError_t launch_mt(const TrainParams& p, int hsplit, cudaStream_t stream) {
    constexpr int G = 2 * MK;
    BwdArgs a;
    memset(&a, 0, sizeof(a));
    const long rows = (long)p.B * p.n;
    const long grid = (long)p.B * p.Hkv * p.Cq;
    a.hsplit = hsplit;
    a.s = p.s;
    a.lse_s = p.lse_s;
    a.idx = p.idx;
    a.lse = p.lse_in;
    a.Dbuf = p.Dbuf;
    a.Mbuf = static_cast<__nv_bfloat16*>(p.Mbuf);
    a.Cbuf = reinterpret_cast<float*>(static_cast<uint8_t*>(p.Mbuf) + bwd_sm100_mass_bytes(p));
    a.o = static_cast<const __nv_bfloat16*>(p.o_in);
    a.dO = static_cast<const __nv_bfloat16*>(p.dO);
    a.dq = static_cast<__nv_bfloat16*>(p.dq);
    a.dk = static_cast<__nv_bfloat16*>(p.dk);
    a.dv = static_cast<__nv_bfloat16*>(p.dv);
    a.ds = p.ds;
    a.status = p.status;
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.n = p.n;
    a.Cq = p.Cq;
    a.top_k = p.top_k;
    a.full_scope = p.full_scope;
    a.gate = p.gate;
    a.scale = p.scale;
    a.scale_log2 = p.scale * kLog2e;
    // query-major kernel: the CTA's query heads of the block (64 tokens x 2 MT heads) per box
    if (!encode_tma_rows(&a.tq, p.q, p.Hq, rows, 2 * MT, kBS) ||
        !encode_tma_rows(&a.tdo, p.dO, p.Hq, rows, 2 * MT, kBS) ||
        !encode_tma_rows(&a.tk, p.k, p.Hkv, rows, 1, kBS) || !encode_tma_rows(&a.tv, p.v, p.Hkv, rows, 1, kBS))
        return cudaErrorInvalidValue;
    const int nl = dq_list_max(p.Cq, p.top_k, p.full_scope, p.gate);
    const bool outer = p.gate == kGateOuter;
    const bool st3 = DqLayout<MT, 3>::bytes(nl) <= kSmemLimit;
    const size_t smem = st3 ? DqLayout<MT, 3>::bytes(nl) : DqLayout<MT, 2>::bytes(nl);
    auto kern = st3 ? (outer ? bwd_dq_sm100_kernel<MT, 3, true> : bwd_dq_sm100_kernel<MT, 3, false>)
                    : (outer ? bwd_dq_sm100_kernel<MT, 2, true> : bwd_dq_sm100_kernel<MT, 2, false>);
    cudaError_t err = cudaSuccess;
    if (hsplit > 1 && (err = cudaMemsetAsync(p.ds, 0, sizeof(float) * (size_t)p.B * p.Hkv * p.Cq * p.Cq, stream)) !=
                          cudaSuccess)
        return err;  // the head splits add their shares of ds
    err = launch_kernel(kern, grid * hsplit, kDqThreads, smem, a, stream);
    if (err != cudaSuccess) return err;
    if (p.phase_event && (err = cudaEventRecord(static_cast<cudaEvent_t>(p.phase_event), stream)) != cudaSuccess)
        return err;
    // key-major kernel: 128-row items (128/G tokens x G heads) per box
    if (!encode_tma_rows(&a.tq, p.q, p.Hq, rows, G, 128 / G) || !encode_tma_rows(&a.tdo, p.dO, p.Hq, rows, G, 128 / G))
        return cudaErrorInvalidValue;
    // a third Q stage where the list of attending query blocks leaves room for it
    if (DkvLayout<3>::bytes(p.Cq) <= kSmemLimit)
        return p.gate == kGateOuter
                   ? launch_kernel(bwd_dkdv_sm100_kernel<MK, true, 3>, grid, kKvThreads, DkvLayout<3>::bytes(p.Cq), a, stream)
                   : launch_kernel(bwd_dkdv_sm100_kernel<MK, false, 3>, grid, kKvThreads, DkvLayout<3>::bytes(p.Cq), a, stream);
    return p.gate == kGateOuter
               ? launch_kernel(bwd_dkdv_sm100_kernel<MK, true, 2>, grid, kKvThreads, DkvLayout<2>::bytes(p.Cq), a, stream)
               : launch_kernel(bwd_dkdv_sm100_kernel<MK, false, 2>, grid, kKvThreads, DkvLayout<2>::bytes(p.Cq), a, stream);
}

}  // namespace

static bool bwd_sm100_shape(const TrainParams& p) {
    const int G = p.Hq / p.Hkv;
    return p.is_bf16 && p.d == kD && p.bs == kBS && (G == 2 || G == 4 || G == 8);
}

size_t bwd_sm100_workspace(const TrainParams& p) {
    // the block masses, then one fp32 coefficient per query row
    if (!bwd_sm100_shape(p)) return 0;
    return bwd_sm100_mass_bytes(p) + sizeof(float) * (size_t)p.B * p.Hq * p.n;
}

bool bwd_sm100_supported(const TrainParams& p) {
    if (!bwd_sm100_shape(p) || !p.Mbuf) return false;
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.k) |
                         reinterpret_cast<uintptr_t>(p.v) | reinterpret_cast<uintptr_t>(p.dO) |
                         reinterpret_cast<uintptr_t>(p.dq) | reinterpret_cast<uintptr_t>(p.dk) |
                         reinterpret_cast<uintptr_t>(p.dv) | reinterpret_cast<uintptr_t>(p.o_in);
    if (al & 15u) return false;
    if ((long)p.B * p.n > 0x7fffffffL || (long)p.B * p.Hkv * p.Cq * (p.Hq / p.Hkv == 8 ? 2 : 1) > 0x7fffffffL)
        return false;
    const int nl = dq_list_max(p.Cq, p.top_k, p.full_scope, p.gate);
    return DqLayout<2, 2>::bytes(nl) <= kSmemLimit && DkvLayout<2>::bytes(p.Cq) <= kSmemLimit;
}

cudaError_t launch_bwd_sm100(const TrainParams& p, cudaStream_t stream) {
    const int G = p.Hq / p.Hkv;
    // dq: G = 2 one tile per CTA, G = 4 two, G = 8 two CTAs of two tiles; dk/dv: G / 2 items per block
    if (G == 2) return launch_mt<1, 1>(p, 1, stream);
    if (G == 4) return launch_mt<2, 2>(p, 1, stream);
    return launch_mt<2, 4>(p, 2, stream);
}

}  // namespace sas
