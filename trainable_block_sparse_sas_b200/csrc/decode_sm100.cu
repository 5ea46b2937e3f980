// decode_sm100.cu -- gate-free hard-Top-K decode for bf16 caches, head_dim 128,
// block size 64 (jaehun.me review of SAS, walkthrough Step 6: at inference the
// gate is dropped and only the Top-K blocks plus the current block are attended).
//
// One thread-block cluster of CL CTAs per (sequence, kv head); one launch per
// decode step, no workspace:
//   1. selection (optional, fused): every CTA finds the row's Top-K blocks on its
//      own (a threshold from the threads' maxima, then an exact rank of the few
//      keys above it; ties to the lower index, list ascending); when too many
//      scores tie at the threshold, the cluster's CTAs split the row and run a
//      4-pass 8-bit radix select with candidates merged over distributed shared
//      memory;
//   2. attention: the attended list (current partial block first, then the
//      history blocks) is split over the CTAs; a TMA ring streams each block's K
//      and V (2 x 16 KB, 128-byte swizzle); all 8 consumer warps take every block,
//      each warp 16 tokens and one half of the head dimension: S = q K^T and
//      O += P V on the tensor cores with mma.sync m16n8k16 (the G <= 16 query heads
//      of the group padded to 16 rows), online softmax in registers;
//   3. the CTA's 8 warp partials merge in shared memory, then every CTA merges a
//      slice of the outputs from the cluster's partials over distributed shared
//      memory and writes it to o.
#include <cstring>

#include "kernels.h"
#include "sm100.cuh"
#include "topk_filter.cuh"

namespace sas {
namespace {

using namespace sm100;

// Phase trace (builds with SAS_PHASE_TRACE only): per CTA of the decode kernel,
// %clock64 at the phase boundaries named below, plus one (%globaltimer,
// %clock64) pair at entry and one at exit that put every CTA on one time line
// (a %globaltimer read costs hundreds of cycles, so it is taken only there, by
// threads not on the critical path).
enum TraceSlot {
    kTrEntry = 0, kTrCtx, kTrClusterSync, kTrScores, kTrTau, kTrCand, kTrSelected, kTrFirstBlock, kTrStreamEnd,
    kTrPartial, kTrIncoming, kTrExit, kTrGtEntry, kTrClkEntry, kTrGtExit, kTrClkExit, kTrSmid, kTrCandCount,
    kTrBlocks, kTrGrid = 31
};
#ifdef SAS_PHASE_TRACE
constexpr int kTraceCtas = 1024, kTraceSlots = 32;
__device__ unsigned long long g_trace[kTraceCtas][kTraceSlots];
__device__ __forceinline__ unsigned long long clk64() {
    unsigned long long c;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(c));
    return c;
}
__device__ __forceinline__ void trace_put(int slot, unsigned long long v) {
    const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x;
    if (cta < (unsigned)kTraceCtas) g_trace[cta][slot] = v;
}
#define SAS_TRACE(slot) trace_put((slot), clk64())
#define SAS_TRACE_VALUE(slot, v) trace_put((slot), (unsigned long long)(v))
#else
#define SAS_TRACE(slot) ((void)0)
#define SAS_TRACE_VALUE(slot, v) ((void)0)
#endif

constexpr int kD = 128;
constexpr int kBS = 64;
constexpr int kThreads = 288;  // warp 0: TMA producer; warps 1..8: consumers
constexpr int kStages = 3;
constexpr uint32_t kHalf = 64 * 128;   // 64 rows x 128 B: one 64-wide d slab of a block
constexpr uint32_t kTile = 2 * kHalf;  // a block of K (or V): 16 KB
constexpr uint32_t kStage = 2 * kTile;  // K + V
constexpr int kQLd = 136;              // padded row (bf16 elements) of the q tile in smem

struct DecArgs {
    // contiguous caches as {d, Tmax, B*Hkv}, box {64, 64, 1}; paged pools as
    // {d, Hkv, num_pages * 64}, box {64, 1, 64}; both land as 64 token rows x 128 B
    CUtensorMap tk, tv;
    const __nv_bfloat16* q;
    const int32_t* ctx_len;
    const int32_t* idx;  // mode 0
    const float* s;      // mode 1
    int32_t* idx_out;    // mode 1, nullable
    __nv_bfloat16* o;
    int* status;
    int B, Hq, Hkv, Tmax, top_k, s_cols, mode;  // mode 0: given idx, 1: fused selection, 2: dense
    int vec_scores;  // the score rows are 16-byte aligned (s_cols % 4 == 0, aligned s): one bulk copy
    int list_cap;    // entries of the attended list (shared-memory layout)
    float scale_log2;
    const int32_t* page_table;  // nullptr: contiguous caches
    int pages_per_seq, num_pages;
};

// TMA coordinates of block `blk` of row (b, h): contiguous caches address it by
// token row within the row's slab; a paged pool by the block's page (a page id
// outside the pool, or a block past the table, lands outside the tensor map and
// reads as zeros).
__device__ __forceinline__ int page_of(const DecArgs& a, int b, int blk) {
    if (blk >= a.pages_per_seq) return a.num_pages;
    if (!SAS_IN_BOUNDS((long)b * a.pages_per_seq + blk, (long)a.B * a.pages_per_seq, a.status)) return a.num_pages;
    const int pg = a.page_table[(long)b * a.pages_per_seq + blk];
    return (pg < 0 || pg >= a.num_pages) ? a.num_pages : pg;
}

__device__ __forceinline__ void load_block(const DecArgs& a, uint32_t dst, uint32_t bar, int b, int h, int bh,
                                           int blk, int page) {
    if (a.page_table) {
        const int row0 = page * kBS;
        tma_load_3d(dst, &a.tk, bar, 0, h, row0);
        tma_load_3d(dst + kHalf, &a.tk, bar, 64, h, row0);
        tma_load_3d(dst + kTile, &a.tv, bar, 0, h, row0);
        tma_load_3d(dst + kTile + kHalf, &a.tv, bar, 64, h, row0);
    } else {
        const int row0 = blk * kBS;
        tma_load_3d(dst, &a.tk, bar, 0, row0, bh);
        tma_load_3d(dst + kHalf, &a.tk, bar, 64, row0, bh);
        tma_load_3d(dst + kTile, &a.tv, bar, 0, row0, bh);
        tma_load_3d(dst + kTile + kHalf, &a.tv, bar, 64, row0, bh);
    }
}

struct Layout {
    static constexpr uint32_t kRing = 0;
    static constexpr uint32_t kQ = kRing + kStages * kStage;  // 16 rows x kQLd bf16
    static constexpr uint32_t kBars = kQ + 16 * kQLd * 2;
    static constexpr uint32_t kMisc = kBars + 8 * (2 * kStages + 2);  // abort, bin, above, count, scratch
    static constexpr uint32_t kHist = kMisc + 64;              // 2 x 256 ints
    static constexpr uint32_t kGsum = kHist + 2 * 256 * 4;     // 256 ints
    static constexpr uint32_t kScan = kGsum + 256 * 4;         // 40 ints
    static constexpr uint32_t kCnt = kScan + 40 * 4;           // 2 ints (gt, eq) of this CTA
    static constexpr uint32_t kCpart = kCnt + 16;              // [G][d + 2] floats
    __host__ __device__ static uint32_t list_off(int G) { return kCpart + 4 * (uint32_t)G * (kD + 2); }
    // the slices of merged outputs received from the cluster's CTAs: [CL][per + 2 G] floats
    __host__ __device__ static uint32_t in_off(int G, int list_cap) {
        return (list_off(G) + 4 * (uint32_t)list_cap + 15) & ~15u;
    }
    static size_t bytes(int G, int list_cap, int CL) {
        const int per = (G * kD + CL - 1) / CL;
        return 1024 + in_off(G, list_cap) + 4 * (size_t)CL * (per + 2 * G);
    }
};

// Histogram increment with one shared-memory atomic per distinct bin in the
// warp (scores concentrate in few top-byte bins, so plain atomics serialise).
// Called by whole warps; bin < 0 means "no increment" for this lane.
__device__ __forceinline__ void hist_add_warp(int* hist, int bin) {
    const unsigned same = __match_any_sync(0xffffffffu, bin);
    if (bin >= 0 && (int)(threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
}

__device__ __forceinline__ int block_sum_int(int v, int* scan) {
    int tot;
    block_exclusive_scan(v, scan, &tot);
    return tot;
}

// Exact Top-K of the row's first Cb block scores, computed by this CTA alone
// (every CTA of the cluster derives the same list, so no exchange is needed).
// The row (s_cols <= kSelMax floats) is staged in ring stage 2 by a bulk copy
// issued at kernel entry; warps 1..4 do the work (warps 1..8 for rows of over
// 2048 scores), the others wait at the closing CTA barrier.  Keys are 32-bit
// order keys:
//   1. every thread keeps the two largest keys of its 16-byte vectors;
//   2. one warp takes, per lane, the two largest of the values the selection
//      warps kept for that lane's column, sorts those 64 values (each a distinct
//      score) and reads off the K-th largest: a lower bound tau of the K-th
//      largest score, since K scores reach it;
//   3. every score whose key is at least tau is a candidate (K to a few more on
//      random rows), placed by a warp-wide scan plus one shared atomic per warp;
//   4. candidates are ranked exactly on the unique 64-bit key (order key << 32 |
//      (2^32 - 1 - index)), so equal scores prefer the lower block index (with
//      exactly K candidates every one is chosen), and the K chosen blocks go to
//      list[1 .. K] in ascending order.
// Returns K, or -1 when more than kCandCap scores reach tau (the caller then
// runs the radix select).  Called by every thread of the CTA.
constexpr int kCandCap = 512;
constexpr int kSelWarpsMax = 8;  // warps 1..8
constexpr int kSelMax = (int)(kStage / 4);  // scores a staged row may hold (8192)

__device__ __forceinline__ void sel_bar(int nthreads) { asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory"); }

__device__ __forceinline__ float4 lds_f4(uint32_t saddr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(saddr));
    return v;
}

__device__ __forceinline__ float lds_f32(uint32_t saddr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(saddr));
    return v;
}

constexpr int kSelVecs = kSelMax / 4 / 128;  // 16-byte vectors per selection thread, at most (16)

__device__ int row_topk_staged(const DecArgs& a, int Cb, uint8_t* base, int* list, uint32_t sbar,
                               volatile int* abort_flag) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.top_k;
    const uint32_t sc = smem_u32(base + Layout::kRing + 2 * kStage);
    // scratch in ring stage 1 (stage 0 may hold the prefetched current block)
    uint32_t* tops = reinterpret_cast<uint32_t*>(base + Layout::kRing + kStage);               // [warps][64]
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(tops + kSelWarpsMax * 64);  // [kCandCap]
    unsigned long long* chosen = cand + kCandCap;                                              // [K]
    int* misc = reinterpret_cast<int*>(base + Layout::kMisc);  // [5]: candidates, [6]: tau
    const int nsw = Cb > 2048 ? 8 : 4;  // selection warps (uniform over the CTA)
    const int nst = 32 * nsw;
    if (warp >= 1 && warp <= nsw) {
        const int t = tid - 32, w = warp - 1;
        const int nv = (Cb + 3) / 4;  // vectors holding the first Cb scores; thread t takes t + 128 u
        const bool ok = warp_wait(sbar, 0, abort_flag, a.status);
        if (!ok) mbar_wait_drain(sbar, 0, a.status);  // the copy lands before its stage is reused
        if (t == 0) SAS_TRACE(kTrScores);
        // the vectors of this thread, four at a time (loads in flight together), as
        // 32-bit keys; 0 for no score (every real key is larger)
        auto keys4 = [&](int u0, uint32_t (&k)[16]) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = t + (u0 + u) * nst;
                v[u] = i < nv ? lds_f4(sc + 16u * (uint32_t)i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int m0 = 4 * (t + (u0 + u) * nst);
                const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) k[4 * u + c] = m0 + c < Cb ? order_key(e[c]) : 0u;
            }
        };
        uint32_t k1 = 0u, k2 = 0u, k1b = 0u, k2b = 0u;
        if (ok) {
#pragma unroll
            for (int u0 = 0; u0 < kSelVecs; u0 += 4) {
                if (t + u0 * nst >= nv) break;
                uint32_t k[16];
                keys4(u0, k);
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    top2_insert(k[j], k1, k2);
                    top2_insert(k[j + 1], k1b, k2b);
                }
            }
        }
        top2_insert(k1b, k1, k2);
        top2_insert(k2b, k1, k2);
        tops[w * 64 + lane] = k1;
        tops[w * 64 + 32 + lane] = k2;
        if (t == 0) misc[5] = 0;
        sel_bar(nst);
        if (w == 0) {
            uint32_t c1 = 0u, c2 = 0u;
#pragma unroll
            for (int w2 = 0; w2 < nsw; ++w2) {
                top2_insert(tops[w2 * 64 + lane], c1, c2);
                top2_insert(tops[w2 * 64 + 32 + lane], c1, c2);
            }
            const uint32_t tau = warp_kth_of_64(c1, c2, K - 1);
            if (lane == 0) misc[6] = (int)tau;
        }
        sel_bar(nst);
        if (t == 0) SAS_TRACE(kTrTau);
        const uint32_t tau = (uint32_t)misc[6];
        // candidates of this thread as a bit mask over its (at most 64) scores
        unsigned long long mask = 0ull;
        if (ok) {
#pragma unroll
            for (int u0 = 0; u0 < kSelVecs; u0 += 4) {
                if (t + u0 * nst >= nv) break;
                uint32_t k[16];
                keys4(u0, k);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const bool in_row = 4 * (t + (u0 + (j >> 2)) * nst) + (j & 3) < Cb;
                    mask |= (in_row && k[j] >= tau) ? (1ull << (4 * u0 + j)) : 0ull;
                }
            }
        }
        const int cnt = __popcll(mask);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int wbase = 0;
        if (lane == 31 && incl > 0) wbase = atomicAdd(&misc[5], incl);
        int pos = __shfl_sync(0xffffffffu, wbase, 31) + incl - cnt;
        while (mask) {
            const int bit = __ffsll((long long)mask) - 1;
            mask &= mask - 1;
            const int m = 4 * (t + (bit >> 2) * nst) + (bit & 3);
            const uint32_t k = order_key(lds_f32(sc + 4u * (uint32_t)m));
            if (pos < kCandCap) cand[pos] = ((unsigned long long)k << 32) | (0xFFFFFFFFu - (uint32_t)m);
            ++pos;
        }
        sel_bar(nst);
        const int C = misc[5];
        if (t == 0) {
            SAS_TRACE(kTrCand);
            SAS_TRACE_VALUE(kTrCandCount, C);
        }
        if (C <= kCandCap) {
            // exactly K candidates: all chosen, only their order by index is needed
            const unsigned long long* pick = cand;
            if (C > K) {
                for (int c = t; c < C; c += nst) {
                    const unsigned long long k = cand[c];
                    const int rk = count_larger(cand, C, k);
                    if (rk < K) chosen[rk] = k;
                }
                sel_bar(nst);
                pick = chosen;
            }
            for (int j = t; j < K; j += nst) {
                const uint32_t m = 0xFFFFFFFFu - (uint32_t)(pick[j] & 0xFFFFFFFFull);
                int p0 = 0, p1 = 0, j2 = 0;
                for (; j2 + 2 <= K; j2 += 2) {
                    p0 += (0xFFFFFFFFu - (uint32_t)(pick[j2] & 0xFFFFFFFFull)) < m ? 1 : 0;
                    p1 += (0xFFFFFFFFu - (uint32_t)(pick[j2 + 1] & 0xFFFFFFFFull)) < m ? 1 : 0;
                }
                if (j2 < K) p0 += (0xFFFFFFFFu - (uint32_t)(pick[j2] & 0xFFFFFFFFull)) < m ? 1 : 0;
                list[1 + p0 + p1] = (int)m;
            }
        }
    }
    // generic-proxy accesses to ring stages 1 and 2 before TMA reuses them
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    return misc[5] <= kCandCap ? K : -1;
}

// Fused Top-K over the row's Cb block scores, split across the cluster.
// Fills list[1 .. K] (ascending) in every CTA; returns the number selected.
template <int CL>
__device__ int cluster_topk(const DecArgs& a, int bh, int Cb, uint32_t rank, uint8_t* base, int* list) {
    const int tid = threadIdx.x;
    const int K = a.top_k;
    if (K >= Cb) {
        for (int i = tid; i < Cb; i += kThreads) list[1 + i] = i;
        __syncthreads();
        return Cb;
    }
    int* hist = reinterpret_cast<int*>(base + Layout::kHist);
    int* gsum = reinterpret_cast<int*>(base + Layout::kGsum);
    int* scan = reinterpret_cast<int*>(base + Layout::kScan);
    int* cnt = reinterpret_cast<int*>(base + Layout::kCnt);
    int* misc = reinterpret_cast<int*>(base + Layout::kMisc);
    const float* srow = a.s + (long)bh * a.s_cols;
    const int lo = (int)((long)rank * Cb / CL), hi = (int)((long)(rank + 1) * Cb / CL);
    uint32_t prefix = 0u, pmask = 0u;
    int remaining = K;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        int* hst = hist + (pass & 1) * 256;
        if (tid < 256) hst[tid] = 0;
        __syncthreads();
        for (int m0 = lo; m0 < hi; m0 += kThreads) {
            const int m = m0 + tid;
            int bin = -1;
            if (m < hi) {
                const uint32_t key = order_key(srow[m]);
                if ((key & pmask) == prefix) bin = (int)((key >> shift) & 255u);
            }
            hist_add_warp(hst, bin);
        }
        cluster_sync();
        if (tid < 256) {
            const uint32_t local = smem_u32(&hst[tid]);
            int tot = 0;
#pragma unroll
            for (int r = 0; r < CL; ++r) tot += (int)ld_dsmem_u32(mapa(local, (uint32_t)r));
            gsum[tid] = tot;
        }
        __syncthreads();
        if (tid < 32) {
            int c8[8], sum = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                c8[q] = gsum[255 - (tid * 8 + q)];
                sum += c8[q];
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
                    if (acc + c8[q] >= remaining) {
                        misc[1] = 255 - (tid * 8 + q);
                        misc[2] = acc;
                        break;
                    }
                    acc += c8[q];
                }
            }
        }
        __syncthreads();
        prefix |= (uint32_t)misc[1] << shift;
        pmask |= 0xFFu << shift;
        remaining -= misc[2];
        __syncthreads();
    }
    // counts above / equal to the threshold key in this CTA's slice
    int gt = 0, eq = 0;
    for (int m = lo + tid; m < hi; m += kThreads) {
        const uint32_t key = order_key(srow[m]);
        gt += key > prefix;
        eq += key == prefix;
    }
    gt = block_sum_int(gt, scan);
    eq = block_sum_int(eq, scan);
    if (tid == 0) {
        cnt[0] = gt;
        cnt[1] = eq;
    }
    cluster_sync();
    // this CTA's output base and its share of the threshold-equal keys (lowest indices first)
    int base_pos = 0, eq_before = 0;
    for (int r = 0; r < (int)rank; ++r) {
        const int g_r = (int)ld_dsmem_u32(mapa(smem_u32(&cnt[0]), (uint32_t)r));
        const int e_r = (int)ld_dsmem_u32(mapa(smem_u32(&cnt[1]), (uint32_t)r));
        base_pos += g_r + max(0, min(e_r, remaining - eq_before));
        eq_before += e_r;
    }
    const int eq_quota = max(0, min(eq, remaining - eq_before));
    int out = base_pos, eq_seen = 0;
    for (int m0 = lo; m0 < hi; m0 += kThreads) {
        const int m = m0 + tid;
        const uint32_t key = m < hi ? order_key(srow[m]) : 0u;
        const int is_eq = (m < hi && key == prefix) ? 1 : 0;
        int tot_eq;
        const int eq_rank = block_exclusive_scan(is_eq, scan, &tot_eq) + eq_seen;
        const int take = (m < hi && (key > prefix || (is_eq && eq_rank < eq_quota))) ? 1 : 0;
        int tot_take;
        const int pos = block_exclusive_scan(take, scan, &tot_take) + out;
        if (take && pos < K) {
            const uint32_t local = smem_u32(&list[1 + pos]);
#pragma unroll
            for (int r = 0; r < CL; ++r) st_dsmem_u32(mapa(local, (uint32_t)r), (uint32_t)m);
        }
        eq_seen += tot_eq;
        out += tot_take;
    }
    cluster_sync();
    return K;
}

// Local exact Top-K of this CTA's slice of the score row (keys staged in ring
// stage 1), candidates sent to CTA 0 (ring stage 2) over distributed shared
// memory; CTA 0 ranks the <= CL*K candidates by (score desc, index asc) and
// writes the chosen blocks, ascending, into every CTA's list[1 .. K].
// Needs a slice of <= kStage/4 keys and CL*K <= kStage/8 candidates.
template <int CL>
__device__ int cluster_topk_fast(const DecArgs& a, int bh, int Cb, uint32_t rank, uint8_t* base, int* list) {
    const int tid = threadIdx.x;
    const int K = a.top_k;
    uint32_t* keys = reinterpret_cast<uint32_t*>(base + Layout::kRing + kStage);
    uint32_t* cand = reinterpret_cast<uint32_t*>(base + Layout::kRing + 2 * kStage);  // [CL*K][2] on CTA 0
    int* hist = reinterpret_cast<int*>(base + Layout::kHist);
    int* gsum = reinterpret_cast<int*>(base + Layout::kGsum);  // [0..CL) candidate counts on CTA 0
    int* scan = reinterpret_cast<int*>(base + Layout::kScan);
    int* misc = reinterpret_cast<int*>(base + Layout::kMisc);
    const float* srow = a.s + (long)bh * a.s_cols;
    const int lo = (int)((long)rank * Cb / CL), hi = (int)((long)(rank + 1) * Cb / CL), n = hi - lo;
    for (int i = tid; i < n; i += kThreads) keys[i] = order_key(srow[lo + i]);
    if (tid == 0) misc[4] = 0;
    __syncthreads();
    uint32_t thr = 0u;   // keys above thr are taken; `rem` keys equal to thr, lowest index first
    int rem = 0, gt = n;
    if (n > K) {
        uint32_t prefix = 0u, pmask = 0u;
        int remaining = K;
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            if (tid < 256) hist[tid] = 0;
            __syncthreads();
            for (int i0 = 0; i0 < n; i0 += kThreads) {
                const int i = i0 + tid;
                int bin = -1;
                if (i < n) {
                    const uint32_t key = keys[i];
                    if ((key & pmask) == prefix) bin = (int)((key >> shift) & 255u);
                }
                hist_add_warp(hist, bin);
            }
            __syncthreads();
            if (tid < 32) {
                int c8[8], sum = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    c8[q] = hist[255 - (tid * 8 + q)];
                    sum += c8[q];
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
                        if (acc + c8[q] >= remaining) {
                            misc[1] = 255 - (tid * 8 + q);
                            misc[2] = acc;
                            break;
                        }
                        acc += c8[q];
                    }
                }
            }
            __syncthreads();
            prefix |= (uint32_t)misc[1] << shift;
            pmask |= 0xFFu << shift;
            remaining -= misc[2];
            __syncthreads();
        }
        thr = prefix;
        rem = remaining;
        gt = K - remaining;
    }
    // every CTA of the cluster is running before its shared memory is written remotely
    cluster_sync();
    // send candidates (key, block index) to CTA 0: all keys above thr, and the
    // `rem` lowest-index keys equal to thr (ordered scan only when that matters)
    const uint32_t cand0 = smem_u32(cand), cnt0 = smem_u32(gsum);
    auto send = [&](int slot, uint32_t key, int m) {
        const uint32_t dst = mapa(cand0 + 8u * (uint32_t)(rank * K + slot), 0u);
        st_dsmem_u32(dst, key);
        st_dsmem_u32(dst + 4u, (uint32_t)m);
    };
    if (n <= K) {
        for (int i = tid; i < n; i += kThreads) send(i, keys[i], lo + i);
        if (tid == 0) st_dsmem_u32(mapa(cnt0 + 4u * rank, 0u), (uint32_t)n);
    } else {
        int eq = 0;
        for (int i = tid; i < n; i += kThreads) eq += keys[i] == thr;
        int eq_tot;
        block_exclusive_scan(eq, scan, &eq_tot);
        if (eq_tot <= rem) {
            for (int i = tid; i < n; i += kThreads)
                if (keys[i] >= thr) send(atomicAdd(&misc[4], 1), keys[i], lo + i);
        } else {
            int out = 0, eq_seen = 0;
            for (int i0 = 0; i0 < n; i0 += kThreads) {
                const int i = i0 + tid;
                const uint32_t key = i < n ? keys[i] : 0u;
                const int is_eq = (i < n && key == thr) ? 1 : 0;
                int te;
                const int er = block_exclusive_scan(is_eq, scan, &te) + eq_seen;
                const int take = (i < n && (key > thr || (is_eq && er < rem))) ? 1 : 0;
                int tt;
                const int pos = block_exclusive_scan(take, scan, &tt) + out;
                if (take) send(pos, key, lo + i);
                eq_seen += te;
                out += tt;
            }
        }
        if (tid == 0) st_dsmem_u32(mapa(cnt0 + 4u * rank, 0u), (uint32_t)(gt + rem));
    }
    cluster_sync();
    if (rank == 0 && K <= 32) {
        // Each list (<= 32 candidates, one per lane) is sorted by warp `r` on the
        // 64-bit key (order key, then the complement of the index: larger = better,
        // equal scores resolve to the lower index).  A candidate's rank is its place in
        // its own list plus, for every other list, how many entries beat it (binary
        // search); ranks are unique, so the chosen K fill slots 0..K-1.
        unsigned long long* sorted = reinterpret_cast<unsigned long long*>(keys);  // [CL][32]
        unsigned long long* chosen = sorted + CL * 32;                              // [K]
        const int w = tid >> 5, ln = tid & 31;
        if (w < CL) {
            const int c = gsum[w];
            unsigned long long v = 0ull;
            if (ln < c) {
                const int s = w * K + ln;
                v = ((unsigned long long)cand[2 * s] << 32) | (0xFFFFFFFFu - cand[2 * s + 1]);
            }
#pragma unroll
            for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
                for (int j = k >> 1; j > 0; j >>= 1) {
                    const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, j);
                    const bool desc = (ln & k) == 0;  // overall order: descending
                    const bool lower = (ln & j) == 0;
                    const bool keep_max = (lower == desc);
                    v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
                }
            }
            sorted[w * 32 + ln] = v;
        }
        __syncthreads();
        for (int s = tid; s < CL * 32; s += kThreads) {
            const int r = s >> 5, pidx = s & 31;
            if (pidx >= gsum[r]) continue;
            const unsigned long long key = sorted[s];
            int rk = pidx;
            for (int r2 = 0; r2 < CL; ++r2) {
                if (r2 == r) continue;
                int lo2 = 0, hi2 = gsum[r2];  // count entries of list r2 greater than key
                while (lo2 < hi2) {
                    const int mid = (lo2 + hi2) >> 1;
                    if (sorted[r2 * 32 + mid] > key) lo2 = mid + 1;
                    else hi2 = mid;
                }
                rk += lo2;
            }
            if (rk < K) chosen[rk] = key;
        }
        __syncthreads();
        for (int j = tid; j < K; j += kThreads) {
            const uint32_t m = 0xFFFFFFFFu - (uint32_t)(chosen[j] & 0xFFFFFFFFull);
            int pos = 0;
            for (int j2 = 0; j2 < K; ++j2) pos += (0xFFFFFFFFu - (uint32_t)(chosen[j2] & 0xFFFFFFFFull)) < m;
            const uint32_t local = smem_u32(&list[1 + pos]);
#pragma unroll
            for (int r = 0; r < CL; ++r) st_dsmem_u32(mapa(local, (uint32_t)r), m);
        }
    } else if (rank == 0) {
        // a candidate is chosen when fewer than K candidates beat it; its place in the
        // ascending list is the number of chosen candidates with a lower index
        const int N = CL * K;
        int* chosen = reinterpret_cast<int*>(keys);  // reuse stage 1: [N] flags
        for (int s = tid; s < N; s += kThreads) {
            const int r = s / K;
            int ok = 0;
            if (s - r * K < gsum[r]) {
                const uint32_t key = cand[2 * s], m = cand[2 * s + 1];
                int beats = 0;
                for (int r2 = 0; r2 < CL; ++r2)
                    for (int s2 = r2 * K; s2 < r2 * K + gsum[r2]; ++s2) {
                        const uint32_t k2 = cand[2 * s2], m2 = cand[2 * s2 + 1];
                        beats += (k2 > key) || (k2 == key && m2 < m);
                    }
                ok = beats < K;
            }
            chosen[s] = ok;
        }
        __syncthreads();
        for (int s = tid; s < N; s += kThreads) {
            if (!chosen[s]) continue;
            const uint32_t m = cand[2 * s + 1];
            int pos = 0;
            for (int s2 = 0; s2 < N; ++s2) pos += chosen[s2] && cand[2 * s2 + 1] < m;
            const uint32_t local = smem_u32(&list[1 + pos]);
#pragma unroll
            for (int r = 0; r < CL; ++r) st_dsmem_u32(mapa(local, (uint32_t)r), m);
        }
    }
    // generic-proxy writes to ring stages 1 and 2 before TMA reuses them
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    cluster_sync();
    return K;
}

template <int CL>
__global__ void __launch_bounds__(kThreads, 2) decode_cluster_kernel(const __grid_constant__ DecArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_align1024(smem_raw);
    const uint32_t sbase = smem_u32(base);
    const uint32_t ring = sbase + Layout::kRing;
    const uint32_t bar0 = sbase + Layout::kBars;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (kStages + s); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base + Layout::kMisc);
    const int G = a.Hq / a.Hkv;
    float* cpart = reinterpret_cast<float*>(base + Layout::kCpart);
    int* list = reinterpret_cast<int*>(base + Layout::list_off(G));
    __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(base + Layout::kQ);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int bh = blockIdx.y;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const uint32_t sbar = bar0 + 8u * (2 * kStages), inbar = sbar + 8u;
    // merged outputs: CTA r finishes outputs [r per, (r + 1) per) of the G*128;
    // every CTA sends it that slice of its partial plus its (max, sum) per head
    const int per = (G * kD + CL - 1) / CL, in_len = per + 2 * G;
    float* incoming = reinterpret_cast<float*>(base + Layout::in_off(G, a.list_cap));  // [CL][in_len]
    // fused selection: the row's scores (every one of its s_cols; those past the
    // history are masked later) are requested first, by one bulk copy into ring
    // stage 2, independently of ctx_len
    const bool staged = a.mode == 1 && a.vec_scores && a.s_cols > 0 && a.s_cols <= kSelMax;
    if (tid == 0) SAS_TRACE(kTrEntry);
    if (tid == kThreads - 1) {
        SAS_TRACE(kTrClkEntry);
        SAS_TRACE_VALUE(kTrGtEntry, globaltimer());
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 8);
        }
        mbar_init(sbar, 1);
        mbar_init(inbar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        if (staged) {
            const uint32_t bytes = 4u * (uint32_t)a.s_cols;
            const long off = (long)bh * a.s_cols;
            mbar_arrive_expect_tx(sbar, bytes);
            if (SAS_IN_BOUNDS(off + a.s_cols - 1, (long)a.B * a.Hkv * a.s_cols, a.status))
                bulk_load(ring + 2 * kStage, a.s + off, bytes, sbar);
        }
        // the pushes of the other CTAs' partials complete this phase
        mbar_arrive_expect_tx(inbar, 4u * (uint32_t)((CL - 1) * in_len));
        prefetch_tmap(&a.tk);
        prefetch_tmap(&a.tv);
    }
    int T = a.ctx_len[b];
    T = max(1, min(T, a.Tmax));
    if (tid == 0) SAS_TRACE(kTrCtx);
    const int t = T - 1, Cb = t / kBS;
    const int Csel = min(Cb, a.s_cols);
    const bool use_filter = staged && a.top_k < Csel && a.top_k <= 64;
    // q of the group, padded to 16 rows: one 16-byte load per thread
    if (tid < 16 * kD / 8) {
        const int r = tid / (kD / 8), e = (tid % (kD / 8)) * 8;
        const long qi = ((long)b * a.Hq + h * G + r) * kD + e;
        const uint4 val = r < G && SAS_IN_BOUNDS(qi + 7, (long)a.B * a.Hq * kD, a.status)
                              ? *reinterpret_cast<const uint4*>(a.q + qi)
                              : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(qs + r * kQLd + e) = val;
    }
    // every CTA of the cluster has initialised its barriers and is running before
    // any shared memory or barrier of it is used remotely (also a CTA barrier)
    cluster_sync();
    if (tid == 0) SAS_TRACE(kTrClusterSync);
    // attended list: entry 0 = current (partial) block, entries 1.. = history blocks ascending
    int nsel;
    if (a.mode == 2) {
        nsel = Cb;
    } else if (a.mode == 0) {
        // the valid prefix of the ascending, -1 padded row: entries before the first
        // one outside [0, Cb)
        int* misc = reinterpret_cast<int*>(base + Layout::kMisc);
        if (tid == 0) misc[3] = a.top_k;
        __syncthreads();
        const int32_t* row = a.idx + (long)bh * a.top_k;
        for (int c = tid; c < a.top_k; c += kThreads) {
            const int v = SAS_IN_BOUNDS((long)bh * a.top_k + c, (long)a.B * a.Hkv * a.top_k, a.status) ? row[c] : -1;
            list[1 + c] = v;
            if (v < 0 || v >= Cb) atomicMin(&misc[3], c);
        }
        __syncthreads();
        nsel = misc[3];
    } else {
        // the current block (entry 0, on CTA 0) loads while the selection runs
        if (rank == 0 && tid == 0) {
            mbar_arrive_expect_tx(full(0), kStage);
            load_block(a, ring, full(0), b, h, bh, Cb, a.page_table ? page_of(a, b, Cb) : 0);
        }
        // the staged row must have landed before ring stage 2 is used otherwise
        if (staged && !use_filter && !warp_wait(sbar, 0, abort_flag, a.status)) mbar_wait_drain(sbar, 0, a.status);
        const int chunk = (Csel + CL - 1) / CL;
        nsel = use_filter ? row_topk_staged(a, Csel, base, list, sbar, abort_flag) : -1;
        if (nsel < 0) {
            if (a.top_k < Csel && chunk <= (int)(kStage / 4) && CL * a.top_k <= (int)(kStage / 8))
                nsel = cluster_topk_fast<CL>(a, bh, Csel, rank, base, list);
            else
                nsel = cluster_topk<CL>(a, bh, Csel, rank, base, list);
        }
        if (rank == 0 && a.idx_out)
            for (int i = tid; i < a.top_k; i += kThreads)
                if (SAS_IN_BOUNDS((long)bh * a.top_k + i, (long)a.B * a.Hkv * a.top_k, a.status))
                    a.idx_out[(long)bh * a.top_k + i] = i < nsel ? list[1 + i] : -1;
    }
    if (tid == 0) SAS_TRACE(kTrSelected);
    const int L = nsel + 1;
    // ceil split: CTA 0 always owns entry 0 (the current block, prefetched in mode 1)
    const int e0 = (int)(((long)rank * L + CL - 1) / CL), e1 = (int)(((long)(rank + 1) * L + CL - 1) / CL);
    auto block_of = [&](int e) { return e == 0 ? Cb : (a.mode == 2 ? e - 1 : list[e]); };

    if (warp == 0) {
        // lane 0 issues the loads; with a paged pool the warp first reads the next 32
        // entries' page ids together (one round trip), so the table lookups do not
        // serialise the stream
        const int first = (a.mode == 1 && rank == 0) ? 1 : 0;  // entry 0 already in flight
        bool ok = true;
        for (int i0 = first; ok && e0 + i0 < e1; i0 += 32) {
            int my_page = 0;
            if (a.page_table && e0 + i0 + lane < e1) my_page = page_of(a, b, block_of(e0 + i0 + lane));
            for (int j = 0; j < 32 && e0 + i0 + j < e1; ++j) {
                const int page = __shfl_sync(0xffffffffu, my_page, j);
                if (lane == 0) {
                    const int i = i0 + j, st = i % kStages;
                    if (i >= kStages && !mbar_wait(empty(st), (i / kStages - 1) & 1, abort_flag, a.status)) ok = false;
                    if (ok) {
                        mbar_arrive_expect_tx(full(st), kStage);
                        load_block(a, ring + st * kStage, full(st), b, h, bh, block_of(e0 + i), page);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
    } else {
        // Every consumer warp takes every block of this CTA (one in-order consumer
        // sequence per ring stage, so parity waits are exact): warp cw covers
        // tokens [16 wg, 16 wg + 16) of the block and head-dim half dh of O.
        const int cw = warp - 1;   // 0..7
        const int wg = cw & 3;     // 16-token slice of the block
        const int dh = cw >> 2;    // 64-wide half of the head dimension for P V
        const int r0 = lane >> 2;  // fragment rows r0 and r0 + 8 (query heads)
        const int cq = lane & 3;
        float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
        float O[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) O[nt][0] = O[nt][1] = O[nt][2] = O[nt][3] = 0.f;
        const uint32_t qbase = smem_u32(qs);
        for (int i = 0; e0 + i < e1; ++i) {
            const int st = i % kStages;
            if (!warp_wait(full(st), (i / kStages) & 1, abort_flag, a.status)) break;
            if (i == 0 && tid == 32) SAS_TRACE(kTrFirstBlock);
            const int blk = block_of(e0 + i);
            const uint32_t kb = ring + st * kStage, vb = kb + kTile;
            const int tok0 = blk * kBS + 16 * wg;  // absolute first token of this warp's slice
            const bool partial = tok0 + 15 > t;
            if (partial) {  // partial block: zero this warp's V rows past the query (their P is 0)
                if (lane < 16 && tok0 + lane > t) {
                    uint8_t* row = base + Layout::kRing + st * kStage + kTile + dh * kHalf + (16 * wg + lane) * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) reinterpret_cast<uint4*>(row)[c] = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }
            float sacc[2][4] = {};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t qa[4];
                {
                    // A = q rows (16) x d (16kk .. 16kk+15)
                    const int rr = (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int cc = 16 * kk + (lane >> 4) * 8;
                    ldmatrix_x4(qbase + (uint32_t)(rr * kQLd + cc) * 2u, qa[0], qa[1], qa[2], qa[3]);
                }
                const int half = kk >> 2, ch = (kk & 3) * 2 + ((lane >> 3) & 1);
                const int j = 16 * wg + ((lane >> 4) & 1) * 8 + (lane & 7);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(kb + half * kHalf + j * 128 + ((ch ^ (j & 7)) << 4), b0, b1, b2, b3);
                mma_16816(sacc[0], qa, b0, b1);
                mma_16816(sacc[1], qa, b2, b3);
            }
            // scores in log2 units; mask tokens past the query
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = tok0 + 8 * nt + 2 * cq + (e & 1);
                    float v = sacc[nt][e] * a.scale_log2;
                    if (tok > t) v = -INFINITY;
                    sacc[nt][e] = v;
                    mx[e >> 1] = fmaxf(mx[e >> 1], v);
                }
            float alpha[2], mref[2];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
                mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
                const float mnew = fmaxf(m_r[rr], mx[rr]);
                mref[rr] = mnew == -INFINITY ? 0.f : mnew;
                alpha[rr] = ex2(m_r[rr] - mref[rr]);
                m_r[rr] = mnew;
            }
            float p[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) p[nt][e] = ex2(sacc[nt][e] - mref[e >> 1]);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) l_r[rr] *= alpha[rr];
            l_r[0] += p[0][0] + p[0][1] + p[1][0] + p[1][1];
            l_r[1] += p[0][2] + p[0][3] + p[1][2] + p[1][3];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                O[nt][0] *= alpha[0];
                O[nt][1] *= alpha[0];
                O[nt][2] *= alpha[1];
                O[nt][3] *= alpha[1];
            }
            uint32_t pa[4];
            pa[0] = pack_bf16x2(p[0][0], p[0][1]);
            pa[1] = pack_bf16x2(p[0][2], p[0][3]);
            pa[2] = pack_bf16x2(p[1][0], p[1][1]);
            pa[3] = pack_bf16x2(p[1][2], p[1][3]);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                const int ch = 2 * np + (lane >> 4);
                const int j = 16 * wg + ((lane >> 3) & 1) * 8 + (lane & 7);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(vb + dh * kHalf + j * 128 + ((ch ^ (j & 7)) << 4), b0, b1, b2, b3);
                mma_16816(O[2 * np], pa, b0, b1);
                mma_16816(O[2 * np + 1], pa, b2, b3);
            }
            // generic-proxy writes (the zeroed rows) before the stage goes back to TMA
            if (partial) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(st));
        }
        if (tid == 32) SAS_TRACE(kTrStreamEnd);
        // row sums over the 4 lanes sharing a row
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 1);
            l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 2);
        }
        // warp partials into the (now idle) ring: [warp][G][d + 2], this warp's d half only
        asm volatile("bar.sync 1, 256;" ::: "memory");
        float* wpart = reinterpret_cast<float*>(base + Layout::kRing);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int g = r0 + 8 * rr;
            if (g < G) {
                float* dst = wpart + ((long)cw * G + g) * (kD + 2);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    dst[64 * dh + 8 * nt + 2 * cq] = O[nt][2 * rr];
                    dst[64 * dh + 8 * nt + 2 * cq + 1] = O[nt][2 * rr + 1];
                }
                if (cq == 0) {
                    dst[kD] = m_r[rr];
                    dst[kD + 1] = l_r[rr];
                }
            }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        // merge the 4 token slices -> this CTA's partial (d < 128: warps of that d half;
        // the running sum: the warps of half 0, which saw the same scores)
        for (int i = tid - 32; i < G * (kD + 1); i += 256) {
            const int g = i / (kD + 1), d = i % (kD + 1);
            const int wbase = d < kD ? 4 * (d >> 6) : 0;
            float M = -INFINITY;
            for (int w = 0; w < 4; ++w) M = fmaxf(M, wpart[((long)(wbase + w) * G + g) * (kD + 2) + kD]);
            float acc = 0.f;
            if (M != -INFINITY) {
                for (int w = 0; w < 4; ++w) {
                    const float* src = wpart + ((long)(wbase + w) * G + g) * (kD + 2);
                    const float f = ex2(src[kD] - M);
                    acc += (d < kD ? src[d] : src[kD + 1]) * f;
                }
            }
            if (d < kD) cpart[g * (kD + 2) + d] = acc;
            else {
                cpart[g * (kD + 2) + kD] = M;
                cpart[g * (kD + 2) + kD + 1] = acc;
            }
        }
    }
    __syncwarp();
    // every CTA's partial is complete (CTA barrier); CTA o gets the slice o of the
    // numerators and the per-head (max, sum) of every CTA, its own by plain stores,
    // the others' by remote stores that complete the bytes its barrier expects
    __syncthreads();
    if (tid == 0) {
        SAS_TRACE(kTrPartial);
        SAS_TRACE_VALUE(kTrBlocks, e1 - e0);
    }
    for (int j = tid; j < CL * in_len; j += kThreads) {
        const int o = j / in_len, e = j - o * in_len;
        float v;
        if (e < per) {
            const int i = o * per + e;
            v = i < G * kD ? cpart[(i / kD) * (kD + 2) + i % kD] : 0.f;
        } else {
            const int q2 = e - per;  // maxima of heads 0..G-1, then their sums
            v = cpart[(q2 % G) * (kD + 2) + kD + (q2 >= G ? 1 : 0)];
        }
        float* slot = incoming + (int)rank * in_len + e;
        if (o == (int)rank) *slot = v;
        else st_async_b32(mapa(smem_u32(slot), (uint32_t)o), __float_as_uint(v), mapa(inbar, (uint32_t)o));
    }
    // wait (ignoring the abort flag: no CTA leaves while others may still write to
    // its shared memory) for the other CTAs' slices
    const bool got = mbar_wait_drain(inbar, 0, a.status, 4 * kWaitLimitNs);
    __syncthreads();
    if (tid == 0) SAS_TRACE(kTrIncoming);
    if (got) {
        const int o0 = (int)rank * per, o1 = min(G * kD, o0 + per);
        for (int i = o0 + tid; i < o1; i += kThreads) {
            const int e = i - o0, g = i / kD, d = i % kD;
            float M = -INFINITY;
#pragma unroll
            for (int r = 0; r < CL; ++r) M = fmaxf(M, incoming[r * in_len + per + g]);
            float n_ = 0.f, d_ = 0.f;
#pragma unroll
            for (int r = 0; r < CL; ++r) {
                const float mr = incoming[r * in_len + per + g];
                if (mr == -INFINITY) continue;
                const float f = ex2(mr - M);
                n_ += incoming[r * in_len + e] * f;
                d_ += incoming[r * in_len + per + G + g] * f;
            }
            const long oi = ((long)b * a.Hq + h * G + g) * kD + d;
            if (SAS_IN_BOUNDS(oi, (long)a.B * a.Hq * kD, a.status)) a.o[oi] = __float2bfloat16_rn(n_ / d_);
        }
    }
    if (tid == 0) {
        SAS_TRACE(kTrExit);
        SAS_TRACE(kTrClkExit);
        SAS_TRACE_VALUE(kTrGtExit, globaltimer());
        SAS_TRACE_VALUE(kTrGrid, gridDim.x * gridDim.y);
        unsigned smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        SAS_TRACE_VALUE(kTrSmid, smid);
    }
}

// The same grid, cluster, block and shared memory as decode_cluster_kernel<CL>,
// doing nothing: its launch time is the floor under the decode's.
template <int CL>
__global__ void __launch_bounds__(kThreads, 2) decode_floor_kernel(const __grid_constant__ DecArgs a) {
    extern __shared__ uint8_t smem_raw[];
    (void)a;
    (void)smem_raw;
}

bool encode_cache(CUtensorMap* map, const void* ptr, int Tmax, long rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)Tmax, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)Tmax * kD * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CL, bool kFloor>
cudaError_t launch_cl(const DecArgs& a, int list_cap, cudaStream_t stream) {
    const int G = a.Hq / a.Hkv;
    const size_t smem = Layout::bytes(G, list_cap, CL);
    auto kernel = kFloor ? decode_floor_kernel<CL> : decode_cluster_kernel<CL>;
    // raise the kernel's shared-memory limit only when a larger size is first needed
    // (no attribute call on the steady path, e.g. inside a CUDA graph capture)
    static size_t smem_set[64] = {};  // per device
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64 || smem > smem_set[dev]) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        if (dev >= 0 && dev < 64) smem_set[dev] = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL, a.B * a.Hkv, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kernel, a);
    if (err == cudaSuccess) count_launch();
    return err;
}

}  // namespace

bool decode_sm100_supported(const DecodeParams& p) {
    if (!p.is_bf16 || p.d != kD || p.bs != kBS) return false;
    const int G = p.Hq / p.Hkv;
    if (G < 1 || G > 16) return false;
    if ((reinterpret_cast<uintptr_t>(p.k) | reinterpret_cast<uintptr_t>(p.v) | reinterpret_cast<uintptr_t>(p.q)) &
        15u)
        return false;
    if ((long)p.B * p.Hkv > 65535) return false;
    return Layout::bytes(G, p.top_k + 1, 8) <= 227 * 1024;  // the largest cluster needs the most
}

// Cluster size: about two CTAs per SM over all rows, at most 8, at most the
// attended blocks of a row.
static int pick_cluster(const DecodeParams& p, int max_entries) {
    const long rows = (long)p.B * p.Hkv;
    int cl = 1;
    while (cl < 8 && rows * cl * 2 <= 2L * 148 && cl * 2 <= max_entries) cl *= 2;
    return cl;
}

static cudaError_t launch_decode_impl(const DecodeParams& p, const float* s, int s_cols, int32_t* idx_out,
                                      bool floor, cudaStream_t stream) {
    DecArgs a;
    memset(&a, 0, sizeof(a));
    const long rows = (long)p.B * p.Hkv;
    if (p.page_table) {
        const long pool_rows = (long)p.num_pages * kBS;
        if (!encode_tma_rows(&a.tk, p.k, p.Hkv, pool_rows, 1, kBS) || !encode_tma_rows(&a.tv, p.v, p.Hkv, pool_rows, 1, kBS))
            return cudaErrorInvalidValue;
        a.page_table = p.page_table;
        a.pages_per_seq = p.pages_per_seq;
        a.num_pages = p.num_pages;
    } else if (!encode_cache(&a.tk, p.k, p.Tmax, rows) || !encode_cache(&a.tv, p.v, p.Tmax, rows)) {
        return cudaErrorInvalidValue;
    }
    a.q = static_cast<const __nv_bfloat16*>(p.q);
    a.ctx_len = p.ctx_len;
    a.idx = p.idx;
    a.s = s;
    a.idx_out = idx_out;
    a.o = static_cast<__nv_bfloat16*>(p.o);
    a.status = p.status;
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.Tmax = p.Tmax;
    a.top_k = p.top_k;
    a.s_cols = s_cols;
    a.mode = s ? 1 : (p.idx ? 0 : 2);
    a.vec_scores = s && (s_cols % 4 == 0) && (reinterpret_cast<uintptr_t>(s) & 15u) == 0;
    a.scale_log2 = p.scale * kLog2e;
    const int max_entries = a.mode == 2 ? (p.Tmax + kBS - 1) / kBS : p.top_k + 1;
    const int list_cap = a.mode == 2 ? 1 : p.top_k + 1;
    a.list_cap = list_cap;
    const int cl = pick_cluster(p, max_entries);
    if (floor) {
        switch (cl) {
            case 1: return launch_cl<1, true>(a, list_cap, stream);
            case 2: return launch_cl<2, true>(a, list_cap, stream);
            case 4: return launch_cl<4, true>(a, list_cap, stream);
            default: return launch_cl<8, true>(a, list_cap, stream);
        }
    }
    switch (cl) {
        case 1: return launch_cl<1, false>(a, list_cap, stream);
        case 2: return launch_cl<2, false>(a, list_cap, stream);
        case 4: return launch_cl<4, false>(a, list_cap, stream);
        default: return launch_cl<8, false>(a, list_cap, stream);
    }
}

cudaError_t launch_decode_sm100(const DecodeParams& p, const float* s, int s_cols, int32_t* idx_out,
                                cudaStream_t stream) {
    return launch_decode_impl(p, s, s_cols, idx_out, false, stream);
}

cudaError_t launch_decode_floor(const DecodeParams& p, const float* s, int s_cols, cudaStream_t stream) {
    return launch_decode_impl(p, s, s_cols, nullptr, true, stream);
}

cudaError_t read_decode_trace(void* dst, size_t bytes) {
#ifdef SAS_PHASE_TRACE
    if (bytes > sizeof(g_trace)) bytes = sizeof(g_trace);
    return cudaMemcpyFromSymbol(dst, g_trace, bytes);
#else
    (void)dst;
    (void)bytes;
    return cudaErrorNotSupported;
#endif
}

}  // namespace sas
