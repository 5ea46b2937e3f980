// kernels.h -- launchers of the libsas kernels (host side, internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sas {

// Host-side count of successful kernel launches (reported by sas_launch_count).
void count_launch(int n = 1);

struct TrainParams {
    const void* q;
    const void* k;
    const void* v;
    const float* s;
    const float* lse_s;
    const int32_t* idx;
    void* o;
    float* lse;
    // backward
    const void* o_in;
    const float* lse_in;
    const void* dO;
    float* Dbuf;  // [B, Hq, n] row dot(dO, o)
    void* Mbuf;   // tensor-core backward: fp16 block masses (bwd_sm100_workspace bytes)
    void* dq;
    void* dk;
    void* dv;
    float* ds;
    int* status;  // device status word (bounded waits)
    void* phase_event;  // host only: cudaEvent_t recorded between the backward's two kernels (nullable)
    int B, Hq, Hkv, d, n, bs, Cq, top_k, full_scope, is_bf16;
    float scale;
    int gate;  // sas_gate: 0 softmax, 1 sigmoid, 2 raw logit, 3 outer, 4 hard STE
};

constexpr int kGateOuter = 3, kGateSte = 4;

// does log g enter the logits (inner gates 0-2)?  The outer gate weights the
// values instead; the hard STE gate's forward value is 1 (bias 0)
__host__ __device__ __forceinline__ bool gate_in_logits(int gate) { return gate <= 2; }
// is g = softmax(s) (so that lse_s is needed)?
__host__ __device__ __forceinline__ bool gate_softmax_family(int gate) { return gate == 0 || gate >= 3; }

// log g of a history block from its score (natural log): g = softmax(s) needs the
// row's LSE; the sigmoid and raw-logit variants do not
__host__ __device__ __forceinline__ float gate_log(float s, float lse, int gate) {
    if (gate == 1) return s >= 0.f ? -log1pf(expf(-s)) : s - log1pf(expf(s));
    if (gate == 2) return s;
    return s - lse;
}

// ds of one history block from its dlogg: the raw-logit gate passes it through,
// the sigmoid gate scales by 1 - g; g = softmax(s) subtracts g * sum(dlogg)
__host__ __device__ __forceinline__ float gate_ds(float dlogg, float logg, float tot, int gate) {
    if (gate == 2) return dlogg;
    if (gate == 1) return dlogg * (1.f - expf(logg));
    return dlogg - expf(logg) * tot;
}

struct DecodeParams {
    const void* q;
    const void* k;
    const void* v;
    const int32_t* ctx_len;
    const int32_t* idx;  // nullptr: dense
    void* o;
    float* part;  // [B*Hkv, nsplit, G, d + 2] partial (o, m, l)
    int* status;  // device status word (bounded waits)
    int B, Hq, Hkv, d, bs, top_k, Tmax, is_bf16, nsplit, per_split, list_max;
    float scale;
    // paged cache (tensor-core decode only): k, v are [num_pages, bs, Hkv, d] pools and
    // page_table[b * pages_per_seq + j] is the page of block j of sequence b
    const int32_t* page_table;  // nullptr: contiguous [B, Hkv, Tmax, d] caches
    int pages_per_seq, num_pages;
};

cudaError_t launch_topk_select(const float* s, int batch, int n_kv_heads, int n_rows, int row_len,
                               const int32_t* ctx_len, int block_size, int top_k, int32_t* idx, float* lse_s,
                               cudaStream_t stream);

cudaError_t launch_fwd_simt(const TrainParams& p, cudaStream_t stream);
bool fwd_sm100_supported(const TrainParams& p);
bool bwd_sm100_supported(const TrainParams& p);
size_t bwd_sm100_workspace(const TrainParams& p);
cudaError_t launch_bwd_sm100(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_fwd_sm100(const TrainParams& p, cudaStream_t stream);
cudaError_t launch_bwd_simt(const TrainParams& p, cudaStream_t stream);
size_t bwd_simt_workspace(const TrainParams& p);

bool pool_shape_ok(int d, int G, int elem_bytes);
size_t pooled_scores_workspace(const TrainParams& p);
cudaError_t launch_pooled_scores(const TrainParams& p, float* s, void* ws, cudaStream_t stream);
cudaError_t launch_pool_keys(const DecodeParams& p, int m0, int m1, void* ksum, int nsum, cudaStream_t stream);
cudaError_t launch_pool_keys_paged(const DecodeParams& p, int m0, int m1, void* ksum, int nsum, cudaStream_t stream);
cudaError_t launch_decode_scores(const DecodeParams& p, const void* ksum, int nsum, float* s, int s_cols,
                                 cudaStream_t stream);
size_t simt_max_smem(int D, int BS, int Cq);

void decode_plan(DecodeParams& p);
size_t decode_workspace(const DecodeParams& p);
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_selftest_wait(int* status, int* trace, unsigned long long limit_ns, cudaStream_t stream);
bool decode_sm100_supported(const DecodeParams& p);
// s != nullptr: fused Top-K selection from s [B, Hkv, s_cols] (idx_out nullable)
cudaError_t launch_decode_sm100(const DecodeParams& p, const float* s, int s_cols, int32_t* idx_out,
                                cudaStream_t stream);
// an empty kernel on the grid, cluster, block and shared memory of the fused decode
// of p (the launch floor under it)
cudaError_t launch_decode_floor(const DecodeParams& p, const float* s, int s_cols, cudaStream_t stream);
// the decode kernel's phase trace (builds with SAS_PHASE_TRACE; cudaErrorNotSupported otherwise)
cudaError_t read_decode_trace(void* dst, size_t bytes);

}  // namespace sas
