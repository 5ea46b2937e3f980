// sas_api.cu -- the C ABI declared in include/sas.h: argument checks (before any
// launch, no side effects on failure), kernel dispatch, and the reading of the
// caller's device status word (which bounded device-side waits set when they
// give up).
#include <math.h>

#include <atomic>
#include <mutex>

#include "kernels.h"
#include "sas.h"

namespace sas {

static std::atomic<unsigned long long> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

namespace {

constexpr int kMaxDevices = 64;

// Read-only device properties, looked up once per device.
struct DeviceInfo {
    bool init = false;
    int n_sm = 0;
    int max_smem_optin = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

// Set-up once per device, with that device current: SM count and shared-memory
// limit.
cudaError_t device_info(DeviceInfo* out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& di = g_dev[dev];
    if (!di.init) {
        err = cudaDeviceGetAttribute(&di.n_sm, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        err = cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (err != cudaSuccess) return err;
        di.init = true;
    }
    *out = di;
    return cudaSuccess;
}

sas_status from_cuda(cudaError_t err) {
    if (err == cudaSuccess) return SAS_OK;
    if (err == cudaErrorNotSupported) return SAS_ERR_UNSUPPORTED;
    return SAS_ERR_CUDA;
}

bool check_train(const sas_attn_desc* d) {
    if (!d) return false;
    if (d->batch <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0) return false;
    if (d->seq_len <= 0 || d->block_size <= 0 || d->top_k < 0) return false;
    if (d->n_q_heads % d->n_kv_heads != 0 || d->seq_len % d->block_size != 0) return false;
    if (d->scope != SAS_SCOPE_SPARSE && d->scope != SAS_SCOPE_FULL) return false;
    if (d->dtype != SAS_F32 && d->dtype != SAS_BF16) return false;
    if (!isfinite(d->softmax_scale)) return false;
    if (d->gate < SAS_GATE_SOFTMAX || d->gate > SAS_GATE_STE) return false;
    return true;
}

bool supported_train(const sas_attn_desc* d) {
    if (d->head_dim != 64 && d->head_dim != 128) return false;
    if (d->block_size != 16 && d->block_size != 32 && d->block_size != 64) return false;
    return true;
}

TrainParams make_train(const sas_attn_desc* d) {
    TrainParams p = {};
    p.B = d->batch;
    p.Hq = d->n_q_heads;
    p.Hkv = d->n_kv_heads;
    p.d = d->head_dim;
    p.n = d->seq_len;
    p.bs = d->block_size;
    p.Cq = d->seq_len / d->block_size;
    p.top_k = d->top_k;
    p.full_scope = d->scope == SAS_SCOPE_FULL ? 1 : 0;
    p.gate = d->gate;
    p.is_bf16 = d->dtype == SAS_BF16 ? 1 : 0;
    p.scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)d->head_dim);
    return p;
}

bool check_decode(const sas_decode_desc* d) {
    if (!d) return false;
    if (d->batch <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0) return false;
    if (d->block_size <= 0 || d->top_k < 0 || d->max_ctx <= 0) return false;
    if (d->n_q_heads % d->n_kv_heads != 0) return false;
    if (d->dtype != SAS_F32 && d->dtype != SAS_BF16) return false;
    if (!isfinite(d->softmax_scale)) return false;
    return true;
}

bool supported_decode(const sas_decode_desc* d) {
    if (d->head_dim != 64 && d->head_dim != 128) return false;
    if (d->block_size % 16 != 0 || d->block_size > 256) return false;
    if (d->n_q_heads / d->n_kv_heads > 16) return false;
    return true;
}

DecodeParams make_decode(const sas_decode_desc* d) {
    DecodeParams p = {};
    p.B = d->batch;
    p.Hq = d->n_q_heads;
    p.Hkv = d->n_kv_heads;
    p.d = d->head_dim;
    p.bs = d->block_size;
    p.top_k = d->top_k;
    p.Tmax = d->max_ctx;
    p.is_bf16 = d->dtype == SAS_BF16 ? 1 : 0;
    p.scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)d->head_dim);
    return p;
}

// Workspace of a decode call: the larger of the sparse and the dense plans, so
// that one query covers both kinds of call.
size_t decode_ws_bytes(const DecodeParams& base) {
    DecodeParams sp = base, dn = base;
    sp.idx = reinterpret_cast<const int32_t*>(1);  // plan only, never dereferenced
    dn.idx = nullptr;
    decode_plan(sp);
    decode_plan(dn);
    const size_t a = decode_workspace(sp), b = decode_workspace(dn);
    return ((a > b ? a : b) + 255) & ~(size_t)255;
}

}  // namespace
}  // namespace sas

using namespace sas;

extern "C" {

sas_status sas_topk_select(const float* s, int32_t batch, int32_t n_kv_heads, int32_t n_rows, int32_t row_len,
                           const int32_t* ctx_len, int32_t block_size, int32_t top_k, int32_t* idx, float* lse_s,
                           sas_stream_t stream) {
    if (!s || batch <= 0 || n_kv_heads <= 0 || n_rows <= 0 || row_len <= 0 || top_k < 0) return SAS_ERR_INVALID_VALUE;
    if (!idx && !lse_s) return SAS_ERR_INVALID_VALUE;
    if (ctx_len && (n_rows != 1 || block_size <= 0)) return SAS_ERR_INVALID_VALUE;
    return from_cuda(launch_topk_select(s, batch, n_kv_heads, n_rows, row_len, ctx_len, block_size, top_k, idx,
                                        lse_s, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_gated_attn_fwd(const sas_attn_desc* desc, const void* q, const void* k, const void* v,
                              const float* s, const float* lse_s, const int32_t* idx, void* o, float* lse,
                              int32_t* status, sas_stream_t stream) {
    if (!check_train(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !k || !v || !s || !o || !lse || !status) return SAS_ERR_INVALID_VALUE;
    if (!lse_s && gate_softmax_family(desc->gate)) return SAS_ERR_INVALID_VALUE;
    if (desc->scope == SAS_SCOPE_SPARSE && desc->top_k > 0 && !idx) return SAS_ERR_INVALID_VALUE;
    if (!supported_train(desc)) return SAS_ERR_UNSUPPORTED;
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return SAS_ERR_CUDA;
    TrainParams p = make_train(desc);
    if (simt_max_smem(p.d, p.bs, p.Cq) > (size_t)di.max_smem_optin) return SAS_ERR_UNSUPPORTED;
    p.q = q;
    p.k = k;
    p.v = v;
    p.s = s;
    p.lse_s = lse_s;
    p.idx = desc->scope == SAS_SCOPE_SPARSE ? idx : nullptr;
    if (desc->scope == SAS_SCOPE_SPARSE && desc->top_k == 0) p.idx = nullptr;
    p.o = o;
    p.lse = lse;
    p.status = status;
    if (fwd_sm100_supported(p)) return from_cuda(launch_fwd_sm100(p, reinterpret_cast<cudaStream_t>(stream)));
    return from_cuda(launch_fwd_simt(p, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_attn_path(const sas_attn_desc* desc, int32_t* fwd_path, int32_t* bwd_path) {
    if (!check_train(desc)) return SAS_ERR_INVALID_VALUE;
    if (!supported_train(desc)) return SAS_ERR_UNSUPPORTED;
    TrainParams p = make_train(desc);
    // aligned stand-ins: the predicates look at shapes and pointer alignment only
    void* const aligned = reinterpret_cast<void*>(uintptr_t(256));
    p.q = p.k = p.v = p.o_in = p.dO = aligned;
    p.o = p.dq = p.dk = p.dv = p.Mbuf = aligned;
    if (fwd_path) *fwd_path = fwd_sm100_supported(p) ? SAS_PATH_TENSOR_CORE : SAS_PATH_SIMT;
    if (bwd_path) *bwd_path = bwd_sm100_supported(p) ? SAS_PATH_TENSOR_CORE : SAS_PATH_SIMT;
    return SAS_OK;
}

size_t sas_gated_attn_bwd_workspace_size(const sas_attn_desc* desc) {
    if (!check_train(desc)) return 0;
    TrainParams p = make_train(desc);
    return ((bwd_simt_workspace(p) + 255) & ~(size_t)255) + ((bwd_sm100_workspace(p) + 255) & ~(size_t)255);
}

static sas_status bwd_impl(const sas_attn_desc* desc, const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dO, const float* s, const float* lse_s, const int32_t* idx,
                           void* dq, void* dk, void* dv, float* ds, void* workspace, size_t ws_bytes, int32_t* status,
                           void* const* events, sas_stream_t stream) {
    if (!check_train(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !k || !v || !o || !lse || !dO || !s || !dq || !dk || !dv || !ds || !status) return SAS_ERR_INVALID_VALUE;
    if (!lse_s && gate_softmax_family(desc->gate)) return SAS_ERR_INVALID_VALUE;
    if (desc->scope == SAS_SCOPE_SPARSE && desc->top_k > 0 && !idx) return SAS_ERR_INVALID_VALUE;
    if (!supported_train(desc)) return SAS_ERR_UNSUPPORTED;
    const size_t need = sas_gated_attn_bwd_workspace_size(desc);
    if (ws_bytes < need) return SAS_ERR_WORKSPACE_TOO_SMALL;
    if (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))) return SAS_ERR_INVALID_VALUE;
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return SAS_ERR_CUDA;
    TrainParams p = make_train(desc);
    if (simt_max_smem(p.d, p.bs, p.Cq) > (size_t)di.max_smem_optin) return SAS_ERR_UNSUPPORTED;
    p.q = q;
    p.k = k;
    p.v = v;
    p.s = s;
    p.lse_s = lse_s;
    p.idx = desc->scope == SAS_SCOPE_SPARSE ? idx : nullptr;
    if (desc->scope == SAS_SCOPE_SPARSE && desc->top_k == 0) p.idx = nullptr;
    p.o_in = o;
    p.lse_in = lse;
    p.dO = dO;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.ds = ds;
    p.Dbuf = static_cast<float*>(workspace);
    if (bwd_sm100_workspace(p) > 0)
        p.Mbuf = static_cast<uint8_t*>(workspace) + ((bwd_simt_workspace(p) + 255) & ~(size_t)255);
    p.status = status;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (events) {
        if (!events[0] || !events[1] || !events[2]) return SAS_ERR_INVALID_VALUE;
        p.phase_event = events[1];
        if (cudaEventRecord(static_cast<cudaEvent_t>(events[0]), st) != cudaSuccess) return SAS_ERR_CUDA;
    }
    err = bwd_sm100_supported(p) ? launch_bwd_sm100(p, st) : launch_bwd_simt(p, st);
    if (err != cudaSuccess) return from_cuda(err);
    if (events && cudaEventRecord(static_cast<cudaEvent_t>(events[2]), st) != cudaSuccess) return SAS_ERR_CUDA;
    return SAS_OK;
}

sas_status sas_gated_attn_bwd(const sas_attn_desc* desc, const void* q, const void* k, const void* v,
                              const void* o, const float* lse, const void* dO, const float* s, const float* lse_s,
                              const int32_t* idx, void* dq, void* dk, void* dv, float* ds, void* workspace,
                              size_t ws_bytes, int32_t* status, sas_stream_t stream) {
    return bwd_impl(desc, q, k, v, o, lse, dO, s, lse_s, idx, dq, dk, dv, ds, workspace, ws_bytes, status, nullptr,
                    stream);
}

sas_status sas_gated_attn_bwd_timed(const sas_attn_desc* desc, const void* q, const void* k, const void* v,
                                    const void* o, const float* lse, const void* dO, const float* s,
                                    const float* lse_s, const int32_t* idx, void* dq, void* dk, void* dv, float* ds,
                                    void* workspace, size_t ws_bytes, void* const* events, int32_t* status,
                                    sas_stream_t stream) {
    if (!events) return SAS_ERR_INVALID_VALUE;
    return bwd_impl(desc, q, k, v, o, lse, dO, s, lse_s, idx, dq, dk, dv, ds, workspace, ws_bytes, status, events,
                    stream);
}

// ---------------------------------------------------------------------------
// pooled-key scorer
// ---------------------------------------------------------------------------

size_t sas_pooled_scores_workspace_size(const sas_attn_desc* desc) {
    if (!check_train(desc)) return 0;
    return (pooled_scores_workspace(make_train(desc)) + 255) & ~(size_t)255;
}

sas_status sas_pooled_scores(const sas_attn_desc* desc, const void* q, const void* k, float* s, void* workspace,
                             size_t ws_bytes, sas_stream_t stream) {
    if (!check_train(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !k || !s) return SAS_ERR_INVALID_VALUE;
    const int eb = desc->dtype == SAS_BF16 ? 2 : 4;
    if (!pool_shape_ok(desc->head_dim, desc->n_q_heads / desc->n_kv_heads, eb)) return SAS_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k)) & 15u) return SAS_ERR_INVALID_VALUE;
    const size_t need = sas_pooled_scores_workspace_size(desc);
    if (ws_bytes < need) return SAS_ERR_WORKSPACE_TOO_SMALL;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SAS_ERR_INVALID_VALUE;
    TrainParams p = make_train(desc);
    p.q = q;
    p.k = k;
    return from_cuda(launch_pooled_scores(p, s, workspace, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_pool_key_blocks(const sas_decode_desc* desc, const void* k_cache, int32_t block_begin,
                               int32_t block_end, void* ksum, int32_t nsum, sas_stream_t stream) {
    if (!check_decode(desc)) return SAS_ERR_INVALID_VALUE;
    if (!k_cache || !ksum) return SAS_ERR_INVALID_VALUE;
    if (block_begin < 0 || block_end < block_begin || block_end > nsum ||
        (long)block_end * desc->block_size > desc->max_ctx)
        return SAS_ERR_INVALID_VALUE;
    const int eb = desc->dtype == SAS_BF16 ? 2 : 4;
    if (!pool_shape_ok(desc->head_dim, 1, eb)) return SAS_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(k_cache) & 15u) return SAS_ERR_INVALID_VALUE;
    DecodeParams p = make_decode(desc);
    p.k = k_cache;
    return from_cuda(launch_pool_keys(p, block_begin, block_end, ksum, nsum, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_pool_key_blocks_paged(const sas_decode_desc* desc, const void* k_pages, const int32_t* page_table,
                                     int32_t pages_per_seq, int32_t num_pages, int32_t block_begin, int32_t block_end,
                                     void* ksum, int32_t nsum, sas_stream_t stream) {
    if (!check_decode(desc)) return SAS_ERR_INVALID_VALUE;
    if (!k_pages || !page_table || !ksum || pages_per_seq <= 0 || num_pages <= 0) return SAS_ERR_INVALID_VALUE;
    if (block_begin < 0 || block_end < block_begin || block_end > nsum || block_end > pages_per_seq)
        return SAS_ERR_INVALID_VALUE;
    const int eb = desc->dtype == SAS_BF16 ? 2 : 4;
    if (!pool_shape_ok(desc->head_dim, 1, eb)) return SAS_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(k_pages) & 15u) return SAS_ERR_INVALID_VALUE;
    DecodeParams p = make_decode(desc);
    p.k = k_pages;
    p.page_table = page_table;
    p.pages_per_seq = pages_per_seq;
    p.num_pages = num_pages;
    return from_cuda(
        launch_pool_keys_paged(p, block_begin, block_end, ksum, nsum, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_decode_scores(const sas_decode_desc* desc, const void* q, const void* ksum, int32_t nsum,
                             const int32_t* ctx_len, float* s, int32_t s_cols, sas_stream_t stream) {
    if (!check_decode(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !ksum || !ctx_len || !s || nsum <= 0 || s_cols <= 0) return SAS_ERR_INVALID_VALUE;
    if (desc->head_dim != 64 && desc->head_dim != 128) return SAS_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(ksum) & 15u) return SAS_ERR_INVALID_VALUE;
    DecodeParams p = make_decode(desc);
    p.q = q;
    p.ctx_len = ctx_len;
    return from_cuda(launch_decode_scores(p, ksum, nsum, s, s_cols, reinterpret_cast<cudaStream_t>(stream)));
}

size_t sas_sparse_decode_workspace_size(const sas_decode_desc* desc) {
    if (!check_decode(desc)) return 0;
    return decode_ws_bytes(make_decode(desc));
}

sas_status sas_sparse_decode(const sas_decode_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* ctx_len, const int32_t* idx, void* o, void* workspace, size_t ws_bytes,
                             int32_t* status, sas_stream_t stream) {
    if (!check_decode(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !k_cache || !v_cache || !ctx_len || !o || !status) return SAS_ERR_INVALID_VALUE;
    if (!supported_decode(desc)) return SAS_ERR_UNSUPPORTED;
    DecodeParams p = make_decode(desc);
    const size_t need = decode_ws_bytes(p);
    if (ws_bytes < need) return SAS_ERR_WORKSPACE_TOO_SMALL;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SAS_ERR_INVALID_VALUE;
    p.q = q;
    p.k = k_cache;
    p.v = v_cache;
    p.ctx_len = ctx_len;
    p.idx = desc->top_k > 0 ? idx : nullptr;
    if (!idx) p.idx = nullptr;
    p.o = o;
    p.part = static_cast<float*>(workspace);
    p.status = status;
    if (decode_sm100_supported(p))
        return from_cuda(launch_decode_sm100(p, nullptr, 0, nullptr, reinterpret_cast<cudaStream_t>(stream)));
    decode_plan(p);
    return from_cuda(launch_decode(p, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_sparse_decode_select(const sas_decode_desc* desc, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* ctx_len, const float* s, int32_t s_cols,
                                    void* o, int32_t* idx_out, int32_t* status, sas_stream_t stream) {
    if (!check_decode(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !k_cache || !v_cache || !ctx_len || !s || !o || !status || s_cols <= 0) return SAS_ERR_INVALID_VALUE;
    DecodeParams p = make_decode(desc);
    p.q = q;
    p.k = k_cache;
    p.v = v_cache;
    p.ctx_len = ctx_len;
    p.idx = nullptr;
    p.o = o;
    if (!supported_decode(desc) || !decode_sm100_supported(p)) return SAS_ERR_UNSUPPORTED;
    p.status = status;
    return from_cuda(launch_decode_sm100(p, s, s_cols, idx_out, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_sparse_decode_launch_floor(const sas_decode_desc* desc, const void* q, const void* k_cache,
                                          const void* v_cache, const int32_t* ctx_len, const float* s,
                                          int32_t s_cols, void* o, sas_stream_t stream) {
    if (!check_decode(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !k_cache || !v_cache || !ctx_len || !s || !o || s_cols <= 0) return SAS_ERR_INVALID_VALUE;
    DecodeParams p = make_decode(desc);
    p.q = q;
    p.k = k_cache;
    p.v = v_cache;
    p.ctx_len = ctx_len;
    p.idx = nullptr;
    p.o = o;
    if (!supported_decode(desc) || !decode_sm100_supported(p)) return SAS_ERR_UNSUPPORTED;
    return from_cuda(launch_decode_floor(p, s, s_cols, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_phase_trace_read(uint64_t* host_dst, int32_t rows) {
    if (!host_dst || rows <= 0 || rows > 1024) return SAS_ERR_INVALID_VALUE;
    cudaError_t err = cudaDeviceSynchronize();
    if (err == cudaSuccess) err = read_decode_trace(host_dst, (size_t)rows * 32 * sizeof(uint64_t));
    if (err == cudaErrorNotSupported) return SAS_ERR_UNSUPPORTED;
    return from_cuda(err);
}

sas_status sas_sparse_decode_paged(const sas_decode_desc* desc, const void* q, const void* k_pages,
                                   const void* v_pages, const int32_t* page_table, int32_t pages_per_seq,
                                   int32_t num_pages, const int32_t* ctx_len, const int32_t* idx, const float* s,
                                   int32_t s_cols, void* o, int32_t* idx_out, int32_t* status, sas_stream_t stream) {
    if (!check_decode(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !k_pages || !v_pages || !page_table || !ctx_len || !o || !status) return SAS_ERR_INVALID_VALUE;
    if (pages_per_seq <= 0 || num_pages <= 0 || (s && s_cols <= 0)) return SAS_ERR_INVALID_VALUE;
    if ((long)desc->max_ctx > (long)pages_per_seq * desc->block_size) return SAS_ERR_INVALID_VALUE;
    if ((reinterpret_cast<uintptr_t>(k_pages) | reinterpret_cast<uintptr_t>(v_pages)) & 15u)
        return SAS_ERR_INVALID_VALUE;
    DecodeParams p = make_decode(desc);
    p.q = q;
    p.k = k_pages;
    p.v = v_pages;
    p.ctx_len = ctx_len;
    p.idx = (s || desc->top_k <= 0) ? nullptr : idx;
    p.o = o;
    p.page_table = page_table;
    p.pages_per_seq = pages_per_seq;
    p.num_pages = num_pages;
    if (!supported_decode(desc) || !decode_sm100_supported(p)) return SAS_ERR_UNSUPPORTED;
    if ((long)num_pages * desc->block_size > 0x7fffffffL) return SAS_ERR_UNSUPPORTED;
    p.status = status;
    return from_cuda(launch_decode_sm100(p, s, s_cols, s ? idx_out : nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_get_device_status(int32_t* status, sas_stream_t stream) {
    if (!status) return SAS_ERR_INVALID_VALUE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SAS_ERR_CUDA;
    int32_t word = 0;
    if (cudaMemcpyAsync(&word, status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SAS_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SAS_ERR_CUDA;
    if (word == 0) return SAS_OK;
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return SAS_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SAS_ERR_CUDA;
    if (word == SAS_ERR_DEVICE_TIMEOUT) return SAS_ERR_DEVICE_TIMEOUT;
    if ((word & 0xff) == SAS_ERR_DEVICE_BOUNDS) return SAS_ERR_DEVICE_BOUNDS;
    return SAS_ERR_CUDA;
}

sas_status sas_selftest_bounded_wait(int32_t limit_ms, int32_t* status, int32_t* trace, sas_stream_t stream) {
    if (limit_ms <= 0 || limit_ms > 10000 || !status) return SAS_ERR_INVALID_VALUE;
    return from_cuda(launch_selftest_wait(status, trace, (unsigned long long)limit_ms * 1000000ull,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

const char* sas_status_string(sas_status status) {
    switch (status) {
        case SAS_OK: return "success";
        case SAS_ERR_INVALID_VALUE: return "invalid argument";
        case SAS_ERR_UNSUPPORTED: return "unsupported problem shape or type";
        case SAS_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case SAS_ERR_CUDA: return "CUDA error";
        case SAS_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
        case SAS_ERR_DEVICE_BOUNDS: return "a device-side index check failed (debug-bounds build)";
    }
    return "unknown status";
}

int32_t sas_version(void) { return 100; }

uint64_t sas_launch_count(void) { return (uint64_t)g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
