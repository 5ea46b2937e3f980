// decode_noalloc.cu -- sas_sparse_decode_noalloc: the sparse / dense decode of
// sas_sparse_decode for callers that cannot allocate device memory.
//
// Who needs it: code that runs where no allocator may be called -- a plugin
// inside a host program that owns every byte of device memory, a serving loop
// that must not call cudaMalloc (it synchronises the device) between decode
// steps, or a caller with no spare pool to carve a workspace from.  Such a
// caller passes only its inputs and outputs.
//
// The dispatch is that of sas_sparse_decode: the tensor-core decode kernel,
// which keeps its partials in shared memory and needs no scratch, takes the
// shapes it supports; the split-K kernels take the rest, and their partials live
// in a fixed array compiled into this library instead of a caller workspace.
//
// The array is file-scope device memory of kScratchFloats floats (4 MiB); every
// GPU that loads the library holds it until the process exits.  Host code may
// not use the array's name as a device address, so the entry point looks the
// address up with cudaGetSymbolAddress, once per device with that device
// current, on its first call on that device.
#include <math.h>

#include <mutex>

#include "kernels.h"
#include "sas.h"

namespace sas {
namespace {

constexpr size_t kScratchFloats = size_t(1) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_decode_scratch[kScratchFloats];

std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(float** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        err = cudaGetSymbolAddress(&ptr, g_decode_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_ptr[dev] = static_cast<float*>(ptr);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool valid(const sas_decode_desc* d) {
    if (!d) return false;
    if (d->batch <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0) return false;
    if (d->block_size <= 0 || d->top_k < 0 || d->max_ctx <= 0) return false;
    if (d->n_q_heads % d->n_kv_heads != 0) return false;
    if (d->dtype != SAS_F32 && d->dtype != SAS_BF16) return false;
    return isfinite(d->softmax_scale);
}

bool supported(const sas_decode_desc* d) {
    if (d->head_dim != 64 && d->head_dim != 128) return false;
    if (d->block_size % 16 != 0 || d->block_size > 256) return false;
    return d->n_q_heads / d->n_kv_heads <= 16;
}

}  // namespace
}  // namespace sas

extern "C" sas_status sas_sparse_decode_noalloc(const sas_decode_desc* desc, const void* q, const void* k_cache,
                                                const void* v_cache, const int32_t* ctx_len, const int32_t* idx,
                                                void* o, int32_t* status, sas_stream_t stream) {
    using namespace sas;
    if (!valid(desc)) return SAS_ERR_INVALID_VALUE;
    if (!q || !k_cache || !v_cache || !ctx_len || !o || !status) return SAS_ERR_INVALID_VALUE;
    if (!supported(desc)) return SAS_ERR_UNSUPPORTED;
    DecodeParams p = {};
    p.B = desc->batch;
    p.Hq = desc->n_q_heads;
    p.Hkv = desc->n_kv_heads;
    p.d = desc->head_dim;
    p.bs = desc->block_size;
    p.top_k = desc->top_k;
    p.Tmax = desc->max_ctx;
    p.is_bf16 = desc->dtype == SAS_BF16 ? 1 : 0;
    p.scale = desc->softmax_scale > 0.f ? desc->softmax_scale : 1.0f / sqrtf((float)desc->head_dim);
    p.q = q;
    p.k = k_cache;
    p.v = v_cache;
    p.ctx_len = ctx_len;
    p.idx = (desc->top_k > 0 && idx) ? idx : nullptr;
    p.o = o;
    p.status = status;
    cudaError_t err;
    if (decode_sm100_supported(p)) {
        // partials in shared memory: no scratch at all
        err = launch_decode_sm100(p, nullptr, 0, nullptr, reinterpret_cast<cudaStream_t>(stream));
    } else {
        decode_plan(p);
        if (decode_workspace(p) > kScratchFloats * sizeof(float)) return SAS_ERR_WORKSPACE_TOO_SMALL;
        float* scratch = nullptr;
        if (scratch_address(&scratch) != cudaSuccess) return SAS_ERR_CUDA;
        p.part = scratch;
        err = launch_decode(p, reinterpret_cast<cudaStream_t>(stream));
    }
    if (err == cudaSuccess) return SAS_OK;
    return err == cudaErrorNotSupported ? SAS_ERR_UNSUPPORTED : SAS_ERR_CUDA;
}
