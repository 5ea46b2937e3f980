"""Thin Python binding of libsas (include/sas.h).

Argument marshalling only: each function passes torch tensors' device pointers
and the current CUDA stream to the C entry point of the same name, and raises
``SasError`` on a non-zero status.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback.  Importing this module loads
``libsas.so`` and fails loudly if it has not been built
(``python -m trainable_block_sparse_sas_b200.build``).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

# SAS_LIBRARY names another build of the same library (the debug-bounds build,
# libsas_debug.so, made by `python -m trainable_block_sparse_sas_b200.build --debug-bounds`)
_LIB_PATH = os.environ.get("SAS_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsas.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libsas.so not built at {_LIB_PATH}: run python -m trainable_block_sparse_sas_b200.build")
lib = ctypes.CDLL(_LIB_PATH)

SAS_OK, SAS_ERR_INVALID_VALUE, SAS_ERR_UNSUPPORTED, SAS_ERR_WORKSPACE_TOO_SMALL, SAS_ERR_CUDA, \
    SAS_ERR_DEVICE_TIMEOUT, SAS_ERR_DEVICE_BOUNDS = range(7)
SAS_F32, SAS_BF16 = 0, 1
SAS_SCOPE_SPARSE, SAS_SCOPE_FULL = 0, 1
SAS_GATE_SOFTMAX, SAS_GATE_SIGMOID, SAS_GATE_RAW, SAS_GATE_OUTER, SAS_GATE_STE = 0, 1, 2, 3, 4
GATES = {"softmax": SAS_GATE_SOFTMAX, "sigmoid": SAS_GATE_SIGMOID, "raw": SAS_GATE_RAW, "outer": SAS_GATE_OUTER,
         "ste": SAS_GATE_STE}


class SasError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.sas_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


class AttnDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("seq_len", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("scope", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("gate", ctypes.c_int32)]


class DecodeDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("max_ctx", ctypes.c_int32), ("dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


_vp, _i32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
lib.sas_status_string.restype = ctypes.c_char_p
lib.sas_status_string.argtypes = [ctypes.c_int]
lib.sas_version.restype = ctypes.c_int32
lib.sas_topk_select.restype = ctypes.c_int
lib.sas_topk_select.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _i32, _i32, _vp, _vp, _vp]
lib.sas_gated_attn_fwd.restype = ctypes.c_int
lib.sas_gated_attn_fwd.argtypes = [ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.sas_attn_path.restype = ctypes.c_int
lib.sas_attn_path.argtypes = [ctypes.POINTER(AttnDesc), ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
lib.sas_gated_attn_bwd_workspace_size.restype = _sz
lib.sas_gated_attn_bwd_workspace_size.argtypes = [ctypes.POINTER(AttnDesc)]
lib.sas_gated_attn_bwd.restype = ctypes.c_int
lib.sas_gated_attn_bwd.argtypes = [ctypes.POINTER(AttnDesc)] + [_vp] * 14 + [_sz, _vp, _vp]
lib.sas_gated_attn_bwd_timed.restype = ctypes.c_int
lib.sas_gated_attn_bwd_timed.argtypes = [ctypes.POINTER(AttnDesc)] + [_vp] * 14 + [_sz, _vp, _vp, _vp]
lib.sas_sparse_decode_workspace_size.restype = _sz
lib.sas_sparse_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeDesc)]
lib.sas_sparse_decode.restype = ctypes.c_int
lib.sas_sparse_decode.argtypes = [ctypes.POINTER(DecodeDesc)] + [_vp] * 7 + [_sz, _vp, _vp]
lib.sas_sparse_decode_select.restype = ctypes.c_int
lib.sas_sparse_decode_select.argtypes = [ctypes.POINTER(DecodeDesc)] + [_vp] * 5 + [_i32, _vp, _vp, _vp, _vp]
lib.sas_sparse_decode_launch_floor.restype = ctypes.c_int
lib.sas_sparse_decode_launch_floor.argtypes = [ctypes.POINTER(DecodeDesc)] + [_vp] * 5 + [_i32, _vp, _vp]
lib.sas_phase_trace_read.restype = ctypes.c_int
lib.sas_phase_trace_read.argtypes = [_vp, _i32]
lib.sas_sparse_decode_paged.restype = ctypes.c_int
lib.sas_sparse_decode_paged.argtypes = [ctypes.POINTER(DecodeDesc), _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _i32,
                                        _vp, _vp, _vp, _vp]
lib.sas_sparse_decode_noalloc.restype = ctypes.c_int
lib.sas_sparse_decode_noalloc.argtypes = [ctypes.POINTER(DecodeDesc)] + [_vp] * 8
lib.sas_selftest_bounded_wait.restype = ctypes.c_int
lib.sas_selftest_bounded_wait.argtypes = [_i32, _vp, _vp, _vp]
lib.sas_launch_count.restype = ctypes.c_uint64
lib.sas_launch_count.argtypes = []
lib.sas_get_device_status.restype = ctypes.c_int
lib.sas_get_device_status.argtypes = [_vp, _vp]
lib.sas_pooled_scores_workspace_size.restype = _sz
lib.sas_pooled_scores_workspace_size.argtypes = [ctypes.POINTER(AttnDesc)]
lib.sas_pooled_scores.restype = ctypes.c_int
lib.sas_pooled_scores.argtypes = [ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _sz, _vp]
lib.sas_pool_key_blocks.restype = ctypes.c_int
lib.sas_pool_key_blocks.argtypes = [ctypes.POINTER(DecodeDesc), _vp, _i32, _i32, _vp, _i32, _vp]
lib.sas_pool_key_blocks_paged.restype = ctypes.c_int
lib.sas_pool_key_blocks_paged.argtypes = [ctypes.POINTER(DecodeDesc), _vp, _vp, _i32, _i32, _i32, _i32, _vp, _i32, _vp]
lib.sas_decode_scores.restype = ctypes.c_int
lib.sas_decode_scores.argtypes = [ctypes.POINTER(DecodeDesc), _vp, _vp, _i32, _vp, _vp, _i32, _vp]


def _p(t):
    """Device pointer of a tensor for the C ABI (every libsas pointer is device
    memory: a host tensor here would be dereferenced by a kernel)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to libsas must be on a CUDA device")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != SAS_OK:
        raise SasError(status, where)


# The C ABI reports device-side failures (a bounded wait that gave up) through a
# caller-owned int32 status word.  Calls take it as `status=`; without one the
# binding passes a word of its own, one per device, created zeroed on first use
# (make a first call on a device outside any CUDA-graph capture).
_default_words = {}


def status_word(device=None) -> torch.Tensor:
    """A zeroed device status word for the C ABI (int32, one element)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return torch.zeros(1, dtype=torch.int32, device=dev)


def _status(status, ref: torch.Tensor):
    if status is not None:
        _need(status, 1, _I32, "status")
        return _p(status)
    dev = ref.device
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    word = _default_words.get(idx)
    if word is None:
        word = status_word(torch.device("cuda", idx))
        _default_words[idx] = word
    return _p(word)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SAS_BF16
    if t.dtype == torch.float32:
        return SAS_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---------------------------------------------------------------------------
# buffer checks: the C ABI sees pointers only, so before each call the binding
# makes sure every tensor holds the elements the descriptor implies, contiguously
# and in the expected dtype (a short buffer would be read or written out of
# bounds on the GPU); _p then refuses host tensors
# ---------------------------------------------------------------------------

_I32 = (torch.int32,)
_F32 = (torch.float32,)


def _dt(desc):
    return (torch.bfloat16,) if desc.dtype == SAS_BF16 else (torch.float32,)


def _need(t, numel: int, dtypes, name: str, optional: bool = False):
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call uses {numel}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} is {t.dtype}; expected {' or '.join(str(d) for d in dtypes)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _train_sizes(desc):
    Cq = desc.seq_len // desc.block_size if desc.block_size > 0 else 0
    q = desc.batch * desc.seq_len * desc.n_q_heads * desc.head_dim
    kv = desc.batch * desc.seq_len * desc.n_kv_heads * desc.head_dim
    return Cq, q, kv


def _check_train(desc, q, k, v, s, lse_s, idx):
    Cq, nq, nkv = _train_sizes(desc)
    dt = _dt(desc)
    _need(q, nq, dt, "q")
    _need(k, nkv, dt, "k")
    _need(v, nkv, dt, "v")
    _need(s, desc.batch * desc.n_kv_heads * Cq * Cq, _F32, "s")
    _need(lse_s, desc.batch * desc.n_kv_heads * Cq, _F32, "lse_s", optional=True)
    _need(idx, desc.batch * desc.n_kv_heads * Cq * max(desc.top_k, 0), _I32, "idx", optional=True)
    return Cq, nq, nkv


def _check_decode(desc, q, o, ctx_len):
    dt = _dt(desc)
    nq = desc.batch * desc.n_q_heads * desc.head_dim
    _need(q, nq, dt, "q")
    _need(o, nq, dt, "o", optional=o is None)
    _need(ctx_len, desc.batch, _I32, "ctx_len")


def attn_desc(q, k, block_size: int, top_k: int, full_scope: bool = False, softmax_scale: float = 0.0,
              gate: str = "softmax") -> AttnDesc:
    """gate: "softmax" (log g = s - LSE(s), the method), "sigmoid" (log sigmoid(s)),
    "raw" (s), "outer" (g = softmax(s) weighting the values outside the softmax) or
    "ste" (hard Top-K forward, straight-through backward to g = softmax(s))."""
    B, n, Hq, d = q.shape
    return AttnDesc(B, Hq, k.shape[2], d, n, block_size, top_k, SAS_SCOPE_FULL if full_scope else SAS_SCOPE_SPARSE,
                    _dtype_code(q), softmax_scale, GATES[gate])


def decode_desc(q, k_cache, block_size: int, top_k: int, softmax_scale: float = 0.0) -> DecodeDesc:
    B, Hq, d = q.shape
    return DecodeDesc(B, Hq, k_cache.shape[1], d, block_size, top_k, k_cache.shape[2], _dtype_code(q), softmax_scale)


def sas_topk_select(s, n_rows, row_len, top_k, idx=None, lse_s=None, ctx_len=None, block_size=0, stream=None):
    """s [B, Hkv, n_rows, row_len] fp32 -> writes idx [B,Hkv,n_rows,top_k] int32 and/or lse_s."""
    B, Hkv = s.shape[0], s.shape[1]
    _need(s, B * Hkv * n_rows * row_len, _F32, "s")
    _need(idx, B * Hkv * n_rows * max(top_k, 0), _I32, "idx", optional=True)
    _need(lse_s, B * Hkv * n_rows, _F32, "lse_s", optional=True)
    _need(ctx_len, B, _I32, "ctx_len", optional=True)
    st = lib.sas_topk_select(_p(s), B, Hkv, n_rows, row_len, _p(ctx_len), block_size, top_k, _p(idx), _p(lse_s),
                             _stream(stream))
    _check(st, "sas_topk_select")


def sas_gated_attn_fwd(desc, q, k, v, s, lse_s, idx, o, lse, stream=None, status=None):
    _, nq, _ = _check_train(desc, q, k, v, s, lse_s, idx)
    _need(o, nq, _dt(desc), "o")
    _need(lse, desc.batch * desc.n_q_heads * desc.seq_len, _F32, "lse")
    _check(lib.sas_gated_attn_fwd(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(s), _p(lse_s), _p(idx), _p(o), _p(lse),
                                  _status(status, q), _stream(stream)), "sas_gated_attn_fwd")


def sas_attn_path(desc) -> tuple[str, str]:
    """("tensor_core" | "simt", same) for the forward and the backward of a problem
    (with 16-byte aligned tensors)."""
    f, b = ctypes.c_int32(-1), ctypes.c_int32(-1)
    _check(lib.sas_attn_path(ctypes.byref(desc), ctypes.byref(f), ctypes.byref(b)), "sas_attn_path")
    name = {0: "simt", 1: "tensor_core"}
    return name[f.value], name[b.value]


def sas_gated_attn_bwd_workspace_size(desc) -> int:
    return int(lib.sas_gated_attn_bwd_workspace_size(ctypes.byref(desc)))


def sas_gated_attn_bwd(desc, q, k, v, o, lse, dO, s, lse_s, idx, dq, dk, dv, ds, workspace, stream=None, status=None):
    Cq, nq, nkv = _check_train(desc, q, k, v, s, lse_s, idx)
    dt = _dt(desc)
    for t, n, name in ((o, nq, "o"), (dO, nq, "dO"), (dq, nq, "dq"), (dk, nkv, "dk"), (dv, nkv, "dv")):
        _need(t, n, dt, name)
    _need(lse, desc.batch * desc.n_q_heads * desc.seq_len, _F32, "lse")
    _need(ds, desc.batch * desc.n_kv_heads * Cq * Cq, _F32, "ds")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.sas_gated_attn_bwd(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o), _p(lse), _p(dO), _p(s), _p(lse_s),
                                  _p(idx), _p(dq), _p(dk), _p(dv), _p(ds), _p(workspace), ws_bytes,
                                  _status(status, q), _stream(stream)), "sas_gated_attn_bwd")


def sas_gated_attn_bwd_timed(desc, q, k, v, o, lse, dO, s, lse_s, idx, dq, dk, dv, ds, workspace, events, stream=None,
                             status=None):
    """sas_gated_attn_bwd with three torch.cuda.Event (timing enabled) recorded by
    the library on the stream: before the dq/ds kernel, between it and the dk/dv
    kernel, and after the latter."""
    Cq, nq, nkv = _check_train(desc, q, k, v, s, lse_s, idx)
    dt = _dt(desc)
    for t, n, name in ((o, nq, "o"), (dO, nq, "dO"), (dq, nq, "dq"), (dk, nkv, "dk"), (dv, nkv, "dv")):
        _need(t, n, dt, name)
    _need(lse, desc.batch * desc.n_q_heads * desc.seq_len, _F32, "lse")
    _need(ds, desc.batch * desc.n_kv_heads * Cq * Cq, _F32, "ds")
    if len(events) != 3:
        raise ValueError("events: three torch.cuda.Event")
    st = stream if stream is not None else torch.cuda.current_stream()
    for e in events:
        if not e.cuda_event:
            e.record(st)  # torch creates the CUDA event on its first record
    handles = (ctypes.c_void_p * 3)(*(e.cuda_event for e in events))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.sas_gated_attn_bwd_timed(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o), _p(lse), _p(dO), _p(s),
                                        _p(lse_s), _p(idx), _p(dq), _p(dk), _p(dv), _p(ds), _p(workspace), ws_bytes,
                                        handles, _status(status, q), _stream(stream)), "sas_gated_attn_bwd_timed")


def sas_sparse_decode_workspace_size(desc) -> int:
    return int(lib.sas_sparse_decode_workspace_size(ctypes.byref(desc)))


def _check_cache(desc, k_cache, v_cache):
    n = desc.batch * desc.n_kv_heads * desc.max_ctx * desc.head_dim
    _need(k_cache, n, _dt(desc), "k_cache")
    _need(v_cache, n, _dt(desc), "v_cache")


def sas_sparse_decode(desc, q, k_cache, v_cache, ctx_len, idx, o, workspace, stream=None, status=None):
    _check_decode(desc, q, o, ctx_len)
    _check_cache(desc, k_cache, v_cache)
    _need(idx, desc.batch * desc.n_kv_heads * max(desc.top_k, 0), _I32, "idx", optional=True)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.sas_sparse_decode(ctypes.byref(desc), _p(q), _p(k_cache), _p(v_cache), _p(ctx_len), _p(idx), _p(o),
                                 _p(workspace), ws_bytes, _status(status, q), _stream(stream)), "sas_sparse_decode")


def sas_sparse_decode_select(desc, q, k_cache, v_cache, ctx_len, s, o, idx_out=None, stream=None, status=None):
    """Fused decode step: Top-K of s [B, Hkv, s_cols] and the gate-free attention."""
    _check_decode(desc, q, o, ctx_len)
    _check_cache(desc, k_cache, v_cache)
    _need(s, desc.batch * desc.n_kv_heads * s.shape[-1], _F32, "s")
    _need(idx_out, desc.batch * desc.n_kv_heads * max(desc.top_k, 0), _I32, "idx_out", optional=True)
    _check(lib.sas_sparse_decode_select(ctypes.byref(desc), _p(q), _p(k_cache), _p(v_cache), _p(ctx_len), _p(s),
                                        s.shape[-1], _p(o), _p(idx_out), _status(status, q), _stream(stream)),
           "sas_sparse_decode_select")


def sas_sparse_decode_launch_floor(desc, q, k_cache, v_cache, ctx_len, s, o, stream=None):
    """An empty kernel on the grid, cluster, block and shared memory of the fused
    decode step with these arguments (the launch floor under it)."""
    _check_decode(desc, q, o, ctx_len)
    _check_cache(desc, k_cache, v_cache)
    _need(s, desc.batch * desc.n_kv_heads * s.shape[-1], _F32, "s")
    _check(lib.sas_sparse_decode_launch_floor(ctypes.byref(desc), _p(q), _p(k_cache), _p(v_cache), _p(ctx_len), _p(s),
                                              s.shape[-1], _p(o), _stream(stream)),
           "sas_sparse_decode_launch_floor")


def sas_phase_trace_read(rows: int):
    """The decode kernel's phase trace (a library built with --phase-trace):
    numpy uint64 [rows, 32], one row per CTA."""
    import numpy as np

    buf = np.zeros((rows, 32), dtype=np.uint64)
    _check(lib.sas_phase_trace_read(buf.ctypes.data_as(ctypes.c_void_p), rows), "sas_phase_trace_read")
    return buf


def paged_decode_desc(q, k_pages, block_size: int, top_k: int, max_ctx: int, softmax_scale: float = 0.0) -> DecodeDesc:
    """Descriptor of a paged-cache decode: k_pages [num_pages, block_size, Hkv, d]."""
    B, Hq, d = q.shape
    return DecodeDesc(B, Hq, k_pages.shape[2], d, block_size, top_k, max_ctx, _dtype_code(q), softmax_scale)


def sas_sparse_decode_paged(desc, q, k_pages, v_pages, page_table, ctx_len, o, s=None, idx=None, idx_out=None,
                            stream=None, status=None):
    """Decode step over a paged cache: page_table [B, pages_per_seq] int32 maps a
    sequence's blocks to pages of k_pages / v_pages [num_pages, block_size, Hkv, d].
    Blocks from the Top-K of s (fused), from idx, or every block when both are None."""
    _check_decode(desc, q, o, ctx_len)
    pool = k_pages.shape[0] * desc.block_size * desc.n_kv_heads * desc.head_dim
    _need(k_pages, pool, _dt(desc), "k_pages")
    _need(v_pages, pool, _dt(desc), "v_pages")
    _need(page_table, desc.batch * page_table.shape[1], _I32, "page_table")
    if s is not None:
        _need(s, desc.batch * desc.n_kv_heads * s.shape[-1], _F32, "s")
    _need(idx, desc.batch * desc.n_kv_heads * max(desc.top_k, 0), _I32, "idx", optional=True)
    _need(idx_out, desc.batch * desc.n_kv_heads * max(desc.top_k, 0), _I32, "idx_out", optional=True)
    _check(lib.sas_sparse_decode_paged(ctypes.byref(desc), _p(q), _p(k_pages), _p(v_pages), _p(page_table),
                                       page_table.shape[1], k_pages.shape[0], _p(ctx_len), _p(idx), _p(s),
                                       0 if s is None else s.shape[-1], _p(o), _p(idx_out), _status(status, q),
                                       _stream(stream)), "sas_sparse_decode_paged")


def sas_pooled_scores_workspace_size(desc) -> int:
    return int(lib.sas_pooled_scores_workspace_size(ctypes.byref(desc)))


def sas_pooled_scores(desc, q, k, s, workspace, stream=None):
    """Pooled-key scores, training shape: s [B,Hkv,Cq,Cq] fp32 (m < c), from the
    mean of q over each query block and group and the mean of k over each block."""
    Cq, nq, nkv = _train_sizes(desc)
    _need(q, nq, _dt(desc), "q")
    _need(k, nkv, _dt(desc), "k")
    _need(s, desc.batch * desc.n_kv_heads * Cq * Cq, _F32, "s")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.sas_pooled_scores(ctypes.byref(desc), _p(q), _p(k), _p(s), _p(workspace), ws_bytes, _stream(stream)),
           "sas_pooled_scores")


def sas_pool_key_blocks(desc, k_cache, block_begin: int, block_end: int, ksum, stream=None):
    """Mean-pooled summaries of the full blocks [block_begin, block_end) of a
    contiguous cache into ksum [B,Hkv,nsum,d] (the cache's dtype)."""
    _need(k_cache, desc.batch * desc.n_kv_heads * desc.max_ctx * desc.head_dim, _dt(desc), "k_cache")
    _need(ksum, desc.batch * desc.n_kv_heads * ksum.shape[2] * desc.head_dim, _dt(desc), "ksum")
    _check(lib.sas_pool_key_blocks(ctypes.byref(desc), _p(k_cache), block_begin, block_end, _p(ksum), ksum.shape[2],
                                   _stream(stream)), "sas_pool_key_blocks")


def sas_pool_key_blocks_paged(desc, k_pages, page_table, block_begin: int, block_end: int, ksum, stream=None):
    """Block summaries from a paged pool k_pages [num_pages, block_size, Hkv, d]
    with page_table [B, pages_per_seq] int32, into ksum [B,Hkv,nsum,d]."""
    _need(k_pages, k_pages.shape[0] * desc.block_size * desc.n_kv_heads * desc.head_dim, _dt(desc), "k_pages")
    _need(page_table, desc.batch * page_table.shape[1], _I32, "page_table")
    _need(ksum, desc.batch * desc.n_kv_heads * ksum.shape[2] * desc.head_dim, _dt(desc), "ksum")
    _check(lib.sas_pool_key_blocks_paged(ctypes.byref(desc), _p(k_pages), _p(page_table), page_table.shape[1],
                                         k_pages.shape[0], block_begin, block_end, _p(ksum), ksum.shape[2],
                                         _stream(stream)), "sas_pool_key_blocks_paged")


def sas_decode_scores(desc, q, ksum, ctx_len, s, stream=None):
    """Decode scores s [B,Hkv,s_cols] fp32 from the block summaries ksum."""
    _check_decode(desc, q, None, ctx_len)
    _need(ksum, desc.batch * desc.n_kv_heads * ksum.shape[2] * desc.head_dim, _dt(desc), "ksum")
    _need(s, desc.batch * desc.n_kv_heads * s.shape[-1], _F32, "s")
    _check(lib.sas_decode_scores(ctypes.byref(desc), _p(q), _p(ksum), ksum.shape[2], _p(ctx_len), _p(s), s.shape[-1],
                                 _stream(stream)), "sas_decode_scores")


def sas_sparse_decode_noalloc(desc, q, k_cache, v_cache, ctx_len, idx, o, stream=None, status=None):
    """sas_sparse_decode without a workspace, for callers that cannot allocate
    device memory: shapes the tensor-core decode takes need no scratch; the
    split-K kernels put their partials in a fixed 4 MiB array inside the library.
    Overlapping calls race on that array."""
    _check_decode(desc, q, o, ctx_len)
    _check_cache(desc, k_cache, v_cache)
    _need(idx, desc.batch * desc.n_kv_heads * max(desc.top_k, 0), _I32, "idx", optional=True)
    _check(lib.sas_sparse_decode_noalloc(ctypes.byref(desc), _p(q), _p(k_cache), _p(v_cache), _p(ctx_len), _p(idx),
                                         _p(o), _status(status, q), _stream(stream)), "sas_sparse_decode_noalloc")


def sas_get_device_status(status=None, stream=None):
    """Synchronise the stream, then read and clear a device status word (the
    binding's word of the current device when status is None); raises SasError
    (SAS_ERR_DEVICE_TIMEOUT) when a bounded device-side wait gave up."""
    if status is None:
        word = _default_words.get(torch.cuda.current_device())
        if word is None:
            return  # nothing has run on this device through the default word
        status = word
    _need(status, 1, _I32, "status")
    _check(lib.sas_get_device_status(_p(status), _stream(stream)), "sas_get_device_status")


def sas_selftest_bounded_wait(limit_ms: int, status=None, trace=None, stream=None):
    """Run the failure path of the tensor-core kernels with a wait limit of
    limit_ms; the timeout lands in `status` (the binding's word when None) and the
    phases reached in `trace` (int32 [4]) when given."""
    if status is not None:
        _need(status, 1, _I32, "status")
    else:
        status = _default_words.setdefault(torch.cuda.current_device(), status_word())
    _need(trace, 4, _I32, "trace", optional=True)
    _check(lib.sas_selftest_bounded_wait(limit_ms, _p(status), _p(trace), _stream(stream)),
           "sas_selftest_bounded_wait")


def sas_launch_count() -> int:
    """Kernels launched by libsas so far in this process."""
    return int(lib.sas_launch_count())


def workspace(nbytes: int, device) -> torch.Tensor:
    """Caller-owned scratch from torch's allocator (256-byte aligned)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# convenience: one training-shape call sequence, and an autograd Function
# ---------------------------------------------------------------------------

def select_train(s, block_size: int, top_k: int, full_scope: bool = False, stream=None):
    """Score rows of a training problem -> (idx or None, lse_s)."""
    B, Hkv, Cq, _ = s.shape
    lse_s = torch.empty((B, Hkv, Cq), dtype=torch.float32, device=s.device)
    idx = None
    if not full_scope and top_k > 0:
        idx = torch.empty((B, Hkv, Cq, top_k), dtype=torch.int32, device=s.device)
    sas_topk_select(s, Cq, Cq, top_k, idx=idx, lse_s=lse_s, stream=stream)
    return idx, lse_s


class _SASAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, s, block_size, top_k, full_scope, softmax_scale, gate):
        q, k, v, s = (t.contiguous() for t in (q, k, v, s))
        desc = attn_desc(q, k, block_size, top_k, full_scope, softmax_scale, gate)
        idx, lse_s = select_train(s, block_size, top_k, full_scope)
        o = torch.empty_like(q)
        lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), dtype=torch.float32, device=q.device)
        sas_gated_attn_fwd(desc, q, k, v, s, lse_s, idx, o, lse)
        ctx.save_for_backward(q, k, v, s, o, lse, lse_s, idx if idx is not None else torch.empty(0))
        ctx.desc = desc
        ctx.has_idx = idx is not None
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, s, o, lse, lse_s, idx = ctx.saved_tensors
        idx = idx if ctx.has_idx else None
        dO = dO.contiguous()
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ds = torch.empty_like(s)
        ws = workspace(sas_gated_attn_bwd_workspace_size(ctx.desc), q.device)
        sas_gated_attn_bwd(ctx.desc, q, k, v, o, lse, dO, s, lse_s, idx, dq, dk, dv, ds, ws)
        return dq, dk, dv, ds, None, None, None, None, None


def sas_attention(q, k, v, s, block_size: int, top_k: int, full_scope: bool = False, softmax_scale: float = 0.0,
                  gate: str = "softmax"):
    """Differentiable SAS gated attention: o = softmax(sigma q K_S^T + log g_S) V_S.

    q [B,n,Hq,d], k/v [B,n,Hkv,d] (bf16 or fp32), s [B,Hkv,n/b,n/b] fp32.
    gate: "softmax" (the method); "sigmoid", "raw", "outer", "ste" (ablations)."""
    return _SASAttention.apply(q, k, v, s, block_size, top_k, full_scope, softmax_scale, gate)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
