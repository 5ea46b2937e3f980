"""fp64 CPU oracle for SAS gated block-sparse attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
shares no code with the CUDA library: the arithmetic lives in ``sas_oracle.c``
(plain loops in double precision), this module only marshals numpy arrays.

Every function follows a definition in the reviews of SAS ("SAS: Simple
Attention Sparsification via End-to-End Optimization of Context Ranking"); the
C file cites each one.  Parity status: every function here (selection, the
gated forward and backward with every gate variant and the bf16-stored-output
option, decode, and the pooled-key scorer) is pinned by the ``-m "not gpu"``
tests in ``tests/test_oracle_pins.py`` (worked example, closed forms, brute
force, dense torch formulations, finite differences, library special cases).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sas_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_sas.so")

ORC_F64, ORC_F32, ORC_BF16 = 0, 1, 2
_ERRORS = {1: "invalid argument", 2: "a query block attending a requested key block is not in qmask",
           3: "out of memory"}


def build(force: bool = False) -> str:
    """Compile the C oracle into liboracle_sas.so next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-std=c11", "-Wall", "-shared", "-fPIC", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


class _Desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("n", ctypes.c_int), ("bs", ctypes.c_int), ("top_k", ctypes.c_int),
                ("full_scope", ctypes.c_int), ("gate", ctypes.c_int), ("sigma", ctypes.c_double)]


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_num_threads.restype = ctypes.c_int
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _in(a):
    """Pass an input array with its element code; bfloat16 arrives as uint16 bits."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float64:
        code = ORC_F64
    elif a.dtype == np.float32:
        code = ORC_F32
    elif a.dtype == np.uint16:
        code = ORC_BF16
    else:
        raise TypeError(f"oracle input dtype {a.dtype} (use float64, float32 or uint16 bf16 bits)")
    return a, code, a.ctypes.data_as(ctypes.c_void_p)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what}: {_ERRORS.get(rc, rc)}")


def select(s, ncand, top_k: int, full_scope: bool = False, idx_cols: int | None = None):
    """Top-K selection and score LSE for rows of s ([..., row_len]).

    ncand: per-row candidate counts (array broadcastable to s.shape[:-1]).
    Returns (idx int32 [..., idx_cols] ascending, -1 padded; lse float64 [...]).
    """
    s_arr, s_code, s_p = _in(s)
    rows_shape = s_arr.shape[:-1]
    nrows = int(np.prod(rows_shape)) if rows_shape else 1
    row_len = s_arr.shape[-1]
    nc = np.ascontiguousarray(np.broadcast_to(np.asarray(ncand, dtype=np.int32), rows_shape).reshape(-1))
    cols = top_k if idx_cols is None else idx_cols
    idx = np.empty((nrows, cols), dtype=np.int32)
    lse = np.empty(nrows, dtype=np.float64)
    rc = lib().oracle_select(s_p, ctypes.c_int(s_code), ctypes.c_long(nrows), ctypes.c_long(row_len),
                             _ptr(nc), ctypes.c_int(top_k), ctypes.c_int(int(full_scope)), _ptr(idx),
                             ctypes.c_int(cols), _ptr(lse))
    _check(rc, "select")
    return idx.reshape(*rows_shape, cols), lse.reshape(rows_shape)


def train_select(s, top_k: int, full_scope: bool = False):
    """Selection for training score rows s [B, Hkv, Cq, Cq]: row c has c candidates."""
    s = np.asarray(s)
    Cq = s.shape[-2]
    ncand = np.broadcast_to(np.arange(Cq, dtype=np.int32)[:, None], s.shape[:-2] + (Cq, 1))[..., 0]
    return select(s, ncand, top_k, full_scope, idx_cols=top_k)


GATES = {"off": 0, "softmax": 1, "sigmoid": 2, "raw": 3, "outer": 4, "ste": 5}


def _gate_code(gate) -> int:
    """True / "softmax": log g = s - LSE(s) (the method); False / "off": no bias;
    "sigmoid": log g = log sigmoid(s); "raw": log g = s (the ablated activations);
    "outer": g = softmax(s) weights the values outside the attention softmax;
    "ste": hard Top-K forward, backward straight through to g = softmax(s)."""
    if isinstance(gate, (bool, np.bool_)):
        return 1 if gate else 0
    return GATES[gate]


def _desc(q, k, bs, top_k, full_scope, gate, sigma):
    B, n, Hq, d = q.shape
    Hkv = k.shape[2]
    if sigma is None:
        sigma = 1.0 / np.sqrt(d)
    return _Desc(B, Hq, Hkv, d, n, bs, top_k, int(full_scope), _gate_code(gate), float(sigma))


def _same_code(*arrs):
    codes = {a.dtype for a in arrs}
    if len(codes) != 1:
        raise TypeError("q, k, v (and dO) must share one element type")


def attn_fwd(q, k, v, s, bs: int, top_k: int, full_scope: bool = False, gate: bool = True, sigma=None,
             qmask=None):
    """Gated forward (Eq. 9). q [B,n,Hq,d], k/v [B,n,Hkv,d], s [B,Hkv,Cq,Cq].

    Returns (o float64 [B,n,Hq,d], lse float64 [B,Hq,n]).  qmask [B,Hkv,Cq] (bool)
    limits the query blocks computed; other outputs are left at 0 / NaN."""
    _same_code(np.asarray(q), np.asarray(k), np.asarray(v))
    qa, code, qp = _in(q)
    ka, _, kp = _in(k)
    va, _, vp = _in(v)
    sa, s_code, sp = _in(s)
    D = _desc(qa, ka, bs, top_k, full_scope, gate, sigma)
    o = np.zeros(qa.shape, dtype=np.float64)
    lse = np.full((D.B, D.Hq, D.n), np.nan, dtype=np.float64)
    qm = None if qmask is None else np.ascontiguousarray(qmask, dtype=np.uint8)
    rc = lib().oracle_attn_fwd(ctypes.byref(D), qp, kp, vp, ctypes.c_int(code), sp, ctypes.c_int(s_code),
                               None if qm is None else _ptr(qm), _ptr(o), _ptr(lse))
    _check(rc, "attn_fwd")
    return o, lse


def attn_bwd(q, k, v, dO, s, bs: int, top_k: int, full_scope: bool = False, gate: bool = True, sigma=None,
             qmask=None, kvmask=None, o_store=None):
    """Backward of L = sum(dO * o).  Returns a dict with o, lse, dq, dk, dv, ds, dlogg
    (float64).  qmask / kvmask [B,Hkv,Cq] limit the query blocks (o, lse, dq, ds) and
    the key blocks (dk, dv) computed.  o_store="bf16": the backward reads o as a
    bf16 output tensor holds it (the o of the inner-gate gradient, and of D_i =
    dO_i . o_i, rounded to bf16); None: the exact o."""
    _same_code(np.asarray(q), np.asarray(k), np.asarray(v), np.asarray(dO))
    qa, code, qp = _in(q)
    ka, _, kp = _in(k)
    va, _, vp = _in(v)
    ga, _, gp = _in(dO)
    sa, s_code, sp = _in(s)
    D = _desc(qa, ka, bs, top_k, full_scope, gate, sigma)
    Cq = D.n // D.bs
    out = {
        "o": np.zeros(qa.shape), "lse": np.zeros((D.B, D.Hq, D.n)), "dq": np.zeros(qa.shape),
        "dk": np.zeros(ka.shape), "dv": np.zeros(ka.shape), "ds": np.zeros((D.B, D.Hkv, Cq, Cq)),
        "dlogg": np.zeros((D.B, D.Hkv, Cq, Cq)),
    }
    qm = None if qmask is None else np.ascontiguousarray(qmask, dtype=np.uint8)
    km = None if kvmask is None else np.ascontiguousarray(kvmask, dtype=np.uint8)
    rc = lib().oracle_attn_bwd(ctypes.byref(D), qp, kp, vp, gp, ctypes.c_int(code), sp, ctypes.c_int(s_code),
                               None if qm is None else _ptr(qm), None if km is None else _ptr(km),
                               ctypes.c_int({None: 0, "bf16": 1}[o_store]), _ptr(out["o"]), _ptr(out["lse"]), _ptr(out["dq"]), _ptr(out["dk"]),
                               _ptr(out["dv"]), _ptr(out["ds"]), _ptr(out["dlogg"]))
    _check(rc, "attn_bwd")
    return out


def decode(q, k_cache, v_cache, ctx_len, s, bs: int, top_k: int, dense: bool = False, sigma=None):
    """Gate-free decode (one new token per sequence).  q [B,Hq,d];
    caches [B,Hkv,Tmax,d]; ctx_len [B] (cached tokens incl. the new one);
    s [B,Hkv,s_cols] fp32.  Returns (o float64 [B,Hq,d], idx int32 [B,Hkv,top_k])."""
    _same_code(np.asarray(q), np.asarray(k_cache), np.asarray(v_cache))
    qa, code, qp = _in(q)
    ka, _, kp = _in(k_cache)
    va, _, vp = _in(v_cache)
    B, Hq, d = qa.shape
    Hkv, Tmax = ka.shape[1], ka.shape[2]
    if sigma is None:
        sigma = 1.0 / np.sqrt(d)
    cl = np.ascontiguousarray(ctx_len, dtype=np.int32)
    if s is None:
        s = np.zeros((B, Hkv, 1), dtype=np.float32)
    sa, s_code, sp = _in(s)
    o = np.zeros((B, Hq, d), dtype=np.float64)
    idx = np.full((B, Hkv, max(top_k, 1)), -1, dtype=np.int32)
    rc = lib().oracle_decode(ctypes.c_int(B), ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(d),
                             ctypes.c_int(bs), ctypes.c_int(Tmax), ctypes.c_int(top_k), ctypes.c_double(sigma),
                             qp, kp, vp, ctypes.c_int(code), _ptr(cl), sp, ctypes.c_int(s_code),
                             ctypes.c_int(sa.shape[-1]), ctypes.c_int(int(dense)), _ptr(o), _ptr(idx))
    _check(rc, "decode")
    return o, idx[..., :top_k]


def pool_scores(q, k, bs: int, sigma=None):
    """Pooled-key scorer, training shape: q [B,n,Hq,d], k [B,n,Hkv,d] ->
    s [B,Hkv,Cq,Cq] float64 with s[c,m] = sigma mean_q(block c) . mean_k(block m)
    for m < c, 0 for m >= c."""
    _same_code(np.asarray(q), np.asarray(k))
    qa, code, qp = _in(q)
    ka, _, kp = _in(k)
    B, n, Hq, d = qa.shape
    Hkv = ka.shape[2]
    if sigma is None:
        sigma = 1.0 / np.sqrt(d)
    Cq = n // bs
    s = np.zeros((B, Hkv, Cq, Cq), dtype=np.float64)
    rc = lib().oracle_pool_scores(B, n, Hq, Hkv, d, bs, ctypes.c_double(sigma), qp, kp, ctypes.c_int(code), _ptr(s))
    _check(rc, "pool_scores")
    return s


def pool_keys(k_cache, bs: int, m0: int, m1: int, nsum: int, round_bf16: bool = False, ksum=None):
    """Mean-pooled key summaries of full blocks [m0, m1) of k_cache [B,Hkv,Tmax,d]
    into ksum [B,Hkv,nsum,d] float64 (rounded to bf16 values when round_bf16)."""
    ka, code, kp = _in(k_cache)
    B, Hkv, Tmax, d = ka.shape
    if ksum is None:
        ksum = np.zeros((B, Hkv, nsum, d), dtype=np.float64)
    rc = lib().oracle_pool_keys(B, Hkv, Tmax, d, bs, kp, ctypes.c_int(code), m0, m1, nsum, int(round_bf16),
                                _ptr(ksum))
    _check(rc, "pool_keys")
    return ksum


def decode_scores(q, ksum, ctx_len, bs: int, s_cols: int, sigma=None):
    """Decode scores s [B,Hkv,s_cols] float64: sigma (mean over the group's heads of
    q) . ksum[b,h,m] for the full history blocks m < (ctx_len-1)//bs, else 0."""
    qa, code, qp = _in(q)
    B, Hq, d = qa.shape
    ks = np.ascontiguousarray(ksum, dtype=np.float64)
    Hkv, nsum = ks.shape[1], ks.shape[2]
    if sigma is None:
        sigma = 1.0 / np.sqrt(d)
    cl = np.ascontiguousarray(ctx_len, dtype=np.int32)
    s = np.zeros((B, Hkv, s_cols), dtype=np.float64)
    rc = lib().oracle_decode_scores(B, Hq, Hkv, d, bs, ctypes.c_double(sigma), qp, ctypes.c_int(code), _ptr(ks),
                                    nsum, _ptr(cl), s_cols, _ptr(s))
    _check(rc, "decode_scores")
    return s
