"""Seeded synthetic inputs for the SAS hot path.

This module only draws random tensors of the workloads' shapes and value
distributions; it holds none of the method's arithmetic.  Both the CUDA path
(bench, GPU tests) and the CPU oracle (tests) consume what it produces.

Workloads (shapes and distributions of the Qwen3 settings the SAS reviews report: block size 64,
training length 32768, budgets of 1024 / 2048 tokens):
  tiny_fp32          B=1, 1 KV head, 2 query heads, d=64, n=512, b=16, Top-K 4, fp32,
                     q,k,v ~ N(0,1)/8, s ~ N(0,1), dO ~ N(0,1)
  train_sparse_32k   B=1, Hq=32, Hkv=8, d=128, n=32768, b=64, Top-K 32, bf16,
                     q,k,v ~ N(0,1), s ~ N(0,2^2) fp32, dO ~ N(0,1)
  train_full_16k     as above with n=16384, every history block attended (full scope)
  decode_128k        B=16, Hq=32, Hkv=8, d=128, 131073 cached tokens, b=64, Top-K 16,
                     bf16 K/V ~ N(0,1), s ~ N(0,1) fp32 per (sequence, kv head, block)
  decode_512k        B=4, Hq=40, Hkv=8, d=128, 524289 cached tokens, b=64, Top-K 32
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class TrainShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    n: int
    bs: int
    top_k: int
    full_scope: bool
    dtype: torch.dtype
    qkv_std: float
    s_std: float

    @property
    def Cq(self) -> int:
        return self.n // self.bs


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int  # cached tokens including the new one
    bs: int
    top_k: int
    dtype: torch.dtype
    s_std: float

    @property
    def C(self) -> int:
        """History blocks before the current (partial) block of the new token."""
        return (self.T - 1) // self.bs


TINY_FP32 = TrainShape("tiny_fp32", 1, 2, 1, 64, 512, 16, 4, False, torch.float32, 1.0 / 8.0, 1.0)
TRAIN_SPARSE_32K = TrainShape("train_sparse_32k", 1, 32, 8, 128, 32768, 64, 32, False, torch.bfloat16, 1.0, 2.0)
TRAIN_FULL_16K = TrainShape("train_full_16k", 1, 32, 8, 128, 16384, 64, 0, True, torch.bfloat16, 1.0, 2.0)
# the 32K sparse workload with 8 query heads per KV head (4 KV heads)
TRAIN_SPARSE_32K_GQA8 = TrainShape("train_sparse_32k_gqa8", 1, 32, 4, 128, 32768, 64, 32, False, torch.bfloat16, 1.0,
                                   2.0)
DECODE_128K = DecodeShape("decode_128k", 16, 32, 8, 128, 131073, 64, 16, torch.bfloat16, 1.0)
DECODE_512K = DecodeShape("decode_512k", 4, 40, 8, 128, 524289, 64, 32, torch.bfloat16, 1.0)

WORKLOADS = {w.name: w for w in (TINY_FP32, TRAIN_SPARSE_32K, TRAIN_FULL_16K, TRAIN_SPARSE_32K_GQA8, DECODE_128K,
                                  DECODE_512K)}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, std, dtype, device, seed):
    g = _gen(device, seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def train_inputs(w: TrainShape, device="cpu", seed: int = 1000) -> dict:
    """q, dO [B,n,Hq,d]; k, v [B,n,Hkv,d]; s [B,Hkv,Cq,Cq] fp32 (row c scores blocks m < c)."""
    q = _randn((w.B, w.n, w.Hq, w.d), w.qkv_std, w.dtype, device, seed + 0)
    k = _randn((w.B, w.n, w.Hkv, w.d), w.qkv_std, w.dtype, device, seed + 1)
    v = _randn((w.B, w.n, w.Hkv, w.d), w.qkv_std, w.dtype, device, seed + 2)
    s = _randn((w.B, w.Hkv, w.Cq, w.Cq), w.s_std, torch.float32, device, seed + 3)
    dO = _randn((w.B, w.n, w.Hq, w.d), 1.0, w.dtype, device, seed + 4)
    return {"q": q, "k": k, "v": v, "s": s, "dO": dO}


def decode_inputs(w: DecodeShape, device="cpu", seed: int = 3000, chunk_tokens: int = 1 << 16) -> dict:
    """q [B,Hq,d]; k_cache, v_cache [B,Hkv,T,d]; ctx_len [B] int32 (= T); s [B,Hkv,C] fp32."""
    q = _randn((w.B, w.Hq, w.d), 1.0, w.dtype, device, seed + 0)
    caches = []
    for which in (1, 2):
        c = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=w.dtype, device=device)
        g = _gen(device, seed + which)
        for t0 in range(0, w.T, chunk_tokens):
            t1 = min(w.T, t0 + chunk_tokens)
            c[:, :, t0:t1].copy_(torch.randn((w.B, w.Hkv, t1 - t0, w.d), generator=g, device=device))
        caches.append(c)
    s = _randn((w.B, w.Hkv, max(w.C, 1)), w.s_std, torch.float32, device, seed + 3)
    ctx_len = torch.full((w.B,), w.T, dtype=torch.int32, device=device)
    return {"q": q, "k_cache": caches[0], "v_cache": caches[1], "ctx_len": ctx_len, "s": s}


def bf16_bits(t: torch.Tensor):
    """Host numpy view of a tensor's exact bits for the oracle: float32/float64
    arrays as they are, bfloat16 as uint16 bit patterns."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()
