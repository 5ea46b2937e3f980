"""Shared helpers of the GPU parity tests: run the CUDA path through the binding,
hand the same input bits to the oracle, and compare element by element."""
from __future__ import annotations

import numpy as np
import torch

# tolerances: bf16 arithmetic (and fp32 outputs derived from bf16 math), and fp32 paths
BF16_TOL = dict(rel_l2=1e-2, max_abs=3e-2)
F32_TOL = dict(rel_l2=1e-4, max_abs=1e-4)


def bits(t: torch.Tensor) -> np.ndarray:
    """Exact host copy for the oracle: bf16 -> uint16 bit patterns, fp32 as is."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bfloat16 ulp at |x|: the rounding error of storing x in bf16."""
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def compare(name: str, got, want, rel_l2: float, max_abs: float, bf16_out: bool = False):
    """Relative L2 and max-abs error of got against the oracle.  For an output
    stored in bf16 the max-abs bound applies beyond the half-ulp rounding of the
    exact value to bf16, which no kernel can avoid (above |x| = 8 that rounding
    alone reaches 0.031)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = got - want
    denom = np.linalg.norm(want)
    rel = np.linalg.norm(err) / denom if denom > 0 else np.linalg.norm(err)
    excess = np.abs(err) - (bf16_half_ulp(want) if bf16_out else 0.0)
    mx = float(np.maximum(excess, 0.0).max()) if err.size else 0.0
    assert rel <= rel_l2 and mx <= max_abs, f"{name}: rel_l2 {rel:.3e} (<= {rel_l2}), max_abs {mx:.3e} (<= {max_abs})"
    return rel, mx


def run_train(api, inp: dict, bs: int, top_k: int, full_scope: bool, backward: bool = True, gate: str = "softmax"):
    q, k, v, s, dO = (inp[x] for x in ("q", "k", "v", "s", "dO"))
    desc = api.attn_desc(q, k, bs, top_k, full_scope, gate=gate)
    idx, lse_s = api.select_train(s, bs, top_k, full_scope)
    if gate in ("sigmoid", "raw"):
        lse_s = None  # these gates do not read the score LSE
    o = torch.empty_like(q)
    lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), dtype=torch.float32, device=q.device)
    api.sas_gated_attn_fwd(desc, q, k, v, s, lse_s, idx, o, lse)
    out = {"idx": idx, "lse_s": lse_s, "o": o, "lse": lse}
    if backward:
        dq, dk, dv, ds = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(s)
        ws = api.workspace(api.sas_gated_attn_bwd_workspace_size(desc), q.device)
        api.sas_gated_attn_bwd(desc, q, k, v, o, lse, dO, s, lse_s, idx, dq, dk, dv, ds, ws)
        out.update(dq=dq, dk=dk, dv=dv, ds=ds)
    torch.cuda.synchronize()
    return out
