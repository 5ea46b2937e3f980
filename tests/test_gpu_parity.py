"""GPU parity of the CUDA path (called through the C ABI) against the fp64 oracle.

Selection is compared bit for bit; floating-point outputs within the stated
tolerances (bf16: relative L2 <= 1e-2 and max |err| <= 3e-2; fp32: both <= 1e-4).
Full-size workloads run exactly as the benchmark runs them; the oracle then
checks sampled query blocks / key blocks of chosen KV heads (KV heads are
independent, so a head slice is an exact sub-problem)."""
import numpy as np
import pytest
import torch

import oracle
from parity import BF16_TOL, F32_TOL, bits, compare, host, run_train
from trainable_block_sparse_sas_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api(cuda_ok):
    from trainable_block_sparse_sas_b200 import api as a

    return a


def _seeded(shape, std, dtype, seed, device="cuda"):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype).to(device)


# --------------------------------------------------------------------------
# selection
# --------------------------------------------------------------------------

def _check_select(api, s, top_k, ctx_len=None, bs=0):
    B, Hkv, R, L = s.shape
    idx = torch.empty((B, Hkv, R, top_k), dtype=torch.int32, device="cuda")
    lse = torch.empty((B, Hkv, R), dtype=torch.float32, device="cuda")
    api.sas_topk_select(s, R, L, top_k, idx=idx, lse_s=lse, ctx_len=ctx_len, block_size=bs)
    torch.cuda.synchronize()
    if ctx_len is None:
        ncand = np.broadcast_to(np.minimum(np.arange(R), L)[None, None, :], (B, Hkv, R))
    else:
        c = np.minimum((ctx_len.cpu().numpy() - 1) // bs, L)
        ncand = np.broadcast_to(c[:, None, None], (B, Hkv, R))
    want_idx, want_lse = oracle.select(bits(s), ncand, top_k, idx_cols=top_k)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    got = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(want_lse)
    assert np.array_equal(np.isfinite(got), fin)
    compare("lse_s", got[fin], want_lse[fin], **F32_TOL)


def test_select_training_rows_bit_exact(api):
    s = _seeded((1, 8, 512, 512), 2.0, torch.float32, 11)
    _check_select(api, s, 32)


def test_select_ties_and_signed_zeros(api):
    s = _seeded((2, 3, 300, 300), 1.0, torch.float32, 12)
    s = torch.round(s * 2) / 2  # many exact ties
    s[0, 0] = 0.0
    s[0, 1, :, ::2] = -0.0
    s[1, 2] = 0.75
    for k in (1, 7, 64, 299, 300, 400):
        _check_select(api, s.contiguous(), k)


def test_select_long_rows_filter_and_fallback(api):
    """Rows of 1024..16384 blocks with K <= 64 take the staged threshold filter:
    tie-heavy training rows (every history length 0..1099 in one call), signed
    zeros, Top-K from 1 to 64 and past it (the radix kernel); all-equal decode rows,
    where every score is a candidate and the filter falls back to the radix
    select on the staged row."""
    s = _seeded((1, 2, 1100, 1100), 1.0, torch.float32, 15)
    s = torch.round(s * 2) / 2
    s[0, 1, :, ::3] = -0.0
    s[0, 1, :, 1::3] = 0.0
    for k in (1, 16, 64, 65):
        _check_select(api, s.contiguous(), k)
    for C, T in ((3000, 64 * 3000 + 1), (9000, 64 * 7000 + 5)):
        s = torch.full((2, 2, 1, C), 0.5, dtype=torch.float32, device="cuda")
        ctx = torch.tensor([T, 64 * 1500 + 1], dtype=torch.int32, device="cuda")
        _check_select(api, s, 64, ctx_len=ctx, bs=64)


def test_select_decode_rows_bit_exact(api):
    for B, Hkv, C, K, T in ((16, 8, 2048, 16, 131073), (4, 8, 8192, 32, 524289)):
        s = _seeded((B, Hkv, 1, C), 1.0, torch.float32, 13)
        ctx = torch.full((B,), T, dtype=torch.int32, device="cuda")
        _check_select(api, s, K, ctx_len=ctx, bs=64)
    s = _seeded((5, 2, 1, 40), 1.0, torch.float32, 14)
    ctx = torch.tensor([1, 64, 65, 200, 2560], dtype=torch.int32, device="cuda")  # 0, 0, 1, 3, 39 history blocks
    _check_select(api, s, 4, ctx_len=ctx, bs=64)


# --------------------------------------------------------------------------
# training-shape forward + backward, whole problems
# --------------------------------------------------------------------------

def _oracle_train(inp, bs, top_k, full_scope, gate="softmax"):
    """The exact oracle (fp64 on the inputs' bits, D_i = dO_i . o_i from the exact
    output) for every path: the tensor-core and the SIMT backward both take D from
    the exact output rather than from the rounded o the forward stored."""
    return oracle.attn_bwd(bits(inp["q"]), bits(inp["k"]), bits(inp["v"]), bits(inp["dO"]), bits(inp["s"]), bs,
                           top_k, full_scope=full_scope, gate=gate)


def _compare_train(got, want, tol, idx_want=None):
    if idx_want is not None and got["idx"] is not None:
        np.testing.assert_array_equal(got["idx"].cpu().numpy(), idx_want)
    b16 = got["o"].dtype == torch.bfloat16
    compare("o", host(got["o"]), want["o"], **tol, bf16_out=b16)
    compare("lse", host(got["lse"]), want["lse"], **tol)
    for key in ("dq", "dk", "dv"):
        compare(key, host(got[key]), want[key], **tol, bf16_out=b16)
    compare("ds", host(got["ds"]), want["ds"], **tol)


def test_tiny_fp32_workload(api):
    """The 1-KV-head fp32 workload (d=64, n=512, b=16, Top-K 4): every output at 1e-4."""
    w = syn.TINY_FP32
    inp = syn.train_inputs(w, device="cuda", seed=1000)
    got = run_train(api, inp, w.bs, w.top_k, w.full_scope)
    want = _oracle_train(inp, w.bs, w.top_k, w.full_scope)
    idx_want, _ = oracle.train_select(bits(inp["s"]), w.top_k)
    _compare_train(got, want, F32_TOL, idx_want)


@pytest.mark.parametrize("B,n,Hq,Hkv,d,bs,K,full", [
    (2, 512, 4, 1, 128, 64, 3, False),   # GQA 4, rows with c < K
    (1, 384, 5, 1, 64, 32, 4, False),    # GQA 5
    (1, 256, 2, 2, 128, 16, 5, False),   # no GQA, small blocks
    (1, 512, 8, 2, 128, 32, 6, False),   # GQA 4 over 2 KV heads, 32-token blocks
    (1, 512, 4, 2, 128, 64, 0, True),    # full scope
    (1, 256, 4, 2, 64, 64, 0, False),    # K = 0: current block only
    (1, 1024, 4, 1, 128, 64, 40, False), # K >= C: sparse == full
    (1, 512, 8, 1, 128, 64, 3, False),   # GQA 8: two CTAs per query block (tensor cores)
    (2, 512, 16, 2, 128, 64, 0, True),   # GQA 8, full scope
])
def test_bf16_shapes(api, B, n, Hq, Hkv, d, bs, K, full):
    Cq = n // bs
    inp = {
        "q": _seeded((B, n, Hq, d), 1.0, torch.bfloat16, 21),
        "k": _seeded((B, n, Hkv, d), 1.0, torch.bfloat16, 22),
        "v": _seeded((B, n, Hkv, d), 1.0, torch.bfloat16, 23),
        "s": _seeded((B, Hkv, Cq, Cq), 2.0, torch.float32, 24),
        "dO": _seeded((B, n, Hq, d), 1.0, torch.bfloat16, 25),
    }
    got = run_train(api, inp, bs, K, full)
    want = _oracle_train(inp, bs, K, full)
    idx_want = None if (full or K == 0) else oracle.train_select(bits(inp["s"]), K)[0]
    _compare_train(got, want, BF16_TOL, idx_want)
    tc = d == 128 and bs == 64 and Hq // Hkv in (2, 4, 8)
    want_path = ("tensor_core",) * 2 if tc else ("simt",) * 2
    assert api.sas_attn_path(api.attn_desc(inp["q"], inp["k"], bs, K, full)) == want_path


def test_fwd_lse_tight(api):
    """The forward's row log-sum-exp against the oracle at 3e-4 (natural-log units),
    far inside the bf16 tolerance of o: S is an fp32 accumulation of exact bf16
    products and the row sum is fp32, so an approximate exponential, a lost
    rescale of the running sum or a wrong log-gate bias shows here first."""
    B, n, Hq, Hkv, d, bs, K = 2, 1024, 8, 2, 128, 64, 6
    Cq = n // bs
    inp = {
        "q": _seeded((B, n, Hq, d), 1.0, torch.bfloat16, 31),
        "k": _seeded((B, n, Hkv, d), 1.0, torch.bfloat16, 32),
        "v": _seeded((B, n, Hkv, d), 1.0, torch.bfloat16, 33),
        "s": _seeded((B, Hkv, Cq, Cq), 2.0, torch.float32, 34),
        "dO": _seeded((B, n, Hq, d), 1.0, torch.bfloat16, 35),
    }
    got = run_train(api, inp, bs, K, False)
    want = _oracle_train(inp, bs, K, False)
    assert api.sas_attn_path(api.attn_desc(inp["q"], inp["k"], bs, K, False))[0] == "tensor_core"
    err = np.abs(host(got["lse"]) - want["lse"])
    assert err.max() <= 3e-4, err.max()


def test_unsupported_block_size_is_refused(api):
    q = torch.zeros((1, 256, 2, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 256, 1, 128), dtype=torch.bfloat16, device="cuda")
    s = torch.zeros((1, 1, 2, 2), dtype=torch.float32, device="cuda")
    desc = api.attn_desc(q, k, 128, 1)
    lse_s = torch.zeros((1, 1, 2), device="cuda")
    idx = torch.zeros((1, 1, 2, 1), dtype=torch.int32, device="cuda")
    o, lse = torch.empty_like(q), torch.empty((1, 2, 256), device="cuda")
    with pytest.raises(api.SasError) as e:
        api.sas_gated_attn_fwd(desc, q, k, k, s, lse_s, idx, o, lse)
    assert e.value.status == api.SAS_ERR_UNSUPPORTED


@pytest.mark.parametrize("gate", ["sigmoid", "raw", "outer", "ste"])
@pytest.mark.parametrize("dtype,d,bs,K,full,G", [
    (torch.bfloat16, 128, 64, 3, False, 2),  # tcgen05 kernels, sparse scope
    (torch.bfloat16, 128, 64, 0, True, 2),   # tcgen05 kernels, full scope
    (torch.bfloat16, 128, 64, 3, False, 8),  # tcgen05 kernels, GQA 8 (head-split dq CTAs add their ds)
    (torch.bfloat16, 64, 32, 4, False, 2),   # SIMT kernels (d = 64)
    (torch.bfloat16, 64, 32, 4, False, 5),   # SIMT kernels, GQA 5
    (torch.bfloat16, 128, 16, 5, False, 4),  # SIMT kernels, 16-token blocks
    (torch.float32, 128, 32, 3, False, 2),   # SIMT kernels, fp32
])
def test_gate_variants(api, gate, dtype, d, bs, K, full, G):
    """The ablated gates against the oracle, every output and gradient: log
    sigmoid(s) and raw-logit gates inside the softmax, the outer gate, and the hard
    STE gate (whose backward also walks the dropped blocks).  Unlike log_softmax
    the sigmoid and raw gates are not normalised, so one history block can hold
    nearly all of a row's mass (raw: weight e^s against the current block's 1);
    its dlogg then sums D_i over all G*b rows of the query block, which is what
    the exact D of both backward paths is tested on here."""
    B, n, Hkv = 1, 512, 2 if G < 5 or G == 8 else 1
    Hq = G * Hkv
    Cq = n // bs
    qk_std = 1.0 if dtype == torch.bfloat16 else 0.3
    inp = {
        "q": _seeded((B, n, Hq, d), qk_std, dtype, 41),
        "k": _seeded((B, n, Hkv, d), qk_std, dtype, 42),
        "v": _seeded((B, n, Hkv, d), 1.0, dtype, 43),
        "s": _seeded((B, Hkv, Cq, Cq), 2.0, torch.float32, 44),
        "dO": _seeded((B, n, Hq, d), 1.0, dtype, 45),
    }
    got = run_train(api, inp, bs, K, full, gate=gate)
    want = _oracle_train(inp, bs, K, full, gate=gate)
    idx_want = None if (full or K == 0) else oracle.train_select(bits(inp["s"]), K)[0]
    _compare_train(got, want, BF16_TOL if dtype == torch.bfloat16 else F32_TOL, idx_want)


def test_fp32_shape_with_gqa(api):
    B, n, Hq, Hkv, d, bs, K = 1, 256, 4, 2, 128, 32, 3
    Cq = n // bs
    inp = {
        "q": _seeded((B, n, Hq, d), 0.3, torch.float32, 31),
        "k": _seeded((B, n, Hkv, d), 0.3, torch.float32, 32),
        "v": _seeded((B, n, Hkv, d), 1.0, torch.float32, 33),
        "s": _seeded((B, Hkv, Cq, Cq), 1.0, torch.float32, 34),
        "dO": _seeded((B, n, Hq, d), 1.0, torch.float32, 35),
    }
    got = run_train(api, inp, bs, K, False)
    want = _oracle_train(inp, bs, K, False)
    _compare_train(got, want, F32_TOL)


def test_autograd_wrapper_matches_entry_points(api):
    w = syn.TINY_FP32
    inp = syn.train_inputs(w, device="cuda", seed=1001)
    direct = run_train(api, inp, w.bs, w.top_k, w.full_scope)
    q, k, v, s = (inp[x].clone().requires_grad_(True) for x in ("q", "k", "v", "s"))
    o = api.sas_attention(q, k, v, s, w.bs, w.top_k)
    o.backward(inp["dO"])
    torch.cuda.synchronize()
    for a, b in ((o, direct["o"]), (q.grad, direct["dq"]), (k.grad, direct["dk"]), (v.grad, direct["dv"]),
                 (s.grad, direct["ds"])):
        assert torch.equal(a, b)
    direct = run_train(api, inp, w.bs, w.top_k, w.full_scope, gate="sigmoid")
    q, k, v, s = (inp[x].clone().requires_grad_(True) for x in ("q", "k", "v", "s"))
    o = api.sas_attention(q, k, v, s, w.bs, w.top_k, gate="sigmoid")
    o.backward(inp["dO"])
    torch.cuda.synchronize()
    assert torch.equal(o, direct["o"]) and torch.equal(s.grad, direct["ds"])


# --------------------------------------------------------------------------
# full-size training workloads, sampled
# --------------------------------------------------------------------------

def _slice_inputs(inp, h, G):
    sl = slice(h * G, (h + 1) * G)
    return {
        "q": bits(inp["q"][:, :, sl]), "k": bits(inp["k"][:, :, h:h + 1]), "v": bits(inp["v"][:, :, h:h + 1]),
        "dO": bits(inp["dO"][:, :, sl]), "s": bits(inp["s"][:, h:h + 1]),
    }


def _sampled_full_size(api, w, q_blocks, kv_blocks, heads, gate="softmax"):
    inp = syn.train_inputs(w, device="cuda", seed=2000)
    got = run_train(api, inp, w.bs, w.top_k, w.full_scope, gate=gate)
    G, Cq, bs = w.Hq // w.Hkv, w.Cq, w.bs
    for h in heads:
        si = _slice_inputs(inp, h, G)
        sel = None
        if not w.full_scope:
            sel, _ = oracle.train_select(si["s"], w.top_k)
            np.testing.assert_array_equal(got["idx"][:, h:h + 1].cpu().numpy(), sel)
        qmask = np.zeros((1, 1, Cq), dtype=bool)
        kvmask = np.zeros((1, 1, Cq), dtype=bool)
        qmask[0, 0, list(q_blocks)] = True
        for m in kv_blocks:
            kvmask[0, 0, m] = True
            qmask[0, 0, m] = True
            for c in range(m + 1, Cq):
                if w.full_scope or m in sel[0, 0, c].tolist():
                    qmask[0, 0, c] = True
        want = oracle.attn_bwd(si["q"], si["k"], si["v"], si["dO"], si["s"], bs, w.top_k, full_scope=w.full_scope,
                               qmask=qmask, kvmask=kvmask, gate=gate)
        rows = np.concatenate([np.arange(c * bs, (c + 1) * bs) for c in q_blocks])
        hs = slice(h * G, (h + 1) * G)
        compare(f"o[h{h}]", host(got["o"][:, rows, hs]), want["o"][:, rows], **BF16_TOL, bf16_out=True)
        compare(f"lse[h{h}]", host(got["lse"][:, hs][:, :, rows]), want["lse"][:, :, rows], **BF16_TOL)
        compare(f"dq[h{h}]", host(got["dq"][:, rows, hs]), want["dq"][:, rows], **BF16_TOL, bf16_out=True)
        compare(f"ds[h{h}]", host(got["ds"][:, h, list(q_blocks)]), want["ds"][:, 0, list(q_blocks)], **BF16_TOL)
        krows = np.concatenate([np.arange(m * bs, (m + 1) * bs) for m in kv_blocks])
        compare(f"dk[h{h}]", host(got["dk"][:, krows, h]), want["dk"][:, krows, 0], **BF16_TOL, bf16_out=True)
        compare(f"dv[h{h}]", host(got["dv"][:, krows, h]), want["dv"][:, krows, 0], **BF16_TOL, bf16_out=True)


def test_train_sparse_32k_sampled(api):
    w = syn.TRAIN_SPARSE_32K
    _sampled_full_size(api, w, q_blocks=(0, 1, 31, 32, 33, 257, 511), kv_blocks=(511, 480, 350), heads=(0, 5))


@pytest.mark.parametrize("gate,kv_blocks", [("outer", (480, 100)), ("ste", (480,))])
def test_train_sparse_32k_gate_variants_sampled(api, gate, kv_blocks):
    """The outer and hard-STE gates on the full 32K workload, as the benchmark
    times them; the STE's dq kernel walks up to 511 dropped blocks per row."""
    w = syn.TRAIN_SPARSE_32K
    _sampled_full_size(api, w, q_blocks=(0, 1, 33, 257, 511), kv_blocks=kv_blocks, heads=(3,), gate=gate)


def test_train_sparse_32k_gqa8_sampled(api):
    """The 32K sparse workload with 8 query heads per KV head, on the tensor-core
    kernels (two dq CTAs per query block adding their ds shares)."""
    w = syn.TRAIN_SPARSE_32K_GQA8
    _sampled_full_size(api, w, q_blocks=(0, 1, 33, 257, 511), kv_blocks=(511, 200), heads=(0, 3))


def test_train_sparse_64k_two_q_stages_sampled(api):
    """64K tokens (1024 query blocks): the list of query blocks attending a key
    block no longer leaves room for a third Q stage, so the dk/dv kernel runs its
    two-stage Q ring; sampled key blocks with short and long lists."""
    import dataclasses

    w = dataclasses.replace(syn.TRAIN_SPARSE_32K, name="train_sparse_64k_small", Hq=8, Hkv=2, n=65536)
    _sampled_full_size(api, w, q_blocks=(0, 1, 33, 700, 1023), kv_blocks=(1022, 400), heads=(1,))


def test_train_full_16k_sampled(api):
    w = syn.TRAIN_FULL_16K
    _sampled_full_size(api, w, q_blocks=(0, 1, 100, 255), kv_blocks=(255, 250), heads=(3,))


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------

def _run_decode(api, inp, bs, top_k, dense=False, fused=False):
    q, kc, vc, ctx, s = (inp[x] for x in ("q", "k_cache", "v_cache", "ctx_len", "s"))
    B, Hkv = kc.shape[0], kc.shape[1]
    desc = api.decode_desc(q, kc, bs, top_k)
    if fused:
        idx = torch.full((B, Hkv, top_k), -7, dtype=torch.int32, device="cuda")
        o = torch.empty_like(q)
        api.sas_sparse_decode_select(desc, q, kc, vc, ctx, s, o, idx)
        torch.cuda.synchronize()
        return o, idx
    idx = None
    if not dense:
        idx = torch.empty((B, Hkv, top_k), dtype=torch.int32, device="cuda")
        api.sas_topk_select(s.view(B, Hkv, 1, -1), 1, s.shape[-1], top_k, idx=idx, ctx_len=ctx, block_size=bs)
    o = torch.empty_like(q)
    ws = api.workspace(api.sas_sparse_decode_workspace_size(desc), q.device)
    api.sas_sparse_decode(desc, q, kc, vc, ctx, idx, o, ws)
    torch.cuda.synchronize()
    return o, idx


def _oracle_decode_rows(inp, rows, bs, top_k, dense):
    """Oracle on (b, h) rows one at a time (caches sliced on the device first)."""
    G = inp["q"].shape[1] // inp["k_cache"].shape[1]
    outs = {}
    for b, h in rows:
        T = int(inp["ctx_len"][b])
        q = bits(inp["q"][b:b + 1, h * G:(h + 1) * G])
        kc = bits(inp["k_cache"][b:b + 1, h:h + 1, :T])
        vc = bits(inp["v_cache"][b:b + 1, h:h + 1, :T])
        s = bits(inp["s"][b:b + 1, h:h + 1])
        o, idx = oracle.decode(q, kc, vc, np.array([T], np.int32), s, bs, top_k, dense=dense)
        outs[(b, h)] = (o[0], idx[0, 0])
    return outs


@pytest.mark.parametrize("w", [syn.DECODE_128K, syn.DECODE_512K], ids=lambda w: w.name)
def test_decode_full_size_sampled(api, w):
    inp = syn.decode_inputs(w, device="cuda", seed=3000)
    o, idx = _run_decode(api, inp, w.bs, w.top_k)
    ncand = np.full((w.B, w.Hkv), w.C, dtype=np.int32)
    want_idx, _ = oracle.select(bits(inp["s"]), ncand, w.top_k)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    G = w.Hq // w.Hkv
    rows = [(0, 0), (w.B - 1, w.Hkv - 1), (w.B // 2, 3)]
    ref = _oracle_decode_rows(inp, rows, w.bs, w.top_k, dense=False)
    for (b, h), (ro, _) in ref.items():
        compare(f"decode o[{b},{h}]", host(o[b, h * G:(h + 1) * G]), ro, **BF16_TOL, bf16_out=True)
    of, idxf = _run_decode(api, inp, w.bs, w.top_k, fused=True)
    np.testing.assert_array_equal(idxf.cpu().numpy(), want_idx)
    for (b, h), (ro, _) in ref.items():
        compare(f"fused decode o[{b},{h}]", host(of[b, h * G:(h + 1) * G]), ro, **BF16_TOL, bf16_out=True)
    if w is syn.DECODE_512K:
        od, _ = _run_decode(api, inp, w.bs, w.top_k, dense=True)
        refd = _oracle_decode_rows(inp, rows[:2], w.bs, w.top_k, dense=True)
        for (b, h), (ro, _) in refd.items():
            compare(f"dense o[{b},{h}]", host(od[b, h * G:(h + 1) * G]), ro, **BF16_TOL, bf16_out=True)


@pytest.mark.parametrize("dtype,d,bs", [
    (torch.bfloat16, 128, 64),  # cluster kernel (tensor cores)
    (torch.bfloat16, 64, 64),   # split-K SIMT kernels, bf16
    (torch.bfloat16, 128, 32),  # split-K SIMT kernels, bf16, 32-token blocks
    (torch.float32, 64, 64),
    (torch.float32, 128, 64),
])
def test_decode_edge_cases(api, dtype, d, bs):
    """Ragged lengths (1 token, a block boundary, one token past it, ...), sparse,
    dense and fused-selection decode against the oracle, on every decode kernel."""
    B, Hq, Hkv, K, Tmax = 7, 10, 2, 3, 1100
    ctx = torch.tensor([1, 2, 64, 65, 129, 300, 1100], dtype=torch.int32, device="cuda")
    inp = {
        "q": _seeded((B, Hq, d), 1.0, dtype, 41),
        "k_cache": _seeded((B, Hkv, Tmax, d), 1.0, dtype, 42),
        "v_cache": _seeded((B, Hkv, Tmax, d), 1.0, dtype, 43),
        "ctx_len": ctx,
        "s": _seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 44),
    }
    tol = BF16_TOL if dtype == torch.bfloat16 else F32_TOL
    G = Hq // Hkv
    rows = [(b, h) for b in range(B) for h in range(Hkv)]
    modes = [("sparse", False, False), ("dense", True, False)]
    if dtype == torch.bfloat16 and d == 128 and bs == 64:
        modes.append(("fused", False, True))
    for name, dense, fused in modes:
        o, idx = _run_decode(api, inp, bs, K, dense=dense, fused=fused)
        ref = _oracle_decode_rows(inp, rows, bs, K, dense)
        for (b, h), (ro, ridx) in ref.items():
            if not dense:
                np.testing.assert_array_equal(idx[b, h].cpu().numpy(), ridx)
            compare(f"o[{b},{h}] {name}", host(o[b, h * G:(h + 1) * G]), ro, **tol,
                    bf16_out=dtype == torch.bfloat16)


def test_decode_cluster_sizes_and_ties(api):
    """Row counts that pick every cluster size (1..8 CTAs per row), tie-heavy scores
    (the selection splits equal keys across CTAs lowest index first), G = 1 and 8."""
    bs = 64
    # rows (B*Hkv) 1, 4, 16 -> 8 CTAs per row; 64 -> 4; 128 -> 2; 320 -> 1
    for B, Hq, Hkv, K, nblk in ((1, 8, 1, 40, 300), (2, 16, 2, 20, 300), (4, 8, 4, 9, 300), (8, 16, 8, 3, 60),
                                (16, 32, 8, 5, 40), (40, 8, 8, 3, 20), (3, 3, 3, 300, 300)):
        Tmax = 64 * nblk + 5
        ctx = torch.tensor([Tmax - 64 * (i % 3) for i in range(B)], dtype=torch.int32, device="cuda")
        s = torch.round(_seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 61) * 2) / 2
        inp = {
            "q": _seeded((B, Hq, 128), 1.0, torch.bfloat16, 62),
            "k_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 63),
            "v_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 64),
            "ctx_len": ctx, "s": s.contiguous(),
        }
        G = Hq // Hkv
        o, idx = _run_decode(api, inp, bs, K, fused=True)
        rows = [(b, h) for b in range(min(B, 3)) for h in range(Hkv)]
        ref = _oracle_decode_rows(inp, rows, bs, K, False)
        for (b, h), (ro, ridx) in ref.items():
            np.testing.assert_array_equal(idx[b, h].cpu().numpy(), ridx)
            compare(f"o[{b},{h}]", host(o[b, h * G:(h + 1) * G]), ro, **BF16_TOL, bf16_out=True)


def test_decode_selection_paths(api):
    """The fused selection's paths, each against the oracle: the per-CTA threshold
    filter (random scores); its fall-back to the radix select when more than 512
    keys reach the threshold (a score that depends only on the block index modulo
    the CTA's thread count, so whole threads' strides tie above it); and Top-K above
    the filter's limit of 64."""
    bs = 64
    nblk = 3000
    Tmax = bs * nblk + 7
    B, Hq, Hkv = 2, 4, 2
    base = {
        "q": _seeded((B, Hq, 128), 1.0, torch.bfloat16, 71),
        "k_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 72),
        "v_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 73),
        "ctx_len": torch.tensor([Tmax, Tmax - 200], dtype=torch.int32, device="cuda"),
    }
    C = Tmax // bs
    m = torch.arange(C, dtype=torch.float32, device="cuda")
    strided = ((m % 288) * 0.01).expand(B, Hkv, C).contiguous()
    strided[1, 1] += 0.003  # rows differ
    cases = (("filter", _seeded((B, Hkv, C), 1.0, torch.float32, 74), 48),
             ("radix fall-back", strided, 64),
             ("K above the filter", _seeded((B, Hkv, C), 1.0, torch.float32, 75), 100))
    G = Hq // Hkv
    rows = [(b, h) for b in range(B) for h in range(Hkv)]
    for name, s, K in cases:
        inp = dict(base, s=s)
        o, idx = _run_decode(api, inp, bs, K, fused=True)
        ref = _oracle_decode_rows(inp, rows, bs, K, False)
        for (b, h), (ro, ridx) in ref.items():
            np.testing.assert_array_equal(idx[b, h].cpu().numpy(), ridx, err_msg=f"{name} idx[{b},{h}]")
            compare(f"{name} o[{b},{h}]", host(o[b, h * G:(h + 1) * G]), ro, **BF16_TOL, bf16_out=True)


def test_decode_selection_long_rows_and_overflow(api):
    """Rows of 3000 and 6000 scores over clusters of 8 CTAs, with histories that
    end early in the row (a few blocks, or far fewer than the row holds), K up to
    64; and all-equal scores on long and 1500-score rows, where every score is a
    candidate and the selection falls back to the radix select (ties to the lower
    index)."""
    bs = 64
    B, Hq, Hkv = 2, 8, 2  # 4 rows: clusters of 8 CTAs
    G = Hq // Hkv
    rows = [(b, h) for b in range(B) for h in range(Hkv)]
    for name, nblk, hist, scores, K in (
            ("long, ragged", 3000, (3000, 2500), "random", 32),
            ("long, short", 3000, (2100, 9), "random", 5),
            ("long, K 64", 6000, (6000, 5000), "random", 64),
            ("long, all equal", 6000, (6000, 4000), "equal", 64),
            ("whole row, all equal", 1500, (1500, 1200), "equal", 40)):
        Tmax = bs * nblk + 3
        C = Tmax // bs
        ctx = torch.tensor([bs * hist[0] + 1, bs * hist[1] + 2], dtype=torch.int32, device="cuda")
        s = (_seeded((B, Hkv, C), 1.0, torch.float32, 81) if scores == "random"
             else torch.full((B, Hkv, C), 0.25, dtype=torch.float32, device="cuda"))
        inp = {"q": _seeded((B, Hq, 128), 1.0, torch.bfloat16, 82),
               "k_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 83),
               "v_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 84),
               "ctx_len": ctx, "s": s.contiguous()}
        o, idx = _run_decode(api, inp, bs, K, fused=True)
        ref = _oracle_decode_rows(inp, rows, bs, K, False)
        for (b, h), (ro, ridx) in ref.items():
            np.testing.assert_array_equal(idx[b, h].cpu().numpy(), ridx, err_msg=f"{name} idx[{b},{h}]")
            compare(f"{name} o[{b},{h}]", host(o[b, h * G:(h + 1) * G]), ro, **BF16_TOL, bf16_out=True)


def _paged_from_cache(kc, vc, bs, seed, spare=5):
    """Scatter contiguous caches [B, Hkv, T, d] into shuffled page pools
    [num_pages, bs, Hkv, d] (a few pages left unused) and the page table."""
    B, Hkv, T, d = kc.shape
    pps = (T + bs - 1) // bs
    num = B * pps + spare
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    table = torch.randperm(num, generator=g)[: B * pps].view(B, pps).to(torch.int32)
    pools = []
    for c in (kc, vc):
        padded = torch.nn.functional.pad(c, (0, 0, 0, pps * bs - T))  # [B, Hkv, pps*bs, d]
        pages = padded.view(B, Hkv, pps, bs, d).permute(0, 2, 3, 1, 4).reshape(B * pps, bs, Hkv, d)
        pool = torch.zeros((num, bs, Hkv, d), dtype=c.dtype, device=c.device)
        pool[table.view(-1).long().to(c.device)] = pages
        pools.append(pool)
    return pools[0], pools[1], table.to(kc.device)


def test_paged_decode_matches_oracle_and_contiguous(api):
    """Paged cache, ragged lengths: the fused selection (bit-exact blocks), given
    blocks, and dense attention against the oracle on the contiguous cache; given
    blocks also bit-identical to the contiguous-cache call."""
    bs, K = 64, 8
    B, Hq, Hkv = 3, 8, 2
    Tmax = bs * 40 + 7
    inp = {
        "q": _seeded((B, Hq, 128), 1.0, torch.bfloat16, 81),
        "k_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 82),
        "v_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 83),
        "ctx_len": torch.tensor([Tmax, Tmax - 150, 700], dtype=torch.int32, device="cuda"),
        "s": _seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 84),
    }
    kp, vp, table = _paged_from_cache(inp["k_cache"], inp["v_cache"], bs, 85)
    q = inp["q"]
    G = Hq // Hkv
    rows = [(b, h) for b in range(B) for h in range(Hkv)]
    desc = api.paged_decode_desc(q, kp, bs, K, Tmax)
    # fused selection
    o = torch.empty_like(q)
    idx = torch.full((B, Hkv, K), -7, dtype=torch.int32, device="cuda")
    api.sas_sparse_decode_paged(desc, q, kp, vp, table, inp["ctx_len"], o, s=inp["s"], idx_out=idx)
    torch.cuda.synchronize()
    ref = _oracle_decode_rows(inp, rows, bs, K, False)
    for (b, h), (ro, ridx) in ref.items():
        np.testing.assert_array_equal(idx[b, h].cpu().numpy(), ridx)
        compare(f"fused o[{b},{h}]", host(o[b, h * G:(h + 1) * G]), ro, **BF16_TOL, bf16_out=True)
    # given blocks: the same blocks, identical to the contiguous cache
    o2 = torch.empty_like(q)
    api.sas_sparse_decode_paged(desc, q, kp, vp, table, inp["ctx_len"], o2, idx=idx)
    o3, _ = _run_decode(api, dict(inp), bs, K, fused=True)
    torch.cuda.synchronize()
    assert torch.equal(o2, o3)
    assert torch.equal(o, o3)
    # dense
    o4 = torch.empty_like(q)
    api.sas_sparse_decode_paged(desc, q, kp, vp, table, inp["ctx_len"], o4)
    torch.cuda.synchronize()
    ref_d = _oracle_decode_rows(inp, rows, bs, K, True)
    for (b, h), (ro, _) in ref_d.items():
        compare(f"dense o[{b},{h}]", host(o4[b, h * G:(h + 1) * G]), ro, **BF16_TOL, bf16_out=True)


def test_paged_decode_in_cuda_graph_and_missing_pages(api):
    """The paged call captured in a CUDA graph replays with new q and scores; a
    page id outside the pool reads as zeros (dense check against the oracle on a
    cache with that block zeroed)."""
    bs, K = 64, 6
    B, Hq, Hkv = 2, 4, 1
    Tmax = bs * 24 + 3
    inp = {
        "q": _seeded((B, Hq, 128), 1.0, torch.bfloat16, 91),
        "k_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 92),
        "v_cache": _seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 93),
        "ctx_len": torch.tensor([Tmax, Tmax - 70], dtype=torch.int32, device="cuda"),
        "s": _seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 94),
    }
    kp, vp, table = _paged_from_cache(inp["k_cache"], inp["v_cache"], bs, 95)
    q = inp["q"].clone()
    s = inp["s"].clone()
    desc = api.paged_decode_desc(q, kp, bs, K, Tmax)
    o = torch.empty_like(q)
    idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        api.sas_sparse_decode_paged(desc, q, kp, vp, table, inp["ctx_len"], o, s=s, idx_out=idx)  # warm-up
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        api.sas_sparse_decode_paged(desc, q, kp, vp, table, inp["ctx_len"], o, s=s, idx_out=idx)
    q.copy_(_seeded((B, Hq, 128), 1.0, torch.bfloat16, 96))
    s.copy_(_seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 97))
    graph.replay()
    torch.cuda.synchronize()
    o_ref = torch.empty_like(q)
    idx_ref = torch.empty_like(idx)
    api.sas_sparse_decode_paged(desc, q, kp, vp, table, inp["ctx_len"], o_ref, s=s, idx_out=idx_ref)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref) and torch.equal(o, o_ref)
    del graph
    # a missing page: block 5 of sequence 0 points outside the pool
    table2 = table.clone()
    table2[0, 5] = kp.shape[0] + 3
    o_miss = torch.empty_like(q)
    api.sas_sparse_decode_paged(desc, q, kp, vp, table2, inp["ctx_len"], o_miss)
    torch.cuda.synchronize()
    zeroed = dict(inp, q=q)
    zeroed["k_cache"] = inp["k_cache"].clone()
    zeroed["v_cache"] = inp["v_cache"].clone()
    zeroed["k_cache"][0, :, 5 * bs:6 * bs] = 0
    zeroed["v_cache"][0, :, 5 * bs:6 * bs] = 0
    ref = _oracle_decode_rows(zeroed, [(0, 0)], bs, K, True)
    G = Hq // Hkv
    compare("missing-page o", host(o_miss[0, 0:G]), ref[(0, 0)][0], **BF16_TOL, bf16_out=True)


# --------------------------------------------------------------------------
# pooled-key scorer
# --------------------------------------------------------------------------

@pytest.mark.parametrize("B,n,Hq,Hkv,d,bs,dtype", [
    (1, 1024, 8, 2, 128, 64, torch.bfloat16),  # G 4, the training workloads' geometry
    (2, 480, 5, 1, 64, 32, torch.bfloat16),    # G 5, ragged count of 32-blocks (Cq 15)
    (1, 256, 4, 2, 64, 16, torch.float32),
    (1, 192, 2, 2, 128, 64, torch.float32),    # Cq 3: one tile
])
def test_pooled_scores_match_oracle(api, B, n, Hq, Hkv, d, bs, dtype):
    q = _seeded((B, n, Hq, d), 1.0, dtype, 51)
    k = _seeded((B, n, Hkv, d), 1.0, dtype, 52)
    desc = api.attn_desc(q, k, bs, 0)
    s = torch.full((B, Hkv, n // bs, n // bs), float("nan"), device="cuda")
    ws = api.workspace(api.sas_pooled_scores_workspace_size(desc), q.device)
    api.sas_pooled_scores(desc, q, k, s, ws)
    torch.cuda.synchronize()
    want = oracle.pool_scores(bits(q), bits(k), bs)
    compare("s", host(s), want, **F32_TOL)
    assert torch.all(torch.triu(s) == 0)  # m >= c: exactly 0


def test_pooled_scores_full_size_and_selection(api):
    """train_sparse_32k geometry: scores of two KV heads against the oracle, then
    the selection of the GPU's scores, bit for bit against the oracle's."""
    w = syn.TRAIN_SPARSE_32K
    inp = syn.train_inputs(w, device="cuda", seed=2100)
    desc = api.attn_desc(inp["q"], inp["k"], w.bs, w.top_k)
    s = torch.empty((w.B, w.Hkv, w.Cq, w.Cq), device="cuda")
    ws = api.workspace(api.sas_pooled_scores_workspace_size(desc), inp["q"].device)
    api.sas_pooled_scores(desc, inp["q"], inp["k"], s, ws)
    idx, _ = api.select_train(s, w.bs, w.top_k)
    torch.cuda.synchronize()
    G = w.Hq // w.Hkv
    for h in (0, w.Hkv - 1):
        want = oracle.pool_scores(bits(inp["q"][:, :, h * G:(h + 1) * G]), bits(inp["k"][:, :, h:h + 1]), w.bs)
        compare(f"s[h{h}]", host(s[:, h:h + 1]), want, **F32_TOL)
        want_idx, _ = oracle.train_select(bits(s[:, h:h + 1]), w.top_k)
        np.testing.assert_array_equal(idx[:, h:h + 1].cpu().numpy(), want_idx)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_decode_scores_match_oracle(api, dtype, d):
    """Block summaries (built in two calls, as a cache grows), then the decode
    scores: summaries within half a bf16 ulp of the exact means, scores against
    the oracle on the GPU's summaries and on the oracle's own rounded ones."""
    B, Hq, Hkv, bs, Tmax = 4, 8, 2, 64, 64 * 40 + 5
    q = _seeded((B, Hq, d), 1.0, dtype, 61)
    kc = _seeded((B, Hkv, Tmax, d), 1.0, dtype, 62)
    ctx = torch.tensor([1, 65, 64 * 17 + 3, Tmax], dtype=torch.int32, device="cuda")  # 0, 1, 17, 40 blocks
    nsum = 40
    desc = api.decode_desc(q, kc, bs, 4)
    ksum = torch.zeros((B, Hkv, nsum, d), dtype=dtype, device="cuda")
    api.sas_pool_key_blocks(desc, kc, 0, 25, ksum)
    api.sas_pool_key_blocks(desc, kc, 25, 40, ksum)
    s_cols = 48
    s = torch.full((B, Hkv, s_cols), float("nan"), device="cuda")
    api.sas_decode_scores(desc, q, ksum, ctx, s)
    torch.cuda.synchronize()
    want_sum = oracle.pool_keys(bits(kc), bs, 0, nsum, nsum, round_bf16=dtype == torch.bfloat16)
    # the summaries against the exact means: within the bf16 storage rounding (plus the fp32 sum's error)
    exact_sum = oracle.pool_keys(bits(kc), bs, 0, nsum, nsum)
    compare("ksum", host(ksum), exact_sum, rel_l2=4e-3 if dtype == torch.bfloat16 else 1e-6, max_abs=1e-6,
            bf16_out=dtype == torch.bfloat16)
    got_sum = host(ksum)
    compare("s (GPU summaries)", host(s), oracle.decode_scores(bits(q), got_sum, ctx.cpu().numpy(), bs, s_cols),
            **F32_TOL)
    compare("s", host(s), oracle.decode_scores(bits(q), want_sum, ctx.cpu().numpy(), bs, s_cols),
            **(BF16_TOL if dtype == torch.bfloat16 else F32_TOL))
    Cb = (ctx.cpu().numpy() - 1) // bs
    for b in range(B):
        assert torch.all(s[b, :, int(Cb[b]):] == 0)


def test_paged_key_summaries_match_contiguous(api):
    """Summaries pooled from a shuffled page pool equal, bit for bit, those pooled
    from the contiguous cache (same rows, same order of the sums); a page id
    outside the pool gives a zero summary."""
    B, Hq, Hkv, d, bs, Tmax = 3, 8, 2, 128, 64, 64 * 40 + 5
    q = _seeded((B, Hq, d), 1.0, torch.bfloat16, 81)
    kc = _seeded((B, Hkv, Tmax, d), 1.0, torch.bfloat16, 82)
    vc = _seeded((B, Hkv, Tmax, d), 1.0, torch.bfloat16, 83)
    kp, _, table = _paged_from_cache(kc, vc, bs, 84)
    desc = api.decode_desc(q, kc, bs, 4)
    nsum = 40
    want = torch.zeros((B, Hkv, nsum, d), dtype=torch.bfloat16, device="cuda")
    got = torch.full_like(want, float("nan"))
    api.sas_pool_key_blocks(desc, kc, 0, nsum, want)
    api.sas_pool_key_blocks_paged(desc, kp, table, 0, 17, got)
    api.sas_pool_key_blocks_paged(desc, kp, table, 17, nsum, got)
    bad = table.clone()
    bad[1, 5] = kp.shape[0] + 7
    got_bad = torch.full_like(want, float("nan"))
    api.sas_pool_key_blocks_paged(desc, kp, bad, 0, nsum, got_bad)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    assert torch.all(got_bad[1, :, 5] == 0)
    got_bad[1, :, 5] = want[1, :, 5]
    assert torch.equal(got_bad, want)


def test_training_step_in_cuda_graph(api):
    """Select, forward and backward captured in one CUDA graph and replayed on new
    inputs copied into the captured buffers: bit-identical to the eager calls
    (no host synchronisation or allocation happens inside the calls)."""
    B, n, Hq, Hkv, d, bs, K = 1, 1024, 8, 2, 128, 64, 4
    Cq = n // bs

    def make(seed):
        return {"q": _seeded((B, n, Hq, d), 1.0, torch.bfloat16, seed),
                "k": _seeded((B, n, Hkv, d), 1.0, torch.bfloat16, seed + 1),
                "v": _seeded((B, n, Hkv, d), 1.0, torch.bfloat16, seed + 2),
                "s": _seeded((B, Hkv, Cq, Cq), 2.0, torch.float32, seed + 3),
                "dO": _seeded((B, n, Hq, d), 1.0, torch.bfloat16, seed + 4)}

    buf = make(91)
    desc = api.attn_desc(buf["q"], buf["k"], bs, K)
    idx = torch.empty((B, Hkv, Cq, K), dtype=torch.int32, device="cuda")
    lse_s = torch.empty((B, Hkv, Cq), device="cuda")
    o = torch.empty_like(buf["q"])
    lse = torch.empty((B, Hq, n), device="cuda")
    dq, dk, dv, ds = (torch.empty_like(buf[x]) for x in ("q", "k", "v", "s"))
    ws = api.workspace(api.sas_gated_attn_bwd_workspace_size(desc), buf["q"].device)

    def step():
        api.sas_topk_select(buf["s"], Cq, Cq, K, idx=idx, lse_s=lse_s)
        api.sas_gated_attn_fwd(desc, buf["q"], buf["k"], buf["v"], buf["s"], lse_s, idx, o, lse)
        api.sas_gated_attn_bwd(desc, buf["q"], buf["k"], buf["v"], o, lse, buf["dO"], buf["s"], lse_s, idx, dq, dk,
                               dv, ds, ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # warm-up outside the capture (kernel attributes set once)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    new = make(191)
    for x in buf:
        buf[x].copy_(new[x])
    graph.replay()
    torch.cuda.synchronize()
    got = [t.clone() for t in (idx, o, lse, dq, dk, dv, ds)]
    step()
    torch.cuda.synchronize()
    for g_, e_ in zip(got, (idx, o, lse, dq, dk, dv, ds)):
        assert torch.equal(g_, e_)
    want = oracle.attn_bwd(bits(new["q"]), bits(new["k"]), bits(new["v"]), bits(new["dO"]), bits(new["s"]), bs, K)
    compare("o", host(got[1]), want["o"], **BF16_TOL, bf16_out=True)
    compare("ds", host(got[6]), want["ds"], **BF16_TOL)
    del graph
