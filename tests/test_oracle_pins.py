"""Pins of the fp64 CPU oracle against facts fixed by the SAS reviews and by mathematics.

None of these tests touches a GPU.  Each pin is independent of the oracle's own
code: printed values of the jaehun.me review's worked example, brute-force selection, dense
attention and its autograd gradients from torch (fp64), an explicit dense-mask
formulation of the gated attention differentiated by torch autograd, central
finite differences, the inner-gate gradient identity (jaehun.me review, "Why the Four
Design Choices Matter", quoting the paper's Eq. 5),
and invariants (shift invariance of s, ds summing to zero, sparse == full scope
when the budget covers the history).
"""
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [float(x) for x in rest]
    return vals


def _rand_train(rng, B, n, Hq, Hkv, d, bs, s_std=1.0, qk_std=0.5):
    Cq = n // bs
    q = rng.standard_normal((B, n, Hq, d)) * qk_std
    k = rng.standard_normal((B, n, Hkv, d)) * qk_std
    v = rng.standard_normal((B, n, Hkv, d))
    s = rng.standard_normal((B, Hkv, Cq, Cq)) * s_std
    dO = rng.standard_normal((B, n, Hq, d))
    return q, k, v, s, dO


def _brute_select(row, c, K):
    if K >= c:
        return list(range(c))
    order = sorted(range(c), key=lambda m: (-row[m], m))
    return sorted(order[:K])


# --------------------------------------------------------------------------
# worked example (jaehun.me review, walkthrough Steps 1-4)
# --------------------------------------------------------------------------

def test_worked_example_gate_and_topk():
    g = _golden("worked_example.txt")
    s_row = np.array(g["scores"])
    C, K = len(s_row), int(g["top_k"][0])
    assert int(g["n"][0]) // int(g["block_size"][0]) == C
    # query in block C (0-based) sees history blocks 0..C-1 with the printed scores
    s = np.zeros((1, 1, C + 1, C + 1))
    s[0, 0, C, :C] = s_row
    idx, lse = oracle.train_select(s, K)
    assert sorted(idx[0, 0, C].tolist()) == sorted(int(x) for x in g["topk_0based"])
    assert idx[0, 0, C].tolist() == sorted(idx[0, 0, C].tolist())  # ascending
    L = lse[0, 0, C]
    assert abs(np.exp(L) - g["exp_sum"][0]) <= g["exp_sum_tol"][0]
    np.testing.assert_allclose(np.exp(s_row), g["exp_scores"], atol=g["exp_scores_tol"][0])
    np.testing.assert_allclose(s_row - L, g["log_gate"], atol=g["log_gate_tol"][0])
    # gates are a distribution over the history blocks
    assert abs(np.exp(s_row - L).sum() - 1.0) < 1e-12


def test_worked_example_attention_mass_closed_form():
    """With q = 0 every logit equals its bias, so the attention mass of a selected
    block is bs*g_m / (sum over selected bs*g + number of current-block keys):
    the current block carries gate 1 and unselected blocks get nothing (Eq. 9)."""
    g = _golden("worked_example.txt")
    s_row = np.array(g["scores"])
    C, K, bs = len(s_row), int(g["top_k"][0]), int(g["block_size"][0])
    n = (C + 1) * bs
    d = C + 1
    q = np.zeros((1, n, 1, d))
    k = np.random.default_rng(0).standard_normal((1, n, 1, d))
    v = np.zeros((1, n, 1, d))
    for j in range(n):
        v[0, j, 0, j // bs] = 1.0  # one-hot block indicator
    s = np.zeros((1, 1, C + 1, C + 1))
    s[0, 0, C, :C] = s_row
    o, lse = oracle.attn_fwd(q, k, v, s, bs, K)
    gate = np.exp(s_row - scipy.special.logsumexp(s_row))
    sel = _brute_select(s_row, C, K)
    for i in (C * bs, C * bs + 17, n - 1):
        cur = i - C * bs + 1
        denom = bs * gate[sel].sum() + cur
        for m in range(C):
            want = bs * gate[m] / denom if m in sel else 0.0
            assert abs(o[0, i, 0, m] - want) < 1e-13
        assert abs(o[0, i, 0, C] - cur / denom) < 1e-13
        assert abs(lse[0, 0, i] - np.log(denom)) < 1e-13


# --------------------------------------------------------------------------
# selection: brute force, ties, signed zeros, degenerate budgets
# --------------------------------------------------------------------------

def test_select_brute_force_with_ties():
    rng = np.random.default_rng(1)
    rows, L = 300, 70
    s = rng.standard_normal((rows, L)).astype(np.float32)
    s[::3] = np.round(s[::3] * 2) / 2  # many exact ties
    s[5, :] = 0.0
    s[6, ::2] = -0.0  # signed zeros compare equal
    s[7, :] = np.float32(1.25)
    ncand = rng.integers(0, L + 1, size=rows).astype(np.int32)
    ncand[:4] = [0, 1, L, 2]
    for K in (0, 1, 4, 16, 69, 70, 100):
        idx, lse = oracle.select(s, ncand, K, idx_cols=max(K, 1))
        for r in range(rows):
            c = int(ncand[r])
            want = _brute_select([float(x) for x in s[r]], c, K)
            got = [x for x in idx[r].tolist() if x >= 0][: max(K, 0)]
            assert got == want, (r, K)
            assert all(x == -1 for x in idx[r].tolist()[len(want):])
            if c == 0:
                assert lse[r] == -np.inf
            else:
                assert abs(lse[r] - scipy.special.logsumexp(s[r, :c].astype(np.float64))) < 1e-12


def test_select_full_scope_keeps_all_history():
    s = np.random.default_rng(2).standard_normal((1, 2, 9, 9))
    idx, _ = oracle.select(s, np.arange(9)[None, None, :], 2, full_scope=True, idx_cols=9)
    for c in range(9):
        assert idx[0, 1, c].tolist() == list(range(c)) + [-1] * (9 - c)


# --------------------------------------------------------------------------
# forward / backward against torch (fp64) library routines
# --------------------------------------------------------------------------

def _dense_masked_torch(q, k, v, s, bs, K, sigma, full_scope=False, gate=True):
    """Explicit dense formulation of Eq. 9 with torch: an n x n bias matrix holding
    log g (log_softmax(s); or logsigmoid(s) / s for the "sigmoid" / "raw" gate
    variants) on the selected history blocks, 0 on the causal current block and
    -inf elsewhere; softmax / matmul from torch.  Selection by brute force."""
    B, n, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    Cq = n // bs
    outs = []
    for b in range(B):
        heads = []
        for hq in range(Hq):
            h = hq // G
            rows = []
            for c in range(Cq):
                bias = torch.full((bs, n), float("-inf"), dtype=torch.float64)
                if c > 0:
                    if gate == "sigmoid":
                        logg = torch.nn.functional.logsigmoid(s[b, h, c, :c])
                    elif gate == "raw":
                        logg = s[b, h, c, :c]
                    else:
                        logg = torch.log_softmax(s[b, h, c, :c], dim=0)
                    row = s[b, h, c, :c].detach().tolist()
                    sel = list(range(c)) if full_scope else _brute_select(row, c, K)
                    for m in sel:
                        bias[:, m * bs:(m + 1) * bs] = (logg[m] if gate else 0.0)
                causal = torch.full((bs, bs), float("-inf"), dtype=torch.float64).triu(1)
                bias[:, c * bs:(c + 1) * bs] = causal
                rows.append(bias)
            bias = torch.cat(rows, 0)
            z = sigma * q[b, :, hq] @ k[b, :, h].T + bias
            p = torch.softmax(z, dim=-1)
            heads.append((p @ v[b, :, h], torch.logsumexp(z, dim=-1)))
        outs.append(heads)
    o = torch.stack([torch.stack([hd[0] for hd in bh], 1) for bh in outs], 0)
    lse = torch.stack([torch.stack([hd[1] for hd in bh], 0) for bh in outs], 0)
    return o, lse


@pytest.mark.parametrize("full_scope", [False, True])
def test_gated_fwd_bwd_vs_torch_dense_mask(full_scope):
    rng = np.random.default_rng(3)
    B, n, Hq, Hkv, d, bs, K = 2, 64, 4, 2, 16, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    sigma = 1 / np.sqrt(d)
    out = oracle.attn_bwd(q, k, v, dO, s, bs, K, full_scope=full_scope, sigma=sigma)
    o_fwd, lse_fwd = oracle.attn_fwd(q, k, v, s, bs, K, full_scope=full_scope, sigma=sigma)
    T = [torch.tensor(x, requires_grad=True) for x in (q, k, v, s)]
    o_t, lse_t = _dense_masked_torch(*T, bs, K, sigma, full_scope=full_scope)
    (o_t * torch.tensor(dO)).sum().backward()
    np.testing.assert_allclose(o_fwd, o_t.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(out["o"], o_fwd, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse_fwd, lse_t.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(out["lse"], lse_fwd, atol=1e-12, rtol=0)
    for name, t in zip(("dq", "dk", "dv", "ds"), T):
        ref = t.grad.numpy()
        np.testing.assert_allclose(out[name], ref, atol=1e-11, rtol=0, err_msg=name)


def test_gate_off_budget_covering_history_is_dense_causal_attention():
    rng = np.random.default_rng(4)
    B, n, Hq, Hkv, d, bs = 1, 48, 6, 2, 8, 8
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    K = n // bs
    out = oracle.attn_bwd(q, k, v, dO, s, bs, K, gate=False)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    G = Hq // Hkv
    o_ref = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(1, 2), tk.repeat_interleave(G, 2).transpose(1, 2), tv.repeat_interleave(G, 2).transpose(1, 2),
        is_causal=True).transpose(1, 2)
    (o_ref * torch.tensor(dO)).sum().backward()
    np.testing.assert_allclose(out["o"], o_ref.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(out["dq"], tq.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(out["dk"], tk.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(out["dv"], tv.grad.numpy(), atol=1e-11, rtol=0)
    assert np.all(out["ds"] == 0.0)


def test_zero_budget_is_block_local_causal_attention():
    rng = np.random.default_rng(5)
    B, n, Hq, Hkv, d, bs = 1, 40, 2, 1, 8, 8
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    o, lse = oracle.attn_fwd(q, k, v, s, bs, 0)
    blk = np.arange(n) // bs
    mask = (blk[:, None] == blk[None, :]) & (np.arange(n)[:, None] >= np.arange(n)[None, :])
    am = torch.where(torch.tensor(mask), 0.0, float("-inf")).double()
    o_ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q).transpose(1, 2), torch.tensor(k).repeat_interleave(2, 2).transpose(1, 2),
        torch.tensor(v).repeat_interleave(2, 2).transpose(1, 2), attn_mask=am).transpose(1, 2)
    np.testing.assert_allclose(o, o_ref.numpy(), atol=1e-12, rtol=0)


def test_sparse_scope_equals_full_scope_when_budget_covers_history():
    rng = np.random.default_rng(6)
    B, n, Hq, Hkv, d, bs = 1, 48, 4, 2, 8, 8
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    a = oracle.attn_bwd(q, k, v, dO, s, bs, n // bs, full_scope=False)
    b = oracle.attn_bwd(q, k, v, dO, s, bs, 0, full_scope=True)
    for key in ("o", "lse", "dq", "dk", "dv", "ds"):
        np.testing.assert_array_equal(a[key], b[key])


def test_score_shift_invariance():
    """o depends on s only through log g = s - LSE(s): s -> s + c changes nothing."""
    rng = np.random.default_rng(7)
    B, n, Hq, Hkv, d, bs, K = 1, 64, 2, 1, 8, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    a = oracle.attn_bwd(q, k, v, dO, s, bs, K)
    b = oracle.attn_bwd(q, k, v, dO, s + 3.75, bs, K)
    for key in ("o", "lse", "dq", "dk", "dv", "ds"):
        np.testing.assert_allclose(a[key], b[key], atol=1e-12, rtol=0, err_msg=key)


# --------------------------------------------------------------------------
# gradients: finite differences, Eq. 5, ds invariants
# --------------------------------------------------------------------------

def test_central_finite_differences():
    rng = np.random.default_rng(8)
    B, n, Hq, Hkv, d, bs, K = 1, 32, 2, 1, 4, 8, 2
    q, k, v, _, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    Cq = n // bs
    # scores with gaps of >= 0.05 so that a 1e-6 step never changes the selection
    s = (rng.permutation(Cq * Cq).reshape(1, 1, Cq, Cq) * 0.05 + rng.uniform(0, 0.01, (1, 1, Cq, Cq)))
    out = oracle.attn_bwd(q, k, v, dO, s, bs, K)
    eps = 1e-6

    def loss(q_, k_, v_, s_):
        o, _ = oracle.attn_fwd(q_, k_, v_, s_, bs, K)
        return float((o * dO).sum())

    for name, arr, pos in (("dq", q, 0), ("dk", k, 1), ("dv", v, 2), ("ds", s, 3)):
        grad = out[name]
        flat_idx = rng.choice(arr.size, size=min(arr.size, 40), replace=False)
        for fi in flat_idx:
            ix = np.unravel_index(fi, arr.shape)
            args_p = [q, k, v, s]
            args_m = [q, k, v, s]
            ap, am = arr.copy(), arr.copy()
            ap[ix] += eps
            am[ix] -= eps
            args_p[pos], args_m[pos] = ap, am
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[ix]) <= 1e-6 * max(1.0, abs(grad[ix])), (name, ix, fd, grad[ix])


def test_inner_gate_gradient_identity_eq5():
    """The inner-gate gradient (jaehun.me review, "Why the Four Design Choices Matter", the
    paper's Eq. 5): dg_m = sum_{i in B_m} (p_i/g_m) do.(v_i - o),
    i.e. d(log g)_m = sum_{i in B_m} p_i do.(v_i - o), summed over the query rows
    sharing the score row.  Evaluated here from the forward outputs only."""
    rng = np.random.default_rng(9)
    B, n, Hq, Hkv, d, bs, K = 1, 64, 4, 2, 8, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    sigma = 1 / np.sqrt(d)
    out = oracle.attn_bwd(q, k, v, dO, s, bs, K, sigma=sigma)
    o, lse = oracle.attn_fwd(q, k, v, s, bs, K, sigma=sigma)
    G, Cq = Hq // Hkv, n // bs
    for h in range(Hkv):
        for c in range(1, Cq):
            row = s[0, h, c, :c]
            logg = row - scipy.special.logsumexp(row)
            sel = _brute_select(row.tolist(), c, K)
            for m in range(c):
                want = 0.0
                if m in sel:
                    for hq in range(h * G, (h + 1) * G):
                        for i in range(c * bs, (c + 1) * bs):
                            for j in range(m * bs, (m + 1) * bs):
                                p = np.exp(sigma * q[0, i, hq] @ k[0, j, h] + logg[m] - lse[0, hq, i])
                                want += p * dO[0, i, hq] @ (v[0, j, h] - o[0, i, hq])
                assert abs(out["dlogg"][0, h, c, m] - want) < 1e-11


def _nearest_bf16(x):
    """Brute force: the nearest of all finite bfloat16 values (ties to the even
    bit pattern), found by search in the sorted table of every pattern."""
    pats = np.arange(1 << 16, dtype=np.uint32)
    f32 = (pats << 16).view(np.float32)
    keep = np.isfinite(f32) & (pats != 0x8000)  # one zero is enough
    vals, pats = f32[keep].astype(np.float64), pats[keep]
    order = np.argsort(vals, kind="stable")
    vals, pats = vals[order], pats[order]
    x = np.asarray(x, dtype=np.float64)
    hi = np.clip(np.searchsorted(vals, x), 1, len(vals) - 1)
    lo = hi - 1
    dl, dh = x - vals[lo], vals[hi] - x
    pick_hi = (dh < dl) | ((dh == dl) & (pats[hi] % 2 == 0))
    return np.where(pick_hi, vals[hi], vals[lo])


def test_nearest_bf16_table_agrees_with_torch_on_float_values():
    rng = np.random.default_rng(21)
    x = (rng.standard_normal(4096) * np.exp(rng.uniform(-20, 20, 4096))).astype(np.float32)
    want = torch.tensor(x).to(torch.bfloat16).double().numpy()  # fp32 -> bf16 needs one rounding only
    np.testing.assert_array_equal(_nearest_bf16(x.astype(np.float64)), want)


def test_stored_bf16_output_in_eq5_and_D():
    """With o_store="bf16" the backward reads o as a bf16 tensor holds it: Eq. 5's
    d(log g)_m = sum_{i in B_m} p_i do.(v_i - o) with o rounded to the nearest bf16
    value, and dq / dk through dS_ij = p_ij (dO_i.v_j - dO_i.o_i) with the same o."""
    rng = np.random.default_rng(22)
    B, n, Hq, Hkv, d, bs, K = 1, 64, 4, 2, 8, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    sigma = 1 / np.sqrt(d)
    out = oracle.attn_bwd(q, k, v, dO, s, bs, K, sigma=sigma, o_store="bf16")
    exact = oracle.attn_bwd(q, k, v, dO, s, bs, K, sigma=sigma)
    np.testing.assert_array_equal(out["o"], exact["o"])  # o itself is reported exact
    o, lse = oracle.attn_fwd(q, k, v, s, bs, K, sigma=sigma)
    ot = _nearest_bf16(o)
    assert np.any(ot != o)
    G, Cq = Hq // Hkv, n // bs
    dq_want = np.zeros_like(q)
    for h in range(Hkv):
        for c in range(Cq):
            row = s[0, h, c, :c]
            logg = row - scipy.special.logsumexp(row) if c else row
            sel = _brute_select(row.tolist(), c, K) if c else []
            for hq in range(h * G, (h + 1) * G):
                for i in range(c * bs, (c + 1) * bs):
                    keys = [(j, logg[m]) for m in sel for j in range(m * bs, (m + 1) * bs)]
                    keys += [(j, 0.0) for j in range(c * bs, i + 1)]
                    for j, bias in keys:
                        p = np.exp(sigma * q[0, i, hq] @ k[0, j, h] + bias - lse[0, hq, i])
                        dq_want[0, i, hq] += sigma * p * (dO[0, i, hq] @ (v[0, j, h] - ot[0, i, hq])) * k[0, j, h]
            for m in range(c):
                want = 0.0
                if m in sel:
                    for hq in range(h * G, (h + 1) * G):
                        for i in range(c * bs, (c + 1) * bs):
                            for j in range(m * bs, (m + 1) * bs):
                                p = np.exp(sigma * q[0, i, hq] @ k[0, j, h] + logg[m] - lse[0, hq, i])
                                want += p * dO[0, i, hq] @ (v[0, j, h] - ot[0, i, hq])
                assert abs(out["dlogg"][0, h, c, m] - want) < 1e-11
    np.testing.assert_allclose(out["dq"], dq_want, atol=1e-11, rtol=0)
    assert np.abs(out["dq"] - exact["dq"]).max() > 1e-6  # the rounding is visible


def test_ds_rows_sum_to_zero_and_unselected_share_one_ratio():
    """ds is the softmax VJP, so each row sums to zero; in sparse scope an
    unselected block m gets ds_m = -g_m * sum(dlogg), one common sign and a
    ratio ds_m/g_m shared by all unselected blocks (shibing624 review, Fig. 4)."""
    rng = np.random.default_rng(10)
    B, n, Hq, Hkv, d, bs, K = 1, 96, 2, 1, 8, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    out = oracle.attn_bwd(q, k, v, dO, s, bs, K)
    ds = out["ds"][0, 0]
    Cq = n // bs
    for c in range(Cq):
        assert abs(ds[c].sum()) < 1e-12
        assert np.all(ds[c, c:] == 0.0)
        if c > K:
            row = s[0, 0, c, :c]
            g = np.exp(row - scipy.special.logsumexp(row))
            sel = set(_brute_select(row.tolist(), c, K))
            ratios = [ds[c, m] / g[m] for m in range(c) if m not in sel]
            np.testing.assert_allclose(ratios, ratios[0], rtol=1e-10, atol=0)


def test_sampled_masks_match_full_run():
    rng = np.random.default_rng(11)
    B, n, Hq, Hkv, d, bs, K = 1, 64, 2, 2, 8, 8, 2
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    full = oracle.attn_bwd(q, k, v, dO, s, bs, K)
    Cq = n // bs
    idx, _ = oracle.train_select(s, K)
    h, m = 1, 5
    qmask = np.zeros((B, Hkv, Cq), dtype=bool)
    kvmask = np.zeros((B, Hkv, Cq), dtype=bool)
    kvmask[0, h, m] = True
    qmask[0, h, m] = True
    for c in range(m + 1, Cq):
        if m in idx[0, h, c].tolist():
            qmask[0, h, c] = True
    part = oracle.attn_bwd(q, k, v, dO, s, bs, K, qmask=qmask, kvmask=kvmask)
    sl = slice(m * bs, (m + 1) * bs)
    np.testing.assert_array_equal(part["dk"][0, sl, h], full["dk"][0, sl, h])
    np.testing.assert_array_equal(part["dv"][0, sl, h], full["dv"][0, sl, h])
    np.testing.assert_array_equal(part["ds"][0, h, m], full["ds"][0, h, m])
    bad = qmask.copy()
    bad[0, h, m] = False
    with pytest.raises(RuntimeError):
        oracle.attn_bwd(q, k, v, dO, s, bs, K, qmask=bad, kvmask=kvmask)


def test_bf16_and_f32_inputs_are_widened_exactly():
    rng = np.random.default_rng(12)
    B, n, Hq, Hkv, d, bs, K = 1, 32, 2, 1, 8, 8, 2
    q, k, v, s, dO = (torch.tensor(x).to(torch.bfloat16) for x in _rand_train(rng, B, n, Hq, Hkv, d, bs))
    bits = [x.view(torch.int16).numpy().view(np.uint16) for x in (q, k, v)]
    wide = [x.double().numpy() for x in (q, k, v)]
    s32 = s.float().numpy()
    a = oracle.attn_fwd(*bits, s32, bs, K)
    b = oracle.attn_fwd(*wide, s32.astype(np.float64), bs, K)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


# --------------------------------------------------------------------------
# decode (jaehun.me review, walkthrough Step 6: Top-K without the gate)
# --------------------------------------------------------------------------

def _decode_torch(q, kc, vc, T, keys, sigma):
    G = q.shape[1] // kc.shape[1]
    B = q.shape[0]
    outs = []
    for b in range(B):
        heads = []
        for hq in range(q.shape[1]):
            h = hq // G
            kk = torch.tensor(kc[b, h, keys[b][h]])
            vv = torch.tensor(vc[b, h, keys[b][h]])
            p = torch.softmax(sigma * (kk @ torch.tensor(q[b, hq])), 0)
            heads.append(p @ vv)
        outs.append(torch.stack(heads))
    return torch.stack(outs).numpy()


def test_decode_sparse_and_dense():
    rng = np.random.default_rng(13)
    B, Hq, Hkv, d, bs, K, Tmax = 3, 4, 2, 16, 8, 3, 100
    q = rng.standard_normal((B, Hq, d))
    kc = rng.standard_normal((B, Hkv, Tmax, d)) * 0.5
    vc = rng.standard_normal((B, Hkv, Tmax, d))
    ctx = np.array([100, 41, 8], dtype=np.int32)  # current block of 4 tokens, 1 token, 8 tokens
    s = rng.standard_normal((B, Hkv, Tmax // bs)).astype(np.float32)
    sigma = 1 / np.sqrt(d)
    o, idx = oracle.decode(q, kc, vc, ctx, s, bs, K)
    keys = []
    for b in range(B):
        t = ctx[b] - 1
        Cb = t // bs
        kb = []
        for h in range(Hkv):
            sel = _brute_select(s[b, h, :Cb].tolist(), Cb, K)
            assert [x for x in idx[b, h].tolist() if x >= 0] == sel
            kb.append([j for m in sel for j in range(m * bs, (m + 1) * bs)] + list(range(Cb * bs, t + 1)))
        keys.append(kb)
    np.testing.assert_allclose(o, _decode_torch(q, kc, vc, ctx, keys, sigma), atol=1e-12, rtol=0)
    od, _ = oracle.decode(q, kc, vc, ctx, None, bs, K, dense=True)
    dense_keys = [[list(range(ctx[b])) for _ in range(Hkv)] for b in range(B)]
    np.testing.assert_allclose(od, _decode_torch(q, kc, vc, ctx, dense_keys, sigma), atol=1e-12, rtol=0)
    # a budget covering the whole history is dense attention
    ob, _ = oracle.decode(q, kc, vc, ctx, s, bs, Tmax)
    np.testing.assert_allclose(ob, od, atol=1e-12, rtol=0)


def test_bf16_half_ulp_allowance():
    """The comparison allowance is exactly the worst-case rounding of x to bf16."""
    import torch
    from parity import bf16_half_ulp

    x = (np.random.default_rng(14).standard_normal(100000)
         * np.exp2(np.random.default_rng(15).integers(-10, 10, 100000))).astype(np.float32)
    r = torch.tensor(x).to(torch.bfloat16).double().numpy()  # one rounding, fp32 -> bf16
    x = x.astype(np.float64)
    assert np.all(np.abs(r - x) <= bf16_half_ulp(x) * (1 + 1e-12))
    assert np.max(np.abs(r - x) / bf16_half_ulp(x)) > 0.99


@pytest.mark.parametrize("gate", ["sigmoid", "raw"])
def test_gate_activation_variants_vs_torch_dense_mask(gate):
    """The ablated gate activations (jaehun.me review, "Why the Four Design Choices
    Matter", gate activation): log g = log sigmoid(s) or the raw logit s inside the
    softmax; every output and gradient against torch autograd of the dense form."""
    rng = np.random.default_rng(31)
    B, n, Hq, Hkv, d, bs, K = 1, 64, 4, 2, 16, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    sigma = 1 / np.sqrt(d)
    for full in (False, True):
        out = oracle.attn_bwd(q, k, v, dO, s, bs, K, full_scope=full, gate=gate, sigma=sigma)
        T = [torch.tensor(x, requires_grad=True) for x in (q, k, v, s)]
        o_t, lse_t = _dense_masked_torch(*T, bs, K, sigma, full_scope=full, gate=gate)
        (o_t * torch.tensor(dO)).sum().backward()
        np.testing.assert_allclose(out["o"], o_t.detach().numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(out["lse"], lse_t.detach().numpy(), atol=1e-12, rtol=0)
        for name, t in zip(("dq", "dk", "dv", "ds"), T):
            np.testing.assert_allclose(out[name], t.grad.numpy(), atol=1e-11, rtol=0, err_msg=(gate, full, name))


@pytest.mark.parametrize("gate", ["sigmoid", "raw", "outer"])
def test_gate_activation_variants_finite_differences(gate):
    rng = np.random.default_rng(32)
    B, n, Hq, Hkv, d, bs, K = 1, 32, 2, 1, 4, 8, 2
    q, k, v, _, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    Cq = n // bs
    s = (rng.permutation(Cq * Cq).reshape(1, 1, Cq, Cq) * 0.05 + rng.uniform(0, 0.01, (1, 1, Cq, Cq))) - 0.3
    out = oracle.attn_bwd(q, k, v, dO, s, bs, K, gate=gate)
    eps = 1e-6

    def loss(q_, s_):
        o, _ = oracle.attn_fwd(q_, k, v, s_, bs, K, gate=gate)
        return float((o * dO).sum())

    for name, arr, pos in (("dq", q, 0), ("ds", s, 1)):
        for fi in rng.choice(arr.size, size=min(arr.size, 30), replace=False):
            ix = np.unravel_index(fi, arr.shape)
            ap, am = arr.copy(), arr.copy()
            ap[ix] += eps
            am[ix] -= eps
            args_p, args_m = [q, s], [q, s]
            args_p[pos], args_m[pos] = ap, am
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - out[name][ix]) <= 1e-6 * max(1.0, abs(out[name][ix])), (gate, name, ix)


def _dense_torch_outer_or_ste(q, k, v, s, bs, K, sigma, gate, full_scope=False):
    """Dense torch forms of the two other ablations (shibing624 review, Fig. 2(a)
    and 2(c); jaehun.me review, section 4.2.2 Eq. 5 and Eq. 7), g = softmax(s):
    "outer": o = (p * W) V with p the gate-free causal softmax over the selected
      history blocks and the current block, W[i, j] = g_{m(j)} (1 on the current
      block);
    "ste": every history block's keys enter the softmax numerator weighted by
      h_m = g_m + (hard_m - g_m).detach(), hard_m = 1 for the selected blocks and
      0 otherwise (1 on the current block): the value is hard Top-K attention and
      the gradient reaches g as if h were g."""
    B, n, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    Cq = n // bs
    outs, lses = [], []
    for b in range(B):
        oh, lh = [], []
        for hq in range(Hq):
            h = hq // G
            z = sigma * q[b, :, hq] @ k[b, :, h].T
            rows_o, rows_l = [], []
            for c in range(Cq):
                zc = z[c * bs:(c + 1) * bs]
                keep = torch.zeros((bs, n), dtype=torch.bool)
                weight = [torch.ones((), dtype=torch.float64)] * Cq
                if c > 0:
                    g = torch.softmax(s[b, h, c, :c], dim=0)
                    row = s[b, h, c, :c].detach().tolist()
                    sel = list(range(c)) if full_scope else _brute_select(row, c, K)
                    for m in range(c):
                        if gate == "outer":
                            if m in sel:
                                keep[:, m * bs:(m + 1) * bs] = True
                                weight[m] = g[m]
                        else:
                            keep[:, m * bs:(m + 1) * bs] = True
                            hard = 1.0 if m in sel else 0.0
                            weight[m] = g[m] + (hard - g[m]).detach()
                keep[:, c * bs:(c + 1) * bs] = torch.ones((bs, bs), dtype=torch.bool).tril()
                wcol = torch.stack([weight[m] for m in range(Cq) for _ in range(bs)])
                zm = zc.masked_fill(~keep, float("-inf"))
                mx = zm.max(dim=-1, keepdim=True).values.detach()
                e = torch.exp(zm - mx)
                if gate == "outer":
                    p = e / e.sum(-1, keepdim=True)
                    rows_o.append((p * wcol) @ v[b, :, h])
                    rows_l.append(torch.log(e.sum(-1)) + mx[:, 0])
                else:
                    eh = e * wcol
                    rows_o.append(eh @ v[b, :, h] / eh.sum(-1, keepdim=True))
                    rows_l.append(torch.log(eh.sum(-1)) + mx[:, 0])
            oh.append(torch.cat(rows_o, 0))
            lh.append(torch.cat(rows_l, 0))
        outs.append(torch.stack(oh, 1))
        lses.append(torch.stack(lh, 0))
    return torch.stack(outs, 0), torch.stack(lses, 0)


@pytest.mark.parametrize("gate", ["outer", "ste"])
def test_outer_and_ste_gates_vs_torch_dense(gate):
    rng = np.random.default_rng(34)
    B, n, Hq, Hkv, d, bs, K = 1, 64, 4, 2, 16, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    sigma = 1 / np.sqrt(d)
    for full in ((False, True) if gate == "outer" else (False,)):
        out = oracle.attn_bwd(q, k, v, dO, s, bs, K, full_scope=full, gate=gate, sigma=sigma)
        T = [torch.tensor(x, requires_grad=True) for x in (q, k, v, s)]
        o_t, lse_t = _dense_torch_outer_or_ste(*T, bs, K, sigma, gate, full_scope=full)
        (o_t * torch.tensor(dO)).sum().backward()
        np.testing.assert_allclose(out["o"], o_t.detach().numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(out["lse"], lse_t.detach().numpy(), atol=1e-12, rtol=0)
        for name, t in zip(("dq", "dk", "dv", "ds"), T):
            np.testing.assert_allclose(out[name], t.grad.numpy(), atol=1e-11, rtol=0, err_msg=(gate, full, name))


def test_ste_forward_is_hard_topk_and_outer_gradient_is_eq5():
    """STE: the forward equals plain block-sparse attention (gate off).  Outer:
    d(log g)_m = g_m dg_m with dg_m = sum_{i in B_m} p_i do.v_i (Eq. 5, outer),
    p the gate-free attention probabilities."""
    rng = np.random.default_rng(35)
    B, n, Hq, Hkv, d, bs, K = 1, 64, 4, 2, 8, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    sigma = 1 / np.sqrt(d)
    ste = oracle.attn_bwd(q, k, v, dO, s, bs, K, gate="ste", sigma=sigma)
    off = oracle.attn_bwd(q, k, v, dO, s, bs, K, gate="off", sigma=sigma)
    for name in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(ste[name], off[name], atol=1e-12, rtol=0, err_msg=name)
    out = oracle.attn_bwd(q, k, v, dO, s, bs, K, gate="outer", sigma=sigma)
    G, Cq = Hq // Hkv, n // bs
    for h in range(Hkv):
        for c in range(1, Cq):
            row = s[0, h, c, :c]
            g = np.exp(row - scipy.special.logsumexp(row))
            sel = _brute_select(row.tolist(), c, K)
            keys = [j for m in sel for j in range(m * bs, (m + 1) * bs)]
            for m in range(c):
                want = 0.0
                if m in sel:
                    for hq in range(h * G, (h + 1) * G):
                        for i in range(c * bs, (c + 1) * bs):
                            kk = keys + list(range(c * bs, i + 1))
                            z = np.array([sigma * q[0, i, hq] @ k[0, j, h] for j in kk])
                            p = np.exp(z - scipy.special.logsumexp(z))
                            for t, j in enumerate(kk):
                                if j // bs == m:
                                    want += p[t] * dO[0, i, hq] @ v[0, j, h]
                assert abs(out["dlogg"][0, h, c, m] - g[m] * want) < 1e-11, (h, c, m)


def test_ste_dropped_block_weights_are_unbounded():
    """Eq. 7: a dropped block's implied weights exp(z - LSE_S) are normalised by
    the selected set only.  Scaling the dropped block's keys along the queries'
    mean direction leaves the forward and the selected block's gradient as they
    are, while the dropped block's straight-through gradient grows without bound."""
    rng = np.random.default_rng(36)
    B, n, Hq, Hkv, d, bs, K = 1, 32, 1, 1, 8, 8, 1
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    s[0, 0, 3, :3] = [0.0, 5.0, 0.0]  # query block 3 selects block 1 only
    qm = q[0, 24:32, 0].mean(0)
    qm /= np.linalg.norm(qm)
    g0 = np.exp(s[0, 0, 3, 0] - scipy.special.logsumexp(s[0, 0, 3, :3]))
    grads, ref = [], None
    for alpha in (0.0, 8.0, 16.0, 32.0):
        ka = k.copy()
        ka[0, 0:8, 0] = qm * alpha  # block 0: dropped by query block 3
        out = oracle.attn_bwd(q, ka, v, dO, s, bs, K, gate="ste")
        if ref is None:
            ref = out
        np.testing.assert_allclose(out["o"][0, 24:32], ref["o"][0, 24:32], atol=1e-12, rtol=0)
        assert abs(out["dlogg"][0, 0, 3, 1] - ref["dlogg"][0, 0, 3, 1]) < 1e-12
        grads.append(abs(out["dlogg"][0, 0, 3, 0]) / g0)
    assert all(b > a for a, b in zip(grads, grads[1:])), grads
    assert grads[-1] > 100 * grads[0], grads


def test_gate_variants_reduce_to_known_cases():
    """The raw-logit gate fed log_softmax(s) is the softmax gate on s (forward); a
    sigmoid gate saturated at 1 (s = 60) is plain block-sparse attention."""
    rng = np.random.default_rng(33)
    B, n, Hq, Hkv, d, bs, K = 1, 64, 4, 2, 8, 8, 3
    q, k, v, s, dO = _rand_train(rng, B, n, Hq, Hkv, d, bs)
    Cq = n // bs
    logg = np.zeros_like(s)
    for c in range(1, Cq):
        row = s[..., c, :c]
        logg[..., c, :c] = row - np.log(np.exp(row - row.max(-1, keepdims=True)).sum(-1, keepdims=True)) \
            - row.max(-1, keepdims=True)
    o_soft, lse_soft = oracle.attn_fwd(q, k, v, s, bs, K, gate="softmax")
    o_raw, lse_raw = oracle.attn_fwd(q, k, v, logg, bs, K, gate="raw")
    np.testing.assert_allclose(o_raw, o_soft, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse_raw, lse_soft, atol=1e-12, rtol=0)
    # selection depends only on the order of s: keep it, saturate the sigmoid
    big = 60.0 + 1e-3 * (s - s.min())
    o_sig = oracle.attn_bwd(q, k, v, dO, big, bs, K, gate="sigmoid")
    o_off = oracle.attn_bwd(q, k, v, dO, big, bs, K, gate="off")
    for name in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(o_sig[name], o_off[name], atol=1e-12, rtol=0, err_msg=name)


def test_pooled_scores_are_block_means_of_the_dense_logits():
    """The pooled-key scorer: by bilinearity, sigma qbar_c . kbar_m is the mean of
    the dense logits sigma q_i . k_j over the tokens i of block c (all G heads of
    the group) and j of block m.  Computed here from a dense torch QK^T."""
    rng = np.random.default_rng(40)
    B, n, Hq, Hkv, d, bs = 2, 64, 4, 2, 16, 8
    q = rng.standard_normal((B, n, Hq, d))
    k = rng.standard_normal((B, n, Hkv, d))
    sigma = 0.3
    s = oracle.pool_scores(q, k, bs, sigma=sigma)
    G, Cq = Hq // Hkv, n // bs
    qt, kt = torch.tensor(q), torch.tensor(k)
    for b in range(B):
        for h in range(Hkv):
            z = torch.stack([sigma * qt[b, :, h * G + g] @ kt[b, :, h].T for g in range(G)])  # [G, n, n]
            zb = z.reshape(G, Cq, bs, Cq, bs).mean(dim=(0, 2, 4)).numpy()
            want = np.tril(zb, -1)
            np.testing.assert_allclose(s[b, h], want, atol=1e-12, rtol=0)


def test_pooled_scores_closed_form_constant_blocks():
    """Blocks whose tokens are all one vector: the summaries are those vectors."""
    B, n, Hq, Hkv, d, bs = 1, 32, 2, 1, 4, 8
    Cq = n // bs
    u = np.arange(Cq * d, dtype=np.float64).reshape(Cq, d) / 8.0  # dyadic: every mean and dot exact
    w = (np.arange(Cq * d, dtype=np.float64).reshape(Cq, d) % 3) - 1.0
    k = np.repeat(u, bs, axis=0)[None, :, None, :]
    q = np.repeat(np.repeat(w, bs, axis=0)[None, :, None, :], Hq, axis=2)
    s = oracle.pool_scores(q, k, bs, sigma=1.0)
    for c in range(Cq):
        for m in range(Cq):
            assert s[0, 0, c, m] == (float(w[c] @ u[m]) if m < c else 0.0)


def test_decode_pooled_scores_brute_force():
    """Decode: key summaries of the full blocks, then sigma (mean over the group's
    heads of q) . kbar_m, equal to the mean of the dense logits over the heads and
    the block's tokens; 0 beyond the history; bf16 summaries are the nearest bf16
    values of the exact means."""
    rng = np.random.default_rng(41)
    B, Hq, Hkv, d, bs, Tmax = 3, 4, 2, 8, 8, 64
    G = Hq // Hkv
    q = rng.standard_normal((B, Hq, d))
    kc = rng.standard_normal((B, Hkv, Tmax, d))
    ctx = np.array([1, 30, 64], dtype=np.int32)  # 0, 3 and 7 full history blocks
    nsum = Tmax // bs
    ksum = oracle.pool_keys(kc, bs, 0, nsum, nsum)
    s = oracle.decode_scores(q, ksum, ctx, bs, nsum, sigma=0.5)
    for b in range(B):
        Cb = (ctx[b] - 1) // bs
        for h in range(Hkv):
            for m in range(nsum):
                want = 0.0
                if m < Cb:
                    want = np.mean([0.5 * q[b, h * G + g] @ kc[b, h, j] for g in range(G)
                                    for j in range(m * bs, (m + 1) * bs)])
                assert abs(s[b, h, m] - want) < 1e-12, (b, h, m)
    part = oracle.pool_keys(kc, bs, 2, 5, nsum)
    assert np.all(part[:, :, :2] == 0) and np.all(part[:, :, 5:] == 0)
    np.testing.assert_array_equal(part[:, :, 2:5], ksum[:, :, 2:5])
    r = oracle.pool_keys(kc, bs, 0, nsum, nsum, round_bf16=True)
    np.testing.assert_array_equal(r, _nearest_bf16(ksum))


@pytest.mark.parametrize("gate", ["softmax", "outer", "ste"])
def test_softmax_family_ds_rows_sum_to_zero_on_random_shapes(gate):
    """Every gate built on g = softmax(s) passes its gradient to s through the
    softmax's vector-Jacobian product, so each ds row sums to zero, whatever the
    shape, budget or scope."""
    rng = np.random.default_rng(50)
    for _ in range(4):
        bs = int(rng.choice([4, 8]))
        Cq = int(rng.integers(2, 7))
        Hkv = int(rng.integers(1, 3))
        G = int(rng.choice([1, 2, 3]))
        d = int(rng.choice([4, 8]))
        K = int(rng.integers(0, Cq + 1))
        full = bool(rng.integers(0, 2)) and gate != "ste"
        q, k, v, s, dO = _rand_train(rng, 1, Cq * bs, Hkv * G, Hkv, d, bs)
        out = oracle.attn_bwd(q, k, v, dO, s, bs, K, full_scope=full, gate=gate)
        for h in range(Hkv):
            for c in range(Cq):
                assert abs(out["ds"][0, h, c, :c].sum()) < 1e-12, (gate, bs, Cq, K, full, h, c)
                assert np.all(out["ds"][0, h, c, c:] == 0)
