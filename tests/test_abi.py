"""Host-only checks of the C ABI: the library builds, loads and exports every
symbol include/sas.h declares; arguments are rejected with the documented
status before any device work; the CUDA library and the oracle are independent.
No test here launches a kernel."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sas.h")
PKG = os.path.join(ROOT, "trainable_block_sparse_sas_b200")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:sas_status|size_t|const char\s*\*|int32_t|uint64_t)\s+(sas_\w+)\s*\(", text,
                                 flags=re.M)))


@pytest.fixture(scope="module")
def api():
    from trainable_block_sparse_sas_b200 import build

    build.build()
    from trainable_block_sparse_sas_b200 import api as a

    return a


def test_header_declares_the_hot_path_entry_points():
    names = _declared()
    for want in ("sas_topk_select", "sas_gated_attn_fwd", "sas_gated_attn_bwd", "sas_sparse_decode"):
        assert want in names


def test_library_exports_every_declared_symbol(api):
    lib = ctypes.CDLL(api._LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", api._LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (sas_\w+)$", out, flags=re.M))
    assert set(_declared()) <= exported


def test_status_strings(api):
    for st in range(7):
        assert api.lib.sas_status_string(st)
    assert api.lib.sas_version() >= 100


def _desc(api, **kw):
    base = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, seq_len=256, block_size=64, top_k=2, scope=0,
                dtype=1, softmax_scale=0.0, gate=0)
    base.update(kw)
    return api.AttnDesc(**base)


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every case below fails validation first


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), 1), (dict(n_q_heads=3), 1), (dict(seq_len=100), 1), (dict(top_k=-1), 1),
    (dict(scope=7), 1), (dict(dtype=5), 1), (dict(gate=5), 1), (dict(gate=-1), 1), (dict(head_dim=96), 2), (dict(block_size=48, seq_len=96), 2), (dict(block_size=128), 2),
])
def test_fwd_rejects_bad_descriptors(api, kw, status):
    d = _desc(api, **kw)
    st = api.lib.sas_gated_attn_fwd(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None)
    assert st == status


def test_fwd_rejects_null_pointers(api):
    """Every pointer of the forward is required (idx only in sparse scope with
    top_k > 0), the device status word included."""
    d = _desc(api)
    args = [FAKE] * 9
    for i in range(9):
        a = list(args)
        a[i] = None
        assert api.lib.sas_gated_attn_fwd(ctypes.byref(d), *a, None) == 1, i


def test_bwd_checks_workspace(api):
    d = _desc(api)
    need = api.lib.sas_gated_attn_bwd_workspace_size(ctypes.byref(d))
    assert need > 0 and need % 256 == 0
    args = [FAKE] * 13
    st = api.lib.sas_gated_attn_bwd(ctypes.byref(d), *args, FAKE, need - 1, FAKE, None)
    assert st == 3
    st = api.lib.sas_gated_attn_bwd(ctypes.byref(d), *args, FAKE, need, None, None)  # no status word
    assert st == 1
    assert api.lib.sas_gated_attn_bwd_workspace_size(None) == 0
    bad = _desc(api, seq_len=100)
    assert api.lib.sas_gated_attn_bwd_workspace_size(ctypes.byref(bad)) == 0


def test_decode_checks(api):
    d = api.DecodeDesc(2, 8, 2, 128, 64, 4, 1000, 1, 0.0)
    need = api.lib.sas_sparse_decode_workspace_size(ctypes.byref(d))
    assert need > 0 and need % 256 == 0
    dec = api.lib.sas_sparse_decode
    assert dec(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, FAKE, None) == 3
    assert dec(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, FAKE, None) == 1
    assert dec(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, None, None) == 1  # no status word
    bad = api.DecodeDesc(2, 8, 3, 128, 64, 4, 1000, 1, 0.0)
    assert dec(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, FAKE, None) == 1
    uns = api.DecodeDesc(2, 8, 2, 96, 64, 4, 1000, 1, 0.0)
    assert dec(ctypes.byref(uns), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, FAKE, None) == 2
    sel = api.lib.sas_sparse_decode_select
    assert sel(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 16, FAKE, None, None, None) == 1  # no status word
    na = api.lib.sas_sparse_decode_noalloc
    assert na(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None) == 1  # no status word
    assert na(ctypes.byref(uns), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None) == 2


def test_select_checks(api):
    L = api.lib
    assert L.sas_topk_select(None, 1, 1, 4, 4, None, 0, 2, FAKE, FAKE, None) == 1
    assert L.sas_topk_select(FAKE, 1, 1, 4, 4, None, 0, -1, FAKE, FAKE, None) == 1
    assert L.sas_topk_select(FAKE, 1, 1, 4, 4, None, 0, 2, None, None, None) == 1
    assert L.sas_topk_select(FAKE, 1, 1, 2, 4, FAKE, 64, 2, FAKE, None, None) == 1  # decode rows need n_rows 1
    assert L.sas_topk_select(FAKE, 1, 1, 1, 4, FAKE, 0, 2, FAKE, None, None) == 1   # decode rows need block_size


def test_attn_path_names_the_kernels_a_shape_runs(api):
    """The tensor-core path takes bf16, d 128, block 64 with 2, 4 or 8 query heads
    per kv head; fp32 and the other shapes run the SIMT kernels."""
    L = api.lib
    f, b = ctypes.c_int32(-1), ctypes.c_int32(-1)

    def path(**kw):
        assert L.sas_attn_path(ctypes.byref(_desc(api, **kw)), ctypes.byref(f), ctypes.byref(b)) == 0
        return f.value, b.value

    for G in (2, 4, 8):
        assert path(n_q_heads=2 * G, n_kv_heads=2) == (1, 1), G
        assert path(n_q_heads=2 * G, n_kv_heads=2, scope=1, top_k=0) == (1, 1), G
    assert path(n_q_heads=2, n_kv_heads=2) == (0, 0)      # one query head per kv head
    assert path(n_q_heads=10, n_kv_heads=2) == (0, 0)     # 5
    assert path(dtype=0) == (0, 0)                        # fp32
    assert path(head_dim=64) == (0, 0)
    assert path(block_size=32, seq_len=256) == (0, 0)
    assert L.sas_attn_path(ctypes.byref(_desc(api, head_dim=96)), None, None) == 2
    assert L.sas_attn_path(ctypes.byref(_desc(api, batch=0)), None, None) == 1
    assert api.sas_attn_path(_desc(api)) == ("tensor_core", "tensor_core")


def test_status_word_and_selftest_checks(api):
    """The status reader and the failure self-test refuse a missing word or an
    out-of-range limit before touching the device."""
    L = api.lib
    assert L.sas_get_device_status(None, None) == 1
    assert L.sas_selftest_bounded_wait(50, None, None, None) == 1
    for bad in (0, -5, 20000):
        assert L.sas_selftest_bounded_wait(bad, FAKE, None, None) == 1


def test_floor_and_trace_checks(api):
    """The launch-floor and phase-trace diagnostics reject bad arguments before
    touching the device."""
    L = api.lib
    assert L.sas_sparse_decode_launch_floor(None, FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, None) == 1
    assert L.sas_phase_trace_read(None, 4) == 1
    for bad in (0, -1, 1025):
        assert L.sas_phase_trace_read(FAKE, bad) == 1


def test_cuda_library_and_oracle_share_nothing(api):
    """The product path never imports, loads or links the oracle, and the oracle
    never includes the library's headers or sources."""
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
                assert "sas_oracle" not in text and "liboracle" not in text, f
    oracle_src = open(os.path.join(ROOT, "oracle", "sas_oracle.c")).read()
    assert "#include \"" not in oracle_src and "sas.h" not in oracle_src
    deps = subprocess.run(["ldd", api._LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in deps


def test_paged_decode_checks(api):
    L = api.lib
    d = api.DecodeDesc(2, 8, 2, 128, 64, 4, 1000, 1, 0.0)  # max_ctx 1000

    def call(desc, pps=16, npages=64, kp=FAKE, s=FAKE, s_cols=16, table=FAKE):
        return L.sas_sparse_decode_paged(ctypes.byref(desc), FAKE, kp, FAKE, table, pps, npages, FAKE, None, s,
                                         s_cols, FAKE, None, FAKE, None)

    assert call(d, table=None) == 1
    assert call(d, pps=0) == 1
    assert call(d, npages=0) == 1
    assert call(d, pps=15) == 1                       # 15 pages of 64 < max_ctx 1000
    assert call(d, s_cols=0) == 1
    assert call(d, kp=ctypes.c_void_p(0x1008)) == 1   # pool not 16-byte aligned
    assert call(api.DecodeDesc(2, 8, 2, 128, 64, 4, 1000, 0, 0.0)) == 2         # fp32
    assert call(api.DecodeDesc(2, 8, 2, 128, 32, 4, 1000, 1, 0.0), pps=32) == 2  # block 32


def test_scorer_checks(api):
    """Argument checks of the pooled-key scorer entry points (nothing is launched)."""
    L = api.lib
    d = _desc(api)
    need = L.sas_pooled_scores_workspace_size(ctypes.byref(d))
    assert need > 0 and need % 256 == 0
    assert L.sas_pooled_scores(ctypes.byref(d), None, FAKE, FAKE, FAKE, need, None) == 1
    assert L.sas_pooled_scores(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, need - 1, None) == 3
    assert L.sas_pooled_scores(ctypes.byref(_desc(api, seq_len=100)), FAKE, FAKE, FAKE, FAKE, need, None) == 1
    wide = _desc(api, n_q_heads=16, n_kv_heads=1, dtype=0)  # fp32, G d = 2048 elements: 8 KB per row
    assert L.sas_pooled_scores(ctypes.byref(wide), FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 2
    assert L.sas_pooled_scores(ctypes.byref(_desc(api, head_dim=20)), FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 2
    dd = api.DecodeDesc(2, 8, 2, 128, 64, 4, 1000, 1, 0.0)  # max_ctx 1000: 15 full blocks
    assert L.sas_pool_key_blocks(ctypes.byref(dd), None, 0, 4, FAKE, 16, None) == 1
    assert L.sas_pool_key_blocks(ctypes.byref(dd), FAKE, 3, 2, FAKE, 16, None) == 1   # empty-negative range
    assert L.sas_pool_key_blocks(ctypes.byref(dd), FAKE, 0, 17, FAKE, 16, None) == 1  # past nsum
    assert L.sas_pool_key_blocks(ctypes.byref(dd), FAKE, 0, 16, FAKE, 16, None) == 1  # past max_ctx
    assert L.sas_decode_scores(ctypes.byref(dd), FAKE, FAKE, 0, FAKE, FAKE, 16, None) == 1
    assert L.sas_decode_scores(ctypes.byref(dd), FAKE, FAKE, 16, None, FAKE, 16, None) == 1
    d96 = api.DecodeDesc(2, 8, 2, 96, 64, 4, 1000, 1, 0.0)
    assert L.sas_decode_scores(ctypes.byref(d96), FAKE, FAKE, 16, FAKE, FAKE, 16, None) == 2
    P = L.sas_pool_key_blocks_paged
    assert P(ctypes.byref(dd), None, FAKE, 16, 40, 0, 4, FAKE, 16, None) == 1
    assert P(ctypes.byref(dd), FAKE, FAKE, 0, 40, 0, 4, FAKE, 16, None) == 1    # pages_per_seq
    assert P(ctypes.byref(dd), FAKE, FAKE, 16, 40, 0, 17, FAKE, 20, None) == 1  # past pages_per_seq
    assert P(ctypes.byref(dd), FAKE, FAKE, 16, 40, 0, 17, FAKE, 16, None) == 1  # past nsum
    assert P(ctypes.byref(dd), ctypes.c_void_p(0x1008), FAKE, 16, 40, 0, 4, FAKE, 16, None) == 1  # misaligned


def test_binding_fails_loudly_without_the_library(tmp_path):
    """A copy of the package without libsas.so cannot be imported: the binding
    raises instead of falling back to anything."""
    import shutil
    import sys

    src = os.path.join(ROOT, "trainable_block_sparse_sas_b200")
    dst = tmp_path / "trainable_block_sparse_sas_b200"
    dst.mkdir()
    for f in ("__init__.py", "api.py", "synthetic.py"):
        shutil.copy(os.path.join(src, f), dst / f)
    r = subprocess.run([sys.executable, "-c", "import trainable_block_sparse_sas_b200.api"], cwd=tmp_path,
                       capture_output=True, text=True, env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode != 0
    assert "libsas.so not built" in r.stderr


def test_binding_refuses_short_mistyped_strided_or_host_buffers(api):
    """The binding checks each buffer against the descriptor before the C call
    (the ABI sees pointers only, so a short buffer would be accessed out of
    bounds on the GPU): size, then dtype, then layout, then device."""
    import torch

    q = torch.zeros((1, 256, 4, 128), dtype=torch.bfloat16)
    k = torch.zeros((1, 256, 2, 128), dtype=torch.bfloat16)
    desc = api.attn_desc(q, k, 64, 2)
    s, lse_s = torch.zeros((1, 2, 4, 4)), torch.zeros((1, 2, 4))
    idx = torch.zeros((1, 2, 4, 2), dtype=torch.int32)
    o, lse = torch.zeros_like(q), torch.zeros((1, 4, 256))
    with pytest.raises(ValueError, match="q holds"):
        api.sas_gated_attn_fwd(desc, q[:, :128], k, k, s, lse_s, idx, o, lse)
    with pytest.raises(ValueError, match="idx holds"):
        api.sas_gated_attn_fwd(desc, q, k, k, s, lse_s, idx[..., :1], o, lse)
    with pytest.raises(TypeError, match="k is torch.float32"):
        api.sas_gated_attn_fwd(desc, q, k.float(), k, s, lse_s, idx, o, lse)
    with pytest.raises(ValueError, match="contiguous"):
        api.sas_gated_attn_fwd(desc, q.transpose(2, 3), k, k, s, lse_s, idx, o, lse)
    with pytest.raises(ValueError, match="CUDA device"):
        api.sas_gated_attn_fwd(desc, q, k, k, s, lse_s, idx, o, lse)
    ds = torch.zeros_like(s)
    with pytest.raises(ValueError, match="ds holds"):
        api.sas_gated_attn_bwd(desc, q, k, k, o, lse, q, s, lse_s, idx, q, k, k, ds[:, :1], None)
    qd = torch.zeros((2, 8, 128), dtype=torch.bfloat16)
    kc = torch.zeros((2, 2, 1000, 128), dtype=torch.bfloat16)
    dd = api.decode_desc(qd, kc, 64, 4)
    ctx = torch.zeros((2,), dtype=torch.int32)
    with pytest.raises(ValueError, match="v_cache holds"):
        api.sas_sparse_decode(dd, qd, kc, kc[:1], ctx, None, torch.zeros_like(qd), None)
    with pytest.raises(ValueError, match="idx holds"):
        api.sas_sparse_decode(dd, qd, kc, kc, ctx, torch.zeros((2, 2, 3), dtype=torch.int32), torch.zeros_like(qd),
                              None)
    with pytest.raises(TypeError, match="ctx_len is torch.int64"):
        api.sas_sparse_decode_select(dd, qd, kc, kc, ctx.long(), torch.zeros((2, 2, 15)), torch.zeros_like(qd))
