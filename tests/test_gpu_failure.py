"""The failure path of the bounded device-side waits, on the GPU and without a
fault.  The self-test runs the tensor-core kernels' own wait routines: a wait on
a barrier that nothing sets gives up after its limit and sets the abort flag, a
second role leaves on that flag, the in-flight MMA drains and the tensor memory
is freed; the host reads SAS_ERR_DEVICE_TIMEOUT from the caller's status word
once, and the context stays usable.  Status words are per caller: a timeout on
one stream's word is not seen through another's."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _select_still_works(api):
    s = torch.tensor([[[[0.8, 1.5, 0.3, 0.6, 0.0]]]], device="cuda")
    idx = torch.empty((1, 1, 1, 2), dtype=torch.int32, device="cuda")
    api.sas_topk_select(s, 1, 5, 2, idx=idx, ctx_len=torch.tensor([5 * 64 + 1], dtype=torch.int32, device="cuda"),
                        block_size=64)
    torch.cuda.synchronize()
    assert idx.cpu().numpy().ravel().tolist() == [0, 1]


def test_bounded_wait_runs_the_kernels_failure_path(cuda_ok):
    from trainable_block_sparse_sas_b200 import api

    word = api.status_word()
    trace = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    api.sas_selftest_bounded_wait(50, status=word, trace=trace)
    torch.cuda.synchronize()
    # gave up on its limit, the other role left on the abort flag, MMAs drained, TMEM freed
    assert trace.cpu().tolist() == [1, 1, 1, 1]
    with pytest.raises(api.SasError) as e:
        api.sas_get_device_status(word)
    assert e.value.status == api.SAS_ERR_DEVICE_TIMEOUT
    api.sas_get_device_status(word)  # reported once, then cleared
    _select_still_works(api)


def test_status_word_is_per_caller(cuda_ok):
    """Stream A times out a wait into its word while stream B runs a tensor-core
    forward with its own word: only A's caller sees the timeout."""
    from trainable_block_sparse_sas_b200 import api

    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    wa, wb = api.status_word(), api.status_word()
    g = torch.Generator(device="cpu")
    g.manual_seed(7)
    B, n, Hq, Hkv, d, bs, K = 1, 512, 4, 1, 128, 64, 3
    q = torch.randn((B, n, Hq, d), generator=g).to(torch.bfloat16).cuda()
    k = torch.randn((B, n, Hkv, d), generator=g).to(torch.bfloat16).cuda()
    v = torch.randn((B, n, Hkv, d), generator=g).to(torch.bfloat16).cuda()
    s = torch.randn((B, Hkv, n // bs, n // bs), generator=g).cuda()
    desc = api.attn_desc(q, k, bs, K)
    idx, lse_s = api.select_train(s, bs, K)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, n), device="cuda")
    torch.cuda.synchronize()
    with torch.cuda.stream(sa):
        api.sas_selftest_bounded_wait(100, status=wa, stream=sa)
    with torch.cuda.stream(sb):
        api.sas_gated_attn_fwd(desc, q, k, v, s, lse_s, idx, o, lse, stream=sb, status=wb)
    api.sas_get_device_status(wb, stream=sb)  # B's caller: no timeout
    with pytest.raises(api.SasError) as e:
        api.sas_get_device_status(wa, stream=sa)
    assert e.value.status == api.SAS_ERR_DEVICE_TIMEOUT
    assert np.isfinite(o.float().cpu().numpy()).all()
    _select_still_works(api)


def test_selftest_rejects_bad_limits(cuda_ok):
    from trainable_block_sparse_sas_b200 import api

    for bad in (0, -5, 20000):
        with pytest.raises(api.SasError) as e:
            api.sas_selftest_bounded_wait(bad, status=api.status_word())
        assert e.value.status == api.SAS_ERR_INVALID_VALUE
