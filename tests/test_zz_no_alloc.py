"""The allocation-free decode entry point (for callers that cannot allocate
device memory) gives the results of the regular entry point.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.  It passes alone in a fresh process and after
the other tests."""
import ctypes

import numpy as np
import pytest
import torch

from parity import BF16_TOL, compare, host

pytestmark = pytest.mark.gpu


def _seeded(shape, std, dtype, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype).to("cuda")


@pytest.mark.parametrize("dense", [False, True])
def test_noalloc_decode_matches_workspace_decode(cuda_ok, dense):
    from trainable_block_sparse_sas_b200 import api

    B, Hq, Hkv, d, bs, K, Tmax = 6, 32, 8, 128, 64, 16, 9000
    ctx = torch.tensor([9000, 1, 65, 1025, 4097, 8193], dtype=torch.int32, device="cuda")
    q = _seeded((B, Hq, d), 1.0, torch.bfloat16, 51)
    kc = _seeded((B, Hkv, Tmax, d), 1.0, torch.bfloat16, 52)
    vc = _seeded((B, Hkv, Tmax, d), 1.0, torch.bfloat16, 53)
    s = _seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 54)
    desc = api.decode_desc(q, kc, bs, K)
    idx = None
    if not dense:
        idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
        api.sas_topk_select(s.view(B, Hkv, 1, -1), 1, s.shape[-1], K, idx=idx, ctx_len=ctx, block_size=bs)
    ref = torch.empty_like(q)
    ws = api.workspace(api.sas_sparse_decode_workspace_size(desc), q.device)
    api.sas_sparse_decode(desc, q, kc, vc, ctx, idx, ref, ws)
    for call in range(2):  # two calls in a row share the built-in scratch
        out = torch.full_like(q, float("nan"))
        api.sas_sparse_decode_noalloc(desc, q, kc, vc, ctx, idx, out)
        torch.cuda.synchronize()
        compare(f"noalloc call {call}", host(out), host(ref), **BF16_TOL, bf16_out=True)


def test_noalloc_rejects_problems_beyond_the_scratch(cuda_ok):
    from trainable_block_sparse_sas_b200 import api

    d = api.DecodeDesc(64, 64, 8, 128, 64, 0, 1 << 20, 1, 0.0)  # dense over a 1M-token cache: partials > 4 MiB
    fake = ctypes.c_void_p(0x1000)  # rejected before any launch, never dereferenced
    st = api.lib.sas_sparse_decode_noalloc(ctypes.byref(d), fake, fake, fake, fake, None, fake, None)
    assert st == api.SAS_ERR_WORKSPACE_TOO_SMALL
