"""The allocation-free decode entry point, for callers that cannot allocate
device memory (a plugin whose host program owns all device memory, a serving
loop that may not call cudaMalloc between steps): on two calls in a row it gives
the results of the regular entry point, sas_sparse_decode, and of the oracle,
on both of its paths -- the tensor-core decode (no scratch) and the split-K
kernels whose partials live in the library's fixed scratch array.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.  It passes alone in a fresh process and after
the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity import BF16_TOL, F32_TOL, bits, compare, host

pytestmark = pytest.mark.gpu


def _seeded(shape, std, dtype, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype).to("cuda")


# (dtype, head_dim, block): the first runs the tensor-core decode, the others the
# split-K kernels with the built-in scratch
PATHS = [(torch.bfloat16, 128, 64), (torch.bfloat16, 64, 64), (torch.bfloat16, 128, 32), (torch.float32, 128, 64)]


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("dtype,d,bs", PATHS)
def test_noalloc_decode_matches_workspace_decode_and_oracle(cuda_ok, dtype, d, bs, dense):
    from trainable_block_sparse_sas_b200 import api

    B, Hq, Hkv, K, Tmax = 6, 32, 8, 16, 9000
    ctx = torch.tensor([9000, 1, 65, 1025, 4097, 8193], dtype=torch.int32, device="cuda")
    q = _seeded((B, Hq, d), 1.0, dtype, 51)
    kc = _seeded((B, Hkv, Tmax, d), 1.0, dtype, 52)
    vc = _seeded((B, Hkv, Tmax, d), 1.0, dtype, 53)
    s = _seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 54)
    desc = api.decode_desc(q, kc, bs, K)
    idx = None
    if not dense:
        idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
        api.sas_topk_select(s.view(B, Hkv, 1, -1), 1, s.shape[-1], K, idx=idx, ctx_len=ctx, block_size=bs)
    ref = torch.empty_like(q)
    ws = api.workspace(api.sas_sparse_decode_workspace_size(desc), q.device)
    api.sas_sparse_decode(desc, q, kc, vc, ctx, idx, ref, ws)
    tol = BF16_TOL if dtype == torch.bfloat16 else F32_TOL
    b16 = dtype == torch.bfloat16
    G = Hq // Hkv
    rows = [(0, 0), (3, 5), (5, 7), (1, 2)]
    want = {}
    for b, h in rows:
        T = int(ctx[b])
        o_ref, _ = oracle.decode(bits(q[b:b + 1, h * G:(h + 1) * G]), bits(kc[b:b + 1, h:h + 1, :T]),
                                 bits(vc[b:b + 1, h:h + 1, :T]), np.array([T], np.int32), bits(s[b:b + 1, h:h + 1]),
                                 bs, K, dense=dense)
        want[(b, h)] = o_ref[0]
    for call in range(2):  # two calls in a row share the built-in scratch
        out = torch.full_like(q, float("nan"))
        api.sas_sparse_decode_noalloc(desc, q, kc, vc, ctx, idx, out)
        torch.cuda.synchronize()
        compare(f"noalloc call {call} vs sas_sparse_decode", host(out), host(ref), **tol, bf16_out=b16)
        for (b, h), o_ref in want.items():
            compare(f"noalloc call {call} o[{b},{h}] vs oracle", host(out[b, h * G:(h + 1) * G]), o_ref, **tol,
                    bf16_out=b16)
    api.sas_get_device_status()


def test_noalloc_rejects_problems_beyond_the_scratch(cuda_ok):
    from trainable_block_sparse_sas_b200 import api

    # fp32 dense over a 1M-token cache runs the split-K kernels: partials > 4 MiB
    d = api.DecodeDesc(64, 64, 8, 128, 64, 0, 1 << 20, 0, 0.0)
    fake = ctypes.c_void_p(0x1000)  # rejected before any launch, never dereferenced
    st = api.lib.sas_sparse_decode_noalloc(ctypes.byref(d), fake, fake, fake, fake, None, fake, fake, None)
    assert st == api.SAS_ERR_WORKSPACE_TOO_SMALL
