"""Small problems of every kernel family run through the library named by
SAS_LIBRARY (the debug-bounds build), each checked against the oracle at the
parity tolerances and followed by a read of the device status word, which must
still hold 0: no index check failed.  Run by tests/test_gpu_debug_bounds.py in
a process of its own (the binding loads one library per process)."""
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
from parity import BF16_TOL, F32_TOL, bits, compare, host, run_train  # noqa: E402
from trainable_block_sparse_sas_b200 import api  # noqa: E402


def seeded(shape, std, dtype, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype).to("cuda")


def word_is_clear(word, what):
    torch.cuda.synchronize()
    raw = int(word.item())
    assert raw == 0, f"{what}: status word {raw:#x} (code {raw & 0xff}, source line {raw >> 8})"


def train_case(word, B, n, Hq, Hkv, d, bs, K, full, dtype, gate="softmax"):
    Cq = n // bs
    std = 1.0 if dtype == torch.bfloat16 else 0.3
    inp = {"q": seeded((B, n, Hq, d), std, dtype, 1), "k": seeded((B, n, Hkv, d), std, dtype, 2),
           "v": seeded((B, n, Hkv, d), 1.0, dtype, 3), "s": seeded((B, Hkv, Cq, Cq), 2.0, torch.float32, 4),
           "dO": seeded((B, n, Hq, d), 1.0, dtype, 5)}
    api._default_words[torch.cuda.current_device()] = word
    got = run_train(api, inp, bs, K, full, gate=gate)
    word_is_clear(word, f"train {Hq}/{Hkv} d{d} b{bs} K{K} full={full} {dtype} {gate}")
    want = oracle.attn_bwd(*(bits(inp[x]) for x in ("q", "k", "v", "dO", "s")), bs, K, full_scope=full, gate=gate)
    tol = BF16_TOL if dtype == torch.bfloat16 else F32_TOL
    b16 = dtype == torch.bfloat16
    for key in ("o", "dq", "dk", "dv"):
        compare(key, host(got[key]), want[key], **tol, bf16_out=b16)
    compare("ds", host(got["ds"]), want["ds"], **tol)


def decode_case(word, dtype, d, bs, mode):
    B, Hq, Hkv, K, Tmax = 3, 8, 2, 4, 64 * 12 + 5
    ctx = torch.tensor([Tmax, 65, 1], dtype=torch.int32, device="cuda")
    q = seeded((B, Hq, d), 1.0, dtype, 11)
    kc = seeded((B, Hkv, Tmax, d), 1.0, dtype, 12)
    vc = seeded((B, Hkv, Tmax, d), 1.0, dtype, 13)
    s = seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 14)
    desc = api.decode_desc(q, kc, bs, K)
    o = torch.empty_like(q)
    idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
    if mode == "fused":
        api.sas_sparse_decode_select(desc, q, kc, vc, ctx, s, o, idx, status=word)
    else:
        api.sas_topk_select(s.view(B, Hkv, 1, -1), 1, s.shape[-1], K, idx=idx, ctx_len=ctx, block_size=bs)
        use = None if mode == "dense" else idx
        if mode == "noalloc":
            api.sas_sparse_decode_noalloc(desc, q, kc, vc, ctx, use, o, status=word)
        else:
            ws = api.workspace(api.sas_sparse_decode_workspace_size(desc), q.device)
            api.sas_sparse_decode(desc, q, kc, vc, ctx, use, o, ws, status=word)
    word_is_clear(word, f"decode {dtype} d{d} b{bs} {mode}")
    G = Hq // Hkv
    tol = BF16_TOL if dtype == torch.bfloat16 else F32_TOL
    for b in range(B):
        for h in range(Hkv):
            T = int(ctx[b])
            ro, _ = oracle.decode(bits(q[b:b + 1, h * G:(h + 1) * G]), bits(kc[b:b + 1, h:h + 1, :T]),
                                  bits(vc[b:b + 1, h:h + 1, :T]), np.array([T], np.int32), bits(s[b:b + 1, h:h + 1]),
                                  bs, K, dense=mode == "dense")
            compare(f"decode o[{b},{h}] {mode}", host(o[b, h * G:(h + 1) * G]), ro[0], **tol,
                    bf16_out=dtype == torch.bfloat16)


def main():
    assert os.environ.get("SAS_LIBRARY", "").endswith("libsas_debug.so"), "run with SAS_LIBRARY=.../libsas_debug.so"
    assert api._LIB_PATH == os.environ["SAS_LIBRARY"]
    word = api.status_word()
    # tensor-core training kernels (G 2, 4 and 8; sparse and full scope; the gates)
    train_case(word, 1, 512, 4, 1, 128, 64, 3, False, torch.bfloat16)
    train_case(word, 1, 512, 8, 1, 128, 64, 3, False, torch.bfloat16)
    train_case(word, 1, 512, 4, 2, 128, 64, 0, True, torch.bfloat16)
    for gate in ("outer", "ste", "sigmoid"):
        train_case(word, 1, 512, 8, 2, 128, 64, 3, False, torch.bfloat16, gate)
    # SIMT training kernels (fp32; bf16 shapes outside the tensor-core ones)
    train_case(word, 1, 256, 4, 2, 128, 32, 3, False, torch.float32)
    train_case(word, 1, 384, 5, 1, 64, 32, 4, False, torch.bfloat16, "raw")
    # decode: the cluster kernel (fused selection, given blocks, dense), the split-K
    # kernels (bf16 d 64, fp32) and the allocation-free entry point on both paths
    for mode in ("fused", "sparse", "dense", "noalloc"):
        decode_case(word, torch.bfloat16, 128, 64, mode)
    for mode in ("sparse", "dense", "noalloc"):
        decode_case(word, torch.bfloat16, 64, 64, mode)
        decode_case(word, torch.float32, 128, 64, mode)
    api.sas_get_device_status(word)
    print("debug-bounds cases ok")


if __name__ == "__main__":
    main()
