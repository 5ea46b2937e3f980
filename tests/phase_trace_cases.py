"""The decode kernel's phase trace (a library built with --phase-trace, named by
SAS_LIBRARY): a fused decode step through the traced kernel matches the oracle,
and its trace rows are consistent -- one row per CTA of the grid, every CTA's
stamps in phase order, the selection stamps between the cluster barrier and the
end of the selection, at least K candidates, and the blocks streamed by a row's
CTAs adding up to its attended list.  Also: the launch-floor kernel runs on the
same arguments.  Run by tests/test_gpu_phase_trace.py in a process of its own."""
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
from parity import BF16_TOL, bits, compare, host  # noqa: E402
from trainable_block_sparse_sas_b200 import api  # noqa: E402

ORDER = (0, 1, 2, 6, 7, 8, 9, 10, 11)  # entry, ctx_len, barrier, selected, first block, stream end, partial,
# slices received, exit
SELECTION = (3, 4, 5)  # scores landed, threshold, candidates


def seeded(shape, std, dtype, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype).to("cuda")


def main():
    assert os.environ.get("SAS_LIBRARY", "").endswith("libsas_trace.so"), "run with SAS_LIBRARY=.../libsas_trace.so"
    B, Hq, Hkv, K, bs, nblk = 4, 16, 4, 16, 64, 300
    Tmax = bs * nblk + 5
    ctx = torch.tensor([Tmax, Tmax - 64, Tmax - 100, 64 * 200 + 1], dtype=torch.int32, device="cuda")
    q = seeded((B, Hq, 128), 1.0, torch.bfloat16, 71)
    kc = seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 72)
    vc = seeded((B, Hkv, Tmax, 128), 1.0, torch.bfloat16, 73)
    s = seeded((B, Hkv, Tmax // bs), 1.0, torch.float32, 74)
    desc = api.decode_desc(q, kc, bs, K)
    o = torch.empty_like(q)
    idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
    api.sas_sparse_decode_launch_floor(desc, q, kc, vc, ctx, s, o)
    api.sas_sparse_decode_select(desc, q, kc, vc, ctx, s, o, idx)
    torch.cuda.synchronize()
    rows = api.sas_phase_trace_read(1024).astype(np.int64)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hkv):
            T = int(ctx[b])
            ro, ridx = oracle.decode(bits(q[b:b + 1, h * G:(h + 1) * G]), bits(kc[b:b + 1, h:h + 1, :T]),
                                     bits(vc[b:b + 1, h:h + 1, :T]), np.array([T], np.int32), bits(s[b:b + 1, h:h + 1]),
                                     bs, K)
            np.testing.assert_array_equal(idx[b, h].cpu().numpy(), ridx[0, 0])
            compare(f"o[{b},{h}]", host(o[b, h * G:(h + 1) * G]), ro[0], **BF16_TOL, bf16_out=True)
    n = int(rows[0, 31])
    cl = n // (B * Hkv)
    assert n == cl * B * Hkv and cl in (1, 2, 4, 8), n
    rows = rows[:n]
    for r in range(n):
        st = rows[r]
        seq = [int(st[k]) for k in ORDER]
        assert all(x <= y for x, y in zip(seq, seq[1:])), (r, seq)
        sel = [int(st[k]) for k in SELECTION]
        assert st[2] <= sel[0] <= sel[1] <= sel[2] <= st[6], (r, sel)
        assert st[17] >= K, (r, int(st[17]))
        assert st[13] <= st[0] + 10 ** 6 and st[15] >= st[11], r  # the clock pairs bracket the phases
        assert st[14] > st[12], r
    for row in range(B * Hkv):
        streamed = int(rows[row * cl:(row + 1) * cl, 18].sum())
        assert streamed == K + 1, (row, streamed)
    print("phase trace cases ok")


if __name__ == "__main__":
    main()
