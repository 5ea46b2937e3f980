#!/usr/bin/env python
"""Benchmark of the SAS gated block-sparse attention hot path on B200.

One step = the whole training hot path over one batch of the 32K workload
(B=1, Hq=32, Hkv=8, d=128, n=32768, block 64, Top-K 32, bf16): score LSE and
Top-K selection, the gated forward, and the backward with dq/dk/dv and ds.
The metric counts tensor-core FLOPs on selected blocks only (4d per attended
(query, key) pair forward, 10d backward; the current block counts its causal
b(b+1)/2 pairs).  Extras (single GPU): full-scope 16K training, the four
ablated gates on the 32K workload, the pooled-key scorer, and the two decode
workloads (selection included; contiguous, two-call, paged and dense forms) in
GB/s of algorithmic bytes, each decode workload with the oracle timed on a
bounded host sample.  `e2e` repeats the 32K step through pinned host buffers,
every step copying its inputs in and its outputs out.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 the driver launches one rank per GPU with torchrun; every rank
processes its own independent batch (no collective on the data path), the
timing is the max over ranks, and `value` is the aggregate over all ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated sparse attn fwd+bwd TFLOP/s & decode selected-KV GB/s, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------
# workload arithmetic (algorithmic work, independent of any implementation)
# ----------------------------------------------------------------------------

def train_pairs(w) -> int:
    """Attended (query row, key) pairs of a training workload, over all heads."""
    hist = sum((c if w.full_scope else min(c, w.top_k)) for c in range(w.Cq))
    per_head = hist * w.bs * w.bs + w.Cq * w.bs * (w.bs + 1) // 2
    return w.B * w.Hq * per_head


def train_flops(w) -> dict:
    pairs = train_pairs(w)
    return {"pairs": pairs, "fwd": 4 * w.d * pairs, "bwd": 10 * w.d * pairs, "total": 14 * w.d * pairs}


def decode_bytes(w, dense: bool = False) -> int:
    """Algorithmic HBM bytes of one decode step: attended K and V rows, the score
    rows (sparse only), q and o."""
    t = w.T - 1
    cur = t - (t // w.bs) * w.bs + 1
    toks = (t + 1) if dense else (min(w.top_k, w.C) * w.bs + cur)
    kv = w.B * w.Hkv * toks * w.d * 2 * 2
    s = 0 if dense else w.B * w.Hkv * w.C * 4
    qo = 2 * w.B * w.Hq * w.d * 2
    return kv + s + qo


def max_over_ranks(value: float, world: int, device="cpu") -> float:
    """Max of a per-rank timing over all ranks (identity for one rank).  The
    collective is plumbing for the measurement only, never on the data path."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flops_per_step: float, steps: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processes its own batch (weak scaling)."""
    return world * flops_per_step * steps / (ms_max * 1e-3) / 1e12


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_sources_sha(names) -> str:
    """Hash of the kernel sources with comments removed, so that an edit to
    comments alone does not retire the counters taken on the same code."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "trainable_block_sparse_sas_b200", "csrc", n), encoding="utf-8") as f:
            code = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
        code = re.sub(r"//[^\n]*", "", code)
        code = "\n".join(ln.strip() for ln in code.splitlines() if ln.strip())  # blank lines, indentation
        h.update(code.encode())
    return h.hexdigest()[:16]


def recorded_traffic(call: str):
    """DRAM bytes per launch of an ABI call from a committed ncu summary, if the
    kernel sources it was taken on are unchanged (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(call)
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    if kernel_sources_sha(rec["sources"]) != rec["sources_sha"]:
        return None
    return rec["dram_bytes_per_launch"]


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.gpu_id], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [ln.strip().split(",") for ln in self.out.read().splitlines() if ln.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def visible_gpu_id(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ----------------------------------------------------------------------------
# oracle on the host cores (CPU baseline and the reference arm)
# ----------------------------------------------------------------------------

def oracle_sample(w, inp_host: dict, tokens: int):
    """The oracle's fwd + bwd on the first `tokens` tokens of KV head 0 (its
    query-head group): a complete sub-problem of the workload, since attention is
    causal and KV heads are independent.  Returns (seconds, FLOPs, threads)."""
    import oracle

    G = w.Hq // w.Hkv
    sub = dataclasses.replace(w, B=1, Hq=G, Hkv=1, n=tokens)
    q = inp_host["q"][:1, :tokens, :G]
    k = inp_host["k"][:1, :tokens, :1]
    v = inp_host["v"][:1, :tokens, :1]
    dO = inp_host["dO"][:1, :tokens, :G]
    Cq = tokens // w.bs
    s = inp_host["s"][:1, :1, :Cq, :Cq]
    import numpy as np

    q, k, v, dO, s = (np.ascontiguousarray(x) for x in (q, k, v, dO, s))
    t0 = time.perf_counter()
    oracle.train_select(s, w.top_k, full_scope=w.full_scope)
    oracle.attn_fwd(q, k, v, s, w.bs, w.top_k, full_scope=w.full_scope)
    oracle.attn_bwd(q, k, v, dO, s, w.bs, w.top_k, full_scope=w.full_scope)
    dt = time.perf_counter() - t0
    return dt, train_flops(sub)["total"], oracle.num_threads()


def host_bits(t):
    import numpy as np
    import torch

    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def run_reference(args, rank: int):
    """The reference arm: the fp64 oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    import torch

    from trainable_block_sparse_sas_b200 import synthetic as syn

    w = syn.WORKLOADS[args.workload]
    import oracle

    oracle.build()
    tokens = args.reference_tokens
    inp = syn.train_inputs(dataclasses.replace(w, n=tokens, B=1), device="cpu", seed=1000)
    host = {k: host_bits(v) for k, v in inp.items()}
    times = []
    flops = 0
    threads = 1
    for i in range(args.warmup + args.steps):
        dt, flops, threads = oracle_sample(w, host, tokens)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = flops * len(times) / total / 1e12
    sample = (f"first {tokens} tokens of KV head 0 ({w.Hq // w.Hkv} query heads) of {w.name}: "
              f"select + fwd + bwd per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    del torch


def tensor_peak(peaks: dict, clk) -> tuple[float, str]:
    """The burst bf16 figure when the clock record of the timed region shows the
    SM clock at its maximum with no throttle reason (a kernel timed over a short
    region runs at full clock), else the sustained figure (measured under the
    power cap at a lower clock)."""
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if clk and not clk["reasons"] and clk["sm_mhz"] >= 0.97 * clk["sm_max_mhz"]:
        return burst, "bf16 burst (clocks at maximum, no throttle reason)"
    return sustained, "bf16 sustained"


def kernel_breakdown(fl: dict, w, per_call: dict, per_kernel_ms: dict, peak: float) -> dict:
    """Per-kernel live times and the MMA FLOPs each kernel executes (the forward:
    S and O = P V, 4d per attended pair; the dq kernel: S, dP and dQ, 6d; the
    dk/dv kernel: S, dP, dV and dK, 8d), as tensor-pipe fractions of the peak.
    The algorithmic count of the backward (10d per pair) credits S and dP once;
    the dk/dv kernel recomputes them, so the two kernels execute 14d."""
    pairs = fl["pairs"]
    ex = {"fwd_sm100": (4 * w.d * pairs, per_call["sas_gated_attn_fwd"]),
          "bwd_dq_sm100": (6 * w.d * pairs, per_kernel_ms["bwd_dq"]),
          "bwd_dkdv_sm100": (8 * w.d * pairs, per_kernel_ms["bwd_dkdv"])}
    step = sum(per_call.values())
    out = {}
    for name, (flops, ms) in ex.items():
        tf = flops / (ms * 1e-3) / 1e12
        out[name] = {"ms": ms, "share_of_step": ms / step, "executed_flops": flops, "executed_tflops": tf,
                     "frac_executed": tf / peak}
    return out


def workload_config(w, n_gpus: int) -> dict:
    return {"workload": w.name, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d, "seq_len": w.n,
            "block_size": w.bs, "top_k": w.top_k, "scope": "full" if w.full_scope else "sparse",
            "parallelism": f"replicas x{n_gpus} (independent batches, no collective)",
            "l2": "inputs larger than L2 (q and dO 268 MB each, k and v 67 MB each)"}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

class TrainRunner:
    """Preallocated buffers and the three ABI calls of one training step."""

    def __init__(self, api, w, inp, gate: str = "softmax"):
        import torch

        self.api, self.w = api, w
        self.inp = inp
        q, k = inp["q"], inp["k"]
        dev = q.device
        self.desc = api.attn_desc(q, k, w.bs, w.top_k, w.full_scope, gate=gate)
        self.lse_s = torch.empty((w.B, w.Hkv, w.Cq), dtype=torch.float32, device=dev)
        self.idx = None if (w.full_scope or w.top_k == 0) else torch.empty(
            (w.B, w.Hkv, w.Cq, w.top_k), dtype=torch.int32, device=dev)
        self.o = torch.empty_like(q)
        self.lse = torch.empty((w.B, w.Hq, w.n), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(inp["v"])
        self.ds = torch.empty_like(inp["s"])
        self.ws = api.workspace(api.sas_gated_attn_bwd_workspace_size(self.desc), dev)

    def step(self, ev=None):
        """One step; with ev (5 timing events) the events bracket the selection, the
        forward, and the backward's two kernels (recorded by the library between
        them through sas_gated_attn_bwd_timed)."""
        api, i = self.api, self.inp
        if ev:
            ev[0].record()
        api.sas_topk_select(i["s"], self.w.Cq, self.w.Cq, self.w.top_k, idx=self.idx, lse_s=self.lse_s)
        if ev:
            ev[1].record()
        api.sas_gated_attn_fwd(self.desc, i["q"], i["k"], i["v"], i["s"], self.lse_s, self.idx, self.o, self.lse)
        args = (self.desc, i["q"], i["k"], i["v"], self.o, self.lse, i["dO"], i["s"], self.lse_s, self.idx, self.dq,
                self.dk, self.dv, self.ds, self.ws)
        if ev:
            api.sas_gated_attn_bwd_timed(*args, events=ev[2:5])
        else:
            api.sas_gated_attn_bwd(*args)

    def outputs(self):
        return {"o": self.o, "dq": self.dq, "dk": self.dk, "dv": self.dv, "ds": self.ds}


def time_decode(api, w, steps: int, mode: str = "fused"):
    """Median device time of one decode step with L2 flushed (a 512 MB read, so
    no dirty lines are written back inside the timed window) before every
    repetition.  mode: "fused" (sas_sparse_decode_select: selection + attention
    in one launch), "two_call" (sas_topk_select then sas_sparse_decode), "dense"
    (sas_sparse_decode over every cached token), or "paged" (the fused step on the
    same cache scattered into a shuffled pool of one-block pages,
    sas_sparse_decode_paged).  Repetitions rotate among 4 score tensors, so the
    attended blocks change from one repetition to the next."""
    import torch

    from trainable_block_sparse_sas_b200 import synthetic as syn

    inp = syn.decode_inputs(w, device="cuda", seed=3000)
    q, kc, vc, ctx, s = (inp[x] for x in ("q", "k_cache", "v_cache", "ctx_len", "s"))
    desc = api.decode_desc(q, kc, w.bs, w.top_k)
    idx = torch.empty((w.B, w.Hkv, w.top_k), dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    ws = api.workspace(api.sas_sparse_decode_workspace_size(desc), q.device)
    flush = torch.ones(128 << 20, dtype=torch.float32, device="cuda")
    gs = torch.Generator(device="cuda")
    gs.manual_seed(3200)
    s_rot = [s] + [torch.randn(s.shape, generator=gs, device="cuda") * w.s_std for _ in range(3)]
    cur = {"s": s}
    if mode == "paged":
        pps = (w.T + w.bs - 1) // w.bs
        g = torch.Generator(device="cpu")
        g.manual_seed(3100)
        table = torch.randperm(w.B * pps, generator=g).view(w.B, pps).to(torch.int32).cuda()
        pools = []
        for c in (kc, vc):
            pool = torch.empty((w.B * pps, w.bs, w.Hkv, w.d), dtype=c.dtype, device="cuda")
            for b in range(w.B):  # one sequence at a time keeps the temporaries small
                pages = torch.nn.functional.pad(c[b], (0, 0, 0, pps * w.bs - w.T))
                pool[table[b].long()] = pages.view(w.Hkv, pps, w.bs, w.d).permute(1, 2, 0, 3)
                del pages
            pools.append(pool)
        inp["k_cache"] = inp["v_cache"] = kc = vc = c = None
        torch.cuda.empty_cache()
        kp, vp = pools
        pdesc = api.paged_decode_desc(q, kp, w.bs, w.top_k, w.T)

    def run():
        sc = cur["s"]
        if mode == "fused":
            api.sas_sparse_decode_select(desc, q, kc, vc, ctx, sc, o, idx)
            return
        if mode == "paged":
            api.sas_sparse_decode_paged(pdesc, q, kp, vp, table, ctx, o, s=sc, idx_out=idx)
            return
        if mode == "two_call":
            api.sas_topk_select(sc.view(w.B, w.Hkv, 1, -1), 1, sc.shape[-1], w.top_k, idx=idx, ctx_len=ctx,
                                block_size=w.bs)
        api.sas_sparse_decode(desc, q, kc, vc, ctx, None if mode == "dense" else idx, o, ws)

    for _ in range(3):
        run()
    times = []
    for i in range(steps):
        cur["s"] = s_rot[i % 4]
        flush.sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    del inp, kc, vc, flush
    torch.cuda.empty_cache()
    return statistics.median(times)


def time_decode_graph(api, w, reps: int = 20, n_steps: int = 16) -> float:
    """Median device time per fused decode step (sas_sparse_decode_select) when
    n_steps steps run back to back from one CUDA graph, as a serving loop replays
    them: events around each replay, time / n_steps.  The steps read n_steps
    different score tensors, so each attends its own blocks: n_steps x the
    attended K/V of a step (1.1 GB for decode_128k, 0.56 GB for decode_512k)
    passes through L2 per replay, and a step's blocks are long evicted when they
    come round again; q and the current block stay in L2, as they would after the
    preceding kernels of a decode step."""
    import torch

    from trainable_block_sparse_sas_b200 import synthetic as syn

    inp = syn.decode_inputs(w, device="cuda", seed=3000)
    q, kc, vc, ctx, s = (inp[x] for x in ("q", "k_cache", "v_cache", "ctx_len", "s"))
    desc = api.decode_desc(q, kc, w.bs, w.top_k)
    idx = torch.empty((w.B, w.Hkv, w.top_k), dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    gs = torch.Generator(device="cuda")
    gs.manual_seed(3200)
    s_rot = [s] + [torch.randn(s.shape, generator=gs, device="cuda") * w.s_std for _ in range(n_steps - 1)]
    for sc in s_rot[:3]:
        api.sas_sparse_decode_select(desc, q, kc, vc, ctx, sc, o, idx)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            for sc in s_rot:
                api.sas_sparse_decode_select(desc, q, kc, vc, ctx, sc, o, idx)
    torch.cuda.current_stream().wait_stream(st)
    for _ in range(3):
        g.replay()
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b) / n_steps)
    del g, inp, kc, vc, s_rot
    torch.cuda.empty_cache()
    return statistics.median(times)


PHASES = ("entry", "ctx_len", "cluster_barrier", "scores_landed", "threshold", "candidates", "selected",
          "first_block", "stream_end", "cta_partial", "slices_received", "exit")


def phase_table(rows) -> dict:
    """Per-phase median and maximum (us after the earliest CTA entry) from the
    decode kernel's trace rows, each CTA's %clock64 stamps put on the common
    %globaltimer line by its entry and exit (timer, clock) pairs."""
    import numpy as np

    raw = np.asarray(rows, dtype=np.int64)
    n = int(raw[0, 31])
    raw = raw[:n]
    # timer values are ns since an epoch (~1e18): offsets first, in integers, so
    # that float64 keeps ns resolution
    gt0 = raw[:, 12].min()
    rows = raw.astype(np.float64)
    gte = (raw[:, 12] - gt0).astype(np.float64)
    rate = (raw[:, 14] - raw[:, 12]).astype(np.float64) / (raw[:, 15] - raw[:, 13]).astype(np.float64)  # ns/clock
    t = gte[:, None] + (raw[:, :12] - raw[:, 13:14]).astype(np.float64) * rate[:, None]
    t0 = t[:, 0].min()
    out = {"ctas": n, "sm_clock_ghz": float(np.median(1.0 / rate))}
    for k, name in enumerate(PHASES):
        v = (t[:, k] - t0) / 1e3
        ok = (rows[:, k] >= rows[:, 13] - 1e6) & (rows[:, k] <= rows[:, 15])  # stamped in this launch
        if ok.all():
            out[name] = [round(float(np.median(v)), 3), round(float(v.max()), 3)]
    out["candidates_median"] = float(np.median(rows[:, 17]))
    out["blocks_per_cta"] = [int(rows[:, 18].min()), int(rows[:, 18].max())]
    return out


def decode_phases(api) -> dict:
    """Launch floor and phase breakdown of the fused decode step on both decode
    workloads: events around one launch (L2 flushed before it) and per step of a
    16-step CUDA graph, for the decode and for an empty kernel on the same grid,
    cluster, block and shared memory (sas_sparse_decode_launch_floor); with a
    library built with --phase-trace, the per-phase table of one flushed launch
    and of the last step of a graph replay."""
    import torch

    from trainable_block_sparse_sas_b200 import synthetic as syn

    traced = True
    out = {}
    for w in (syn.DECODE_128K, syn.DECODE_512K):
        inp = syn.decode_inputs(w, device="cuda", seed=3000)
        q, kc, vc, ctx, s = (inp[x] for x in ("q", "k_cache", "v_cache", "ctx_len", "s"))
        desc = api.decode_desc(q, kc, w.bs, w.top_k)
        idx = torch.empty((w.B, w.Hkv, w.top_k), dtype=torch.int32, device="cuda")
        o = torch.empty_like(q)
        flush = torch.ones(128 << 20, dtype=torch.float32, device="cuda")
        gs = torch.Generator(device="cuda")
        gs.manual_seed(3200)
        s_rot = [s] + [torch.randn(s.shape, generator=gs, device="cuda") * w.s_std for _ in range(15)]
        rec = {}
        calls = {"decode": lambda sc: api.sas_sparse_decode_select(desc, q, kc, vc, ctx, sc, o, idx),
                 "floor": lambda sc: api.sas_sparse_decode_launch_floor(desc, q, kc, vc, ctx, sc, o)}
        for name, call in calls.items():
            for sc in s_rot[:3]:
                call(sc)
            ts = []
            for i in range(20):
                flush.sum()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                call(s_rot[i % 16])
                b.record()
                b.synchronize()
                ts.append(a.elapsed_time(b) * 1e3)
            rec[name + "_single_us"] = statistics.median(ts)
            if name == "decode" and traced:
                try:
                    rec["phases_single"] = phase_table(api.sas_phase_trace_read(1024))
                except api.SasError:  # a library built without the trace
                    traced = False
            g = torch.cuda.CUDAGraph()
            st = torch.cuda.Stream()
            st.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(st):
                with torch.cuda.graph(g, stream=st):
                    for sc in s_rot:
                        call(sc)
            torch.cuda.current_stream().wait_stream(st)
            g.replay()
            ts = []
            for _ in range(20):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                g.replay()
                b.record()
                b.synchronize()
                ts.append(a.elapsed_time(b) * 1e3 / 16)
            rec[name + "_graph_us"] = statistics.median(ts)
            if name == "decode" and traced:
                rec["phases_graph_last_step"] = phase_table(api.sas_phase_trace_read(1024))
            del g
        rec["stream_bytes"] = decode_bytes(w)
        out[w.name] = rec
        del inp, kc, vc, flush, s_rot
        torch.cuda.empty_cache()
    return out


def decode_oracle_sample(w) -> dict:
    """The oracle's decode (selection + attention, fp64) timed on the host cores
    on a bounded sample of the workload: sequence 0 and kv head 0 (its G query
    heads) at the full context length, reported as GB/s of that row's algorithmic
    bytes (the decode_bytes count for one row)."""
    import oracle
    from trainable_block_sparse_sas_b200 import synthetic as syn

    inp = syn.decode_inputs(w, device="cuda", seed=3000)
    G = w.Hq // w.Hkv
    host = {"q": syn.bf16_bits(inp["q"][0:1, 0:G]), "k": syn.bf16_bits(inp["k_cache"][0:1, 0:1]),
            "v": syn.bf16_bits(inp["v_cache"][0:1, 0:1]), "s": inp["s"][0:1, 0:1].cpu().numpy(),
            "ctx": inp["ctx_len"][0:1].cpu().numpy()}
    del inp
    t0 = time.perf_counter()
    oracle.decode(host["q"], host["k"], host["v"], host["ctx"], host["s"], w.bs, w.top_k)
    dt = time.perf_counter() - t0
    by = decode_bytes(w) // (w.B * w.Hkv)
    return {"value": by / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"sequence 0, kv head 0 ({G} query heads) at {w.T} tokens: {dt * 1e3:.1f} ms"}


def time_decode_scores(api, w, hbm: float) -> dict:
    """Pooled-key decode scores over the workload's block summaries (one bf16 row
    per full block): the selector-scoring pass that precedes selection."""
    import torch

    g = torch.Generator(device="cpu")
    g.manual_seed(3100)
    Cb = (w.T - 1) // w.bs
    q = (torch.randn((w.B, w.Hq, w.d), generator=g)).to(w.dtype).cuda()
    ksum = (torch.randn((w.B, w.Hkv, Cb, w.d), generator=g) * 0.2).to(w.dtype).cuda()
    ctx = torch.full((w.B,), w.T, dtype=torch.int32, device="cuda")
    s = torch.empty((w.B, w.Hkv, Cb), dtype=torch.float32, device="cuda")
    desc = api.DecodeDesc(w.B, w.Hq, w.Hkv, w.d, w.bs, w.top_k, w.T, api.SAS_BF16, 0.0)
    flush = torch.empty(128 << 20, dtype=torch.float32, device="cuda")
    for _ in range(3):
        api.sas_decode_scores(desc, q, ksum, ctx, s)
    ts = []
    for _ in range(10):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        api.sas_decode_scores(desc, q, ksum, ctx, s)
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    us = sorted(ts)[len(ts) // 2]
    by = ksum.numel() * ksum.element_size() + s.numel() * 4 + q.numel() * q.element_size()
    return {"us": us, "bytes": by, "gbs": by / (us * 1e-6) / 1e9, "frac_of_hbm": by / (us * 1e-6) / 1e9 / hbm,
            "l2": "flushed (512 MB write) before every repetition"}


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from trainable_block_sparse_sas_b200 import api
    from trainable_block_sparse_sas_b200 import synthetic as syn

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = syn.WORKLOADS[args.workload]
    inp = syn.train_inputs(w, device=dev, seed=1000 + rank)
    runner = TrainRunner(api, w, inp)
    fl = train_flops(w)
    peaks, peak_kind = load_peaks()

    def barrier():
        if world > 1:
            t = torch.ones(1, device=dev)
            dist.all_reduce(t)
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        runner.step()
    barrier()
    clocks = ClockSampler(visible_gpu_id(local_rank))
    clocks.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for e in (e for es in evs for e in es):
        e.record()  # torch creates a CUDA event on its first record: outside the timed region
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = api.sas_launch_count()
    barrier()
    start.record()
    for i in range(args.steps):
        runner.step(evs[i])
    end.record()
    torch.cuda.synchronize()
    launches = api.sas_launch_count() - launches0
    barrier()
    clk = clocks.stop()
    ms_max = max_over_ranks(start.elapsed_time(end), world, dev)
    per_call = {
        "sas_topk_select": statistics.mean(e[0].elapsed_time(e[1]) for e in evs),
        "sas_gated_attn_fwd": statistics.mean(e[1].elapsed_time(e[2]) for e in evs),
        "sas_gated_attn_bwd": statistics.mean(e[2].elapsed_time(e[4]) for e in evs),
    }
    per_kernel_ms = {  # the backward's two kernels, from the events the library records between them
        "bwd_dq": statistics.mean(e[2].elapsed_time(e[3]) for e in evs),
        "bwd_dkdv": statistics.mean(e[3].elapsed_time(e[4]) for e in evs),
    }
    value = aggregate_tflops(world, fl["total"], args.steps, ms_max)

    # end to end through host buffers: every step copies its inputs in from pinned
    # host memory and its outputs back.  Two device buffer sets let the copies of
    # the neighbouring steps (one copy engine each way) overlap a step's kernels.
    # At least 16 steps, so that the pipeline's fill (the first step's inputs) and
    # drain (the last step's outputs) weigh little in the per-step figure.
    e2e_steps = max(16, min(args.steps, 64))
    host_in = {k: v.cpu().pin_memory() for k, v in inp.items()}
    host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in runner.outputs().items()}
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(v.numel() * v.element_size() for v in host_out.values())
    inp2 = {k: torch.empty_like(v) for k, v in inp.items()}
    runners = [runner, TrainRunner(api, w, inp2)]
    bufs = [inp, inp2]
    s_in, s_out, s_run = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.current_stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    run_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    torch.cuda.synchronize()
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_run)
    s_in.wait_stream(s_run)
    s_out.wait_stream(s_run)
    for i in range(e2e_steps):
        sl = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(run_done[sl])  # step i-2 has finished reading this buffer
            for k_, v_ in host_in.items():
                bufs[sl][k_].copy_(v_, non_blocking=True)
            in_done[sl].record(s_in)
        s_run.wait_event(in_done[sl])
        if i >= 2:
            s_run.wait_event(out_done[sl])  # step i-2's outputs have left this buffer
        runners[sl].step()
        run_done[sl].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(run_done[sl])
            for k_, v_ in runners[sl].outputs().items():
                host_out[k_].copy_(v_, non_blocking=True)
            out_done[sl].record(s_out)
    s_run.wait_stream(s_in)
    s_run.wait_stream(s_out)
    b.record(s_run)
    torch.cuda.synchronize()
    e2e_value = aggregate_tflops(world, fl["total"], e2e_steps, max_over_ranks(a.elapsed_time(b), world, dev))
    del host_in, host_out, runners, bufs, inp2

    if rank != 0:
        barrier()
        return
    dom = max(per_call, key=per_call.get)
    dom_flops = {"sas_topk_select": 0, "sas_gated_attn_fwd": fl["fwd"], "sas_gated_attn_bwd": fl["bwd"]}[dom]
    peak, peak_name = tensor_peak(peaks, clk)
    achieved = dom_flops / (per_call[dom] * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w, world),
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": recorded_traffic(dom),
                     "peak_source": f"{peak_kind} {peak_name}", "per_call_ms": per_call,
                     "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained",
                                                               FALLBACK_PEAKS["bf16_tflops_sustained"]),
                     "frac_of_datasheet_2250": achieved / 2250.0,
                     "kernels": kernel_breakdown(fl, w, per_call, per_kernel_ms, peak),
                     "flops_per_step": fl},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        host = {k: host_bits(v) for k, v in inp.items()}
        dt, flops, threads = oracle_sample(w, host, args.cpu_tokens)
        line["cpu_baseline"] = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": f"first {args.cpu_tokens} tokens of KV head 0 (4 query heads): select + "
                                          f"fwd + bwd, {dt:.1f} s"}
    del runner, inp
    torch.cuda.empty_cache()
    if world == 1 and not args.no_extra:
        line["extra"] = extras(api, args, peaks, peak_kind)
    print(json.dumps(line), flush=True)
    barrier()


def extras(api, args, peaks, peak_kind) -> dict:
    import torch

    from trainable_block_sparse_sas_b200 import synthetic as syn

    out = {}
    # full-scope training
    w = syn.TRAIN_FULL_16K
    inp = syn.train_inputs(w, device="cuda", seed=1500)
    r = TrainRunner(api, w, inp)
    for _ in range(2):
        r.step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(2, min(args.steps, 5))
    a.record()
    for _ in range(n):
        r.step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    fl = train_flops(w)
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    out[w.name] = {"ms_per_step": ms, "tflops": fl["total"] / (ms * 1e-3) / 1e12,
                   "frac_of_bf16_peak": fl["total"] / (ms * 1e-3) / 1e12 / peak,
                   "peak_source": f"{peak_kind} bf16 burst"}
    del r, inp
    torch.cuda.empty_cache()
    # 8 query heads per KV head (two forward and dq CTAs per query block)
    w = syn.TRAIN_SPARSE_32K_GQA8
    inp = syn.train_inputs(w, device="cuda", seed=1700)
    r = TrainRunner(api, w, inp)
    for _ in range(2):
        r.step()
    torch.cuda.synchronize()
    a.record()
    for _ in range(n):
        r.step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    fl = train_flops(w)
    out[w.name] = {"ms_per_step": ms, "tflops": fl["total"] / (ms * 1e-3) / 1e12,
                   "frac_of_bf16_peak": fl["total"] / (ms * 1e-3) / 1e12 / peak,
                   "path": list(api.sas_attn_path(r.desc))}
    del r, inp
    torch.cuda.empty_cache()
    # the ablated gates on the headline training workload (same FLOP convention;
    # the hard STE gate's dq kernel also walks every dropped block, uncounted)
    w = syn.TRAIN_SPARSE_32K
    inp = syn.train_inputs(w, device="cuda", seed=1600)
    fl = train_flops(w)
    gates = {}
    for gate in ("sigmoid", "raw", "outer", "ste"):
        r = TrainRunner(api, w, inp, gate=gate)
        for _ in range(2):
            r.step()
        torch.cuda.synchronize()
        a.record()
        for _ in range(n):
            r.step()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / n
        gates[gate] = {"ms_per_step": ms, "tflops": fl["total"] / (ms * 1e-3) / 1e12}
        del r
        torch.cuda.empty_cache()
    out["gate_variants_" + w.name] = gates
    # pooled-key scorer on the same workload: one pass over q and k (HBM bound)
    desc = api.attn_desc(inp["q"], inp["k"], w.bs, w.top_k)
    s = torch.empty_like(inp["s"])
    ws = api.workspace(api.sas_pooled_scores_workspace_size(desc), inp["q"].device)
    for _ in range(3):
        api.sas_pooled_scores(desc, inp["q"], inp["k"], s, ws)
    reps = 10
    a.record()
    for _ in range(reps):
        api.sas_pooled_scores(desc, inp["q"], inp["k"], s, ws)
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) / reps * 1e3
    by = inp["q"].numel() * inp["q"].element_size() + inp["k"].numel() * inp["k"].element_size()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    out["pooled_scores_" + w.name] = {"us": us, "bytes": by, "gbs": by / (us * 1e-6) / 1e9,
                                      "frac_of_hbm": by / (us * 1e-6) / 1e9 / hbm,
                                      "l2": "q and k (335 MB) exceed L2"}
    del inp, s, ws
    torch.cuda.empty_cache()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    for w in (syn.DECODE_128K, syn.DECODE_512K):
        ms = time_decode_graph(api, w)
        ms1 = time_decode(api, w, steps=20, mode="fused")
        by = decode_bytes(w)
        gbs = by / (ms * 1e-3) / 1e9
        rec = {"ms": ms, "bytes": by, "gbs": gbs, "frac_of_hbm": gbs / hbm, "hbm_peak_gbs": hbm,
               "peak_source": f"{peak_kind} copy", "frac_of_8tbs": gbs / 8000.0,
               "timing": "per step of 16 back-to-back steps replayed from one CUDA graph, each step with its own "
                         "score tensor (inputs larger than L2: the steps' attended blocks differ)",
               "includes": "Top-K selection + sparse decode in one launch (sas_sparse_decode_select)",
               "single_launch_ms": ms1,
               "single_launch_timing": "events around one launch, L2 flushed (512 MB read) before each; includes "
                                       "the event and launch floor of a lone kernel (an empty kernel on the same "
                                       "grid measures ~5-6 us this way)",
               "two_call_ms": time_decode(api, w, steps=10, mode="two_call"),
               "paged_ms": time_decode(api, w, steps=10, mode="paged")}
        rec["decode_scores"] = time_decode_scores(api, w, hbm)
        rec["cpu_oracle"] = decode_oracle_sample(w)
        if w is syn.DECODE_512K:
            msd = time_decode(api, w, steps=5, mode="dense")
            byd = decode_bytes(w, dense=True)
            rec["dense_ms"] = msd
            rec["dense_gbs"] = byd / (msd * 1e-3) / 1e9
            # the dense stream can exceed the torch-copy figure; the best rate seen is the tighter ceiling
            rec["frac_of_best_stream"] = gbs / max(hbm, rec["dense_gbs"])
            rec["sparse_over_dense_speedup"] = msd / ms1
        out[w.name] = rec
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="train_sparse_32k")
    ap.add_argument("--no-extra", action="store_true", help="skip the full-scope and decode extras")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=4096, help="tokens of the oracle's CPU-baseline sample")
    ap.add_argument("--reference-tokens", type=int, default=1024, help="tokens of the reference arm's sample")
    ap.add_argument("--profile-train", type=int, default=0, metavar="N",
                    help="only run training steps of the 32K workload's geometry at sequence length N (a small "
                         "case for profiler captures) and print the per-kernel timing")
    ap.add_argument("--profile-decode", type=int, default=0, metavar="T",
                    help="only run the fused decode of the 128K workload's geometry with a T-token cache "
                         "(a small case for profiler captures) and print its timing")
    ap.add_argument("--decode-phases", action="store_true",
                    help="only measure the decode launch floor and (with a --phase-trace build loaded through "
                         "SAS_LIBRARY) the per-phase breakdown of the fused decode step")
    ap.add_argument("--profile-scores", type=int, default=0, metavar="N",
                    help="only run the pooled-key scorer of the 32K workload's geometry at sequence length N (a "
                         "small case for profiler captures) and print its timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.profile_train:
        import torch

        from trainable_block_sparse_sas_b200 import api
        from trainable_block_sparse_sas_b200 import synthetic as syn

        w = dataclasses.replace(syn.TRAIN_SPARSE_32K, name="train_sparse_geometry", n=args.profile_train)
        r = TrainRunner(api, w, syn.train_inputs(w, device="cuda", seed=1000))
        for _ in range(args.warmup):
            r.step()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
        for i in range(args.steps):
            r.step(evs[i])
        torch.cuda.synchronize()
        ms = {k: statistics.mean(e[a].elapsed_time(e[b]) for e in evs)
              for k, (a, b) in {"select": (0, 1), "fwd": (1, 2), "bwd_dq": (2, 3), "bwd_dkdv": (3, 4)}.items()}
        print(json.dumps({"workload": w.name, "n": w.n, "ms": ms}))
        return
    if args.decode_phases:
        from trainable_block_sparse_sas_b200 import api

        print(json.dumps(decode_phases(api)))
        return
    if args.profile_scores:
        import torch

        from trainable_block_sparse_sas_b200 import api
        from trainable_block_sparse_sas_b200 import synthetic as syn

        w = dataclasses.replace(syn.TRAIN_SPARSE_32K, name="scores_geometry", n=args.profile_scores)
        inp = syn.train_inputs(w, device="cuda", seed=2100)
        desc = api.attn_desc(inp["q"], inp["k"], w.bs, w.top_k)
        s = torch.empty((w.B, w.Hkv, w.Cq, w.Cq), device="cuda")
        ws = api.workspace(api.sas_pooled_scores_workspace_size(desc), inp["q"].device)
        for _ in range(args.warmup):
            api.sas_pooled_scores(desc, inp["q"], inp["k"], s, ws)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in evs:
            a.record()
            api.sas_pooled_scores(desc, inp["q"], inp["k"], s, ws)
            b.record()
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        print(json.dumps({"workload": w.name, "n": w.n, "ms": ms}))
        return
    if args.profile_decode:
        from trainable_block_sparse_sas_b200 import api
        from trainable_block_sparse_sas_b200 import synthetic as syn

        w = dataclasses.replace(syn.DECODE_128K, name="decode_128k_geometry", T=args.profile_decode)
        ms = time_decode(api, w, steps=args.steps, mode="fused")
        print(json.dumps({"workload": w.name, "T": w.T, "ms": ms, "gbs": decode_bytes(w) / (ms * 1e-3) / 1e9}))
        return
    if world > 1:
        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
