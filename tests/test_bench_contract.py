"""bench.py's command-line contract, checked on the host: the reference arm (the
oracle on the host cores) prints one JSON line with the keys the harness reads,
and too few warm-up steps are refused."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=600)


def test_reference_arm_prints_the_contract_line():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "3", "--reference-tokens", "256")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["config"]["workload"] == "train_sparse_32k"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]


def test_too_few_warmup_steps_are_refused():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "2")
    assert r.returncode != 0 and "--warmup must be >= 3" in r.stderr


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    """The traffic record stays valid through comment and blank-line edits and is
    retired by any change to the code itself."""
    import importlib.util

    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    csrc = tmp_path / "trainable_block_sparse_sas_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = csrc / "k.cu"
    f.write_text("int f(int a) {\n    return a + 1;  // one\n}\n")
    base = bench.kernel_sources_sha(["k.cu"])
    f.write_text("/* header */\nint f(int a) {\n\n    // a new comment line\n  return a + 1;\n}\n")
    assert bench.kernel_sources_sha(["k.cu"]) == base
    f.write_text("int f(int a) {\n    return a + 2;  // one\n}\n")
    assert bench.kernel_sources_sha(["k.cu"]) != base


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the harness launches N > 1 (torchrun, one process per rank):
    rank 0 alone prints the line and every rank exits 0."""
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
                        "--reference-tokens", "256"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["impl"] == "reference"


def _bench():
    import importlib.util

    spec = importlib.util.spec_from_file_location("bench_mod2", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    return bench


def test_tensor_peak_follows_the_clock_record():
    """Burst peak when the timed region ran at the maximum clock with no throttle
    reason; the sustained (power-capped) figure otherwise or without a record."""
    bench = _bench()
    peaks = {"bf16_tflops": 1595.8, "bf16_tflops_sustained": 1385.2}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.tensor_peak(peaks, at_max)[0] == 1595.8
    assert bench.tensor_peak(peaks, dict(at_max, reasons=["sw_power_cap"]))[0] == 1385.2
    assert bench.tensor_peak(peaks, dict(at_max, sm_mhz=1500.0))[0] == 1385.2
    assert bench.tensor_peak(peaks, None)[0] == 1385.2


def test_kernel_breakdown_is_reproducible_from_the_times():
    """Per-kernel executed FLOPs (4d, 6d, 8d per attended pair) over the live
    times, as fractions of the named peak."""
    bench = _bench()
    from trainable_block_sparse_sas_b200 import synthetic as syn

    w = syn.TRAIN_SPARSE_32K
    fl = bench.train_flops(w)
    per_call = {"sas_topk_select": 0.04, "sas_gated_attn_fwd": 1.1, "sas_gated_attn_bwd": 5.0}
    out = bench.kernel_breakdown(fl, w, per_call, {"bwd_dq": 2.0, "bwd_dkdv": 3.0}, 1595.8)
    assert set(out) == {"fwd_sm100", "bwd_dq_sm100", "bwd_dkdv_sm100"}
    k = out["bwd_dkdv_sm100"]
    assert k["executed_flops"] == 8 * w.d * fl["pairs"]
    assert abs(k["executed_tflops"] - k["executed_flops"] / 3.0e-3 / 1e12) < 1e-6
    assert abs(k["frac_executed"] - k["executed_tflops"] / 1595.8) < 1e-12
    assert abs(sum(v["share_of_step"] for v in out.values()) - (1.1 + 5.0) / 6.14) < 1e-9


def test_phase_table_puts_ctas_on_one_time_line():
    """bench.phase_table: each CTA's %clock64 stamps are placed on the common
    %globaltimer line through its entry and exit (timer, clock) pairs, with the
    earliest entry as 0, in µs; the timer epoch (~1e18 ns) must not cost
    precision."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import bench

    rows = np.zeros((1024, 32), dtype=np.uint64)
    epoch = 1_700_000_000_000_000_000  # ns, as %globaltimer reads
    for cta, (gt0, clk0, ghz) in enumerate(((epoch + 1000, 5_000, 2.0), (epoch + 1037, 900_000, 1.0))):
        # phases 0..11 at 100 ns steps of this CTA's own clock after entry
        stamps = [clk0 + int(100 * k * ghz) for k in range(12)]
        rows[cta, :12] = stamps
        rows[cta, 12], rows[cta, 13] = gt0, clk0  # entry pair
        rows[cta, 15] = stamps[11]  # exit clock, read with the exit timer
        rows[cta, 14] = gt0 + 1100
        rows[cta, 17] = 16 + cta
        rows[cta, 18] = 8 + cta
    rows[0, 31] = 2
    t = bench.phase_table(rows)
    import pytest

    assert t["ctas"] == 2 and abs(t["sm_clock_ghz"] - 1.5) < 1e-9
    # [median, latest] in µs; the second CTA entered 37 ns after the first
    assert t["entry"] == pytest.approx([0.0185, 0.037], abs=1e-3)
    assert t["threshold"] == pytest.approx([0.4185, 0.437], abs=1e-3)  # phase 4: 400 ns after entry
    assert t["exit"] == pytest.approx([1.1185, 1.137], abs=1e-3)
    assert t["candidates_median"] == 16.5 and t["blocks_per_cta"] == [8, 9]
