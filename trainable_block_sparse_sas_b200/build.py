"""Build libsas.so (the CUDA kernels and their C ABI) in-tree for sm_100a.

    python -m trainable_block_sparse_sas_b200.build [--force] [-v] [--debug-bounds | --phase-trace]

Each csrc/*.cu is compiled to an object under _build/ (in parallel, skipped when
up to date), then linked into trainable_block_sparse_sas_b200/libsas.so.  With
--debug-bounds the same sources are built with -DSAS_DEBUG_BOUNDS (every kernel
checks the global-memory indices it computes against its buffers' extents and
records a failure in the caller's status word instead of making the access) into
libsas_debug.so, objects under _build/debug_bounds/.  With --phase-trace they are
built with -DSAS_PHASE_TRACE (the decode kernel records %clock64 at its phase
boundaries, read back by sas_phase_trace_read) into libsas_trace.so, objects
under _build/phase_trace/.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsas.so")
LIB_DEBUG = os.path.join(PKG, "libsas_debug.so")
LIB_TRACE = os.path.join(PKG, "libsas_trace.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-Xptxas", "-warn-spills", f"-I{INCLUDE}", f"-I{CSRC}"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    files = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return max((os.path.getmtime(f) for f in files), default=0.0)


def _compile(src: str, obj: str, verbose: bool, extra=()) -> str:
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stderr}")
    return r.stderr


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False, phase_trace: bool = False) -> str:
    if debug_bounds and phase_trace:
        raise ValueError("one variant at a time")
    if debug_bounds:
        out_dir, lib, extra = os.path.join(BUILD, "debug_bounds"), LIB_DEBUG, ("-DSAS_DEBUG_BOUNDS",)
    elif phase_trace:
        out_dir, lib, extra = os.path.join(BUILD, "phase_trace"), LIB_TRACE, ("-DSAS_PHASE_TRACE",)
    else:
        out_dir, lib, extra = BUILD, LIB, ()
    os.makedirs(out_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = _deps_mtime()
    jobs = []
    objs = []
    for src in srcs:
        obj = os.path.join(out_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), deps):
            jobs.append((src, obj))
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for (src, _), log in zip(jobs, ex.map(lambda j: _compile(j[0], j[1], verbose, extra), jobs)):
            if verbose and log:
                sys.stderr.write(f"== {os.path.basename(src)}\n{log}")
    if jobs or force or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        tmp = lib + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", *objs, "-o", tmp, "-lcuda"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug_bounds="--debug-bounds" in sys.argv,
                phase_trace="--phase-trace" in sys.argv))
