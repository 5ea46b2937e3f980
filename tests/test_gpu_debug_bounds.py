"""The debug-bounds build (compute-sanitizer's stand-in on this GPU pool): the
library built with -DSAS_DEBUG_BOUNDS checks every global-memory index its
kernels compute against the extent of the buffer it addresses and records a
failure in the caller's status word instead of making the access.  Small
problems of every kernel family run through it in a process of their own, match
the oracle, and leave the status word at 0."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_bounds_build_runs_clean(cuda_ok):
    from trainable_block_sparse_sas_b200 import build

    lib = build.build(debug_bounds=True)
    env = dict(os.environ, SAS_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_bounds_cases.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    assert "debug-bounds cases ok" in r.stdout
