"""The phase-trace build of the library (-DSAS_PHASE_TRACE): the traced decode
kernel still matches the oracle and records a consistent trace; the launch-floor
entry point runs."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_phase_trace_build(cuda_ok):
    from trainable_block_sparse_sas_b200 import build

    lib = build.build(phase_trace=True)
    env = dict(os.environ, SAS_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "phase_trace_cases.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    assert "phase trace cases ok" in r.stdout


def test_release_build_has_no_trace(cuda_ok):
    from trainable_block_sparse_sas_b200 import api

    with pytest.raises(api.SasError) as e:
        api.sas_phase_trace_read(4)
    assert e.value.status == api.SAS_ERR_UNSUPPORTED
