"""The transposed decode LM head (lmhead_tn.cuh: the batch as the M operand,
vocab slabs as N), which TPL_LMHEAD_TN=1 selects for batches of up to 32 rows.
The variable is read once per process, so the LM-head parity tests (every case,
the planted ids and cross-shard ties, the full-size decode workload, the merged
ranks and the static-scratch entry point) run again in a child process with it
set; they compare against the same fp64 oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_lmhead_parity_with_the_transposed_kernel():
    env = dict(os.environ, TPL_LMHEAD_TN="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
           "tests/test_gpu_kernels.py", "tests/test_gpu_workloads.py", "tests/test_gpu_ranks.py",
           "tests/test_zz_no_alloc.py", "-k", "lmhead or argmax or no_alloc or static"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "deselected" in r.stdout
