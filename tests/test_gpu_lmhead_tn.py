"""The decode LM head's other kernels.  For batches of up to 32 rows the
library runs the transposed kernel with a 64-row A operand (lmhead_tn.cuh,
TPL_LMHEAD_TN=2, the default); TPL_LMHEAD_TN=1 selects its 128-row form and
TPL_LMHEAD_TN=0 the swap-AB kernel (lmhead.cuh), which larger batches always
use.  The transposed kernel walks one contiguous vocab range per CTA in
256-row slabs by default; TPL_LMHEAD_RANGES=0 gives it uniform slabs dealt out
in turn.  TPL_LMHEAD_TN is read once per process, so the LM-head parity tests (every case,
the planted ids and cross-shard ties, the full-size decode workload, the merged
ranks and the static-scratch entry point) run again in a child process with it
set; they compare against the same fp64 oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("setting", [("TPL_LMHEAD_TN", "0"), ("TPL_LMHEAD_TN", "1"),
                                     ("TPL_LMHEAD_RANGES", "0")])
def test_lmhead_parity_with_the_other_kernels(setting):
    env = dict(os.environ, **{setting[0]: setting[1]})
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
           "tests/test_gpu_kernels.py", "tests/test_gpu_workloads.py", "tests/test_gpu_ranks.py",
           "tests/test_zz_no_alloc.py", "-k", "lmhead or argmax or no_alloc or static"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "deselected" in r.stdout
