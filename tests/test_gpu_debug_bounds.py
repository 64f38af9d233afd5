"""The GPU parity suite once more, on the debug build of the library
(libslope_debug.so, compiled with -DSLOPE_DEBUG_BOUNDS).

In that build every plain global-memory load and store of every kernel
checks its index range against the extent of its buffer that the host
derived from the call's sizes (TMA tiles are bounded by their tensor maps);
an access outside is skipped and recorded, and the next slope_status_sync,
which every parity test calls, fails with SLOPE_ERR_BOUNDS.  With the canary
guard bands of the parity suite this stands in for a device memory checker:
every shape of the suite, the full-size sampled ones included, runs with no
index outside its buffer.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.gpu
def test_parity_suite_under_bounds_checks():
    env = dict(os.environ, SLOPE_DEBUG_BOUNDS="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_parity.py"), os.path.join(HERE, "test_zz_no_alloc.py")]
    res = subprocess.run(cmd, env=env, cwd=ROOT, capture_output=True, text=True, timeout=3000)
    tail = res.stdout[-4000:] + res.stderr[-2000:]
    assert res.returncode == 0, tail
    assert " passed" in res.stdout and "SLOPE_ERR_BOUNDS" not in res.stdout, tail
