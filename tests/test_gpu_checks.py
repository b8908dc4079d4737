"""The GPU suite against the range-checking library (libkvc_checks.so, built with KVC_CHECKS=1).

The binding loads one library per process, so the suite runs in a child pytest with
KVC_CHECKS=1: the odd-shape sweep (N one past a tile and below one tile, budgets
n_sink + window + 1 and N, windows 1 to 128, pool widths 1 to 13), every oracle parity
module and the full-size configurations.  Each test must pass its own oracle comparison
and, through the autouse fixture in conftest.py, end with the device error word clear, so
no index, coordinate or slot that a kernel formed left the extent of the buffer it
addresses.  compute-sanitizer is closed on the machines these tests target; this build
stands in for its bounds checking.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

MODULES = ["test_gpu_odd_shapes.py", "test_gpu_parity.py", "test_gpu_configs.py", "test_gpu_csm.py",
           "test_gpu_decode.py", "test_gpu_pivot_metrics.py", "test_gpu_sharded.py", "test_zz_no_alloc.py"]


def test_gpu_suite_under_range_checks():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    if os.environ.get("KVC_CHECKS") == "1":
        pytest.skip("already the checks run")
    from long_context_kv_kvc_b200 import build
    build.build(checks=True)
    env = dict(os.environ, KVC_CHECKS="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           *[os.path.join(HERE, m) for m in MODULES]]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=2400)
    tail = (r.stdout + r.stderr)[-6000:]
    print(tail)
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout
