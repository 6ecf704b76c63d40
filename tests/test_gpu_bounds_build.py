"""GPU: the bounds-checked build runs the parity cases clean.

compute-sanitizer is not available here. In its place the library is built a
second time with SS_BOUNDS_CHECK=1: its kernels check the indices they compute
(candidate and target positions, the overflow row list, TMEM columns, the
dW scatter row, TMA box alignment) before each guarded access and record
SS_ERR_BAD_INDEX (detail 200 + site) in dev_status[8..9] instead of touching
memory out of range. This runs the small, edge and extreme-loss parity cases
and the headline-size builder through that build, in a child process that
loads it (SAMPLED_CE_LIB); every case also checks dev_status[8] == 0.
"""

import os
import subprocess
import sys

import pytest

from sampled_softmax_cross_b200 import build_lib

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_cases_pass_on_the_bounds_checked_build():
    lib = build_lib.build(bounds_check=True)
    env = dict(os.environ, SAMPLED_CE_LIB=lib)
    sel = ("small_shapes or edge_shapes or tiny_workload or huge_loss or all_ignored or "
           "empty_microbatch or builder_bit_exact or builder_edge")
    out = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-k", sel,
                          "-p", "no:cacheprovider", "tests/test_gpu_parity.py"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-2000:]
    assert " passed" in out.stdout and "failed" not in out.stdout
