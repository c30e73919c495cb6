"""The checking build (libeplb_checks.so, -DEPLB_CHECKS): the kernels check
the indices they derive from data (permutation slots, candidate experts,
replica slots, table rows and columns) and report EPLB_ERR_INTERNAL instead
of touching memory outside a buffer.  A slice of the GPU parity suite runs
against it in a child process: every plan, redirect and count must still
equal the oracle's and no check may fire (the parity tests assert status 0)."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checking_library_reports_itself():
    from moe_expert_load_eplb_b200 import build, load_library
    assert load_library().eplb_checking_build() == 0
    if os.path.exists(build.CHECKS_LIB):
        import ctypes
        lib = ctypes.CDLL(build.CHECKS_LIB)
        assert lib.eplb_checking_build() == 1
        assert lib.eplb_abi_version() == load_library().eplb_abi_version()


@pytest.mark.gpu
def test_parity_slice_under_the_checking_build():
    from moe_expert_load_eplb_b200 import build
    build.build(checks=True)  # no-op when up to date
    env = dict(os.environ, EPLB_LIBRARY="checks")
    sel = ("rebalance_shapes or rebalance_fuzz or redirect_ragged or redirect_arbitrary or "
           "count_redirect_ragged or serve_step_matches_oracle or rebalance_global_policy or "
           "fused_quality_shapes or rebalance_on_counted_loads")
    res = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_parity.py"),
                          "-m", "gpu", "-q", "-x", "-k", sel, "-p", "no:cacheprovider"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = (res.stdout + res.stderr)[-3000:]
    assert res.returncode == 0, tail
    assert " passed" in res.stdout and " failed" not in res.stdout, tail
