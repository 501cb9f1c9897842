"""The parity suites again, on the build with device bounds checks.

libkvzip_debug.so (``build.build(debug=True)``) tests every computed index of
the compaction, selection, scorer normaliser / score-update and decode kernels
against its buffer before the access, and records a failure instead of
faulting.  This runs the GPU parity, decode, variant, sharded-selection and
allocation-free tests in a fresh interpreter that loads the debug build
(KVZIP_LIBRARY); the conftest then checks after every test that no bounds
check failed.  The inputs are the ordinary valid ones: nothing is made to
fault.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_parity.py", "tests/test_gpu_decode.py", "tests/test_gpu_variants.py",
          "tests/test_gpu_context.py",
          "tests/test_gpu_sharded.py::test_shard_protocol_matches_global_selection",
          "tests/test_zz_no_alloc.py"]


def test_parity_suites_pass_on_debug_build_with_clean_bounds():
    from attention_score_reduction_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, KVZIP_LIBRARY=lib, KVZIP_EXPECT_DEBUG="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        *SUITES], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
