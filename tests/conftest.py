import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(autouse=True)
def _debug_bounds_clean(request):
    """When the suite runs against the debug build (KVZIP_EXPECT_DEBUG set, see
    test_gpu_debug_build.py), every GPU test must leave no failed bounds check."""
    yield
    if os.environ.get("KVZIP_EXPECT_DEBUG") and "gpu" in request.keywords:
        from attention_score_reduction_b200 import kvzip
        lib = kvzip.library()
        assert lib.kvzip_debug_checks() == 1, "expected the debug build"
        assert lib.kvzip_debug_bounds_status() == kvzip.OK, "a device bounds check failed"


def pytest_collection_modifyitems(config, items):
    # GPU tests need CUDA; on a CPU-only machine they are skipped, not failed,
    # when someone runs the whole suite without a marker filter.
    try:
        import torch
        has_cuda = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_cuda = False
    if has_cuda:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
