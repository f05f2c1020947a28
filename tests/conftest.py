import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(autouse=True)
def _debug_build_bounds_report(request):
    """Under the bounds-checked debug build (SQ_LIBRARY=...libsegquant_debug.so),
    every GPU test must end with the device error word clear: a store that a
    kernel skipped as out of bounds fails the test even where the compared
    outputs do not show it."""
    yield
    if request.node.get_closest_marker("gpu") is None or not os.environ.get("SQ_LIBRARY"):
        return
    from w8a8_gemm_b200 import binding as B
    if B.sq_debug_bounds_checks():
        assert B.sq_get_device_status() == B.SQ_OK, "a kernel skipped an out-of-bounds store"
