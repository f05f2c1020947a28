"""Cases that only the bounds-checked debug build runs (tests/test_gpu_debug_build.py
starts them in a child process with SQ_LIBRARY naming libsegquant_debug.so, since
a process loads one build of the library)."""
import pytest
import torch

from w8a8_gemm_b200 import binding as B

pytestmark = pytest.mark.gpu


def test_the_debug_build_is_loaded():
    assert B.sq_debug_bounds_checks()


@pytest.mark.parametrize("n", [1, 37, 1 << 20])
def test_bounds_probe_is_reported_and_skipped(n):
    """A store one past the extent the check is given: skipped (the guard
    element keeps its value) and reported as SQ_ERR_DEVICE_BOUNDS; the next
    read finds the word clear again."""
    buf = torch.full((n + 1,), 7, dtype=torch.int32, device="cuda")
    B.sq_debug_bounds_probe(buf, n)
    assert B.sq_get_device_status() == B.SQ_ERR_DEVICE_BOUNDS
    assert int(buf[n]) == 7
    assert bool((buf == 7).all())
    assert B.sq_get_device_status() == B.SQ_OK
