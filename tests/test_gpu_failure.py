"""Failure reporting on the GPU without a fault: a kernel's bounded barrier
wait runs out on a barrier nothing signals, the kernel records the timeout in
the library's device error word and returns, and the context stays usable."""
import numpy as np
import pytest
import torch

from w8a8_gemm_b200 import binding as B

pytestmark = pytest.mark.gpu
SQ_ERR_DEVICE_TIMEOUT = -6


def test_bounded_wait_reports_timeout_and_context_survives():
    assert B.sq_get_device_status() == 0          # clean to start with
    B.sq_debug_timeout_probe(2000)                # 2 ms limit
    assert B.sq_get_device_status() == SQ_ERR_DEVICE_TIMEOUT
    assert B.sq_get_device_status() == 0          # reading clears it
    # the context still runs the real kernels
    x = torch.full((64, 32), 0.5, dtype=torch.bfloat16, device="cuda")
    s_act = torch.tensor([[[1 / 64, 1 / 512]]], device="cuda")
    planes = torch.empty(1, 2, 64, 32, dtype=torch.int8, device="cuda")
    B.sq_quantize_act(x, None, s_act, B.Segments(), planes)
    torch.cuda.synchronize()
    assert B.sq_get_device_status() == 0
    assert bool((planes[0, 0] == 32).all()) and bool((planes[0, 1] == 0).all())


def test_probe_rejects_bad_limits():
    with pytest.raises(B.SegQuantError):
        B.sq_debug_timeout_probe(0)
    with pytest.raises(B.SegQuantError):
        B.sq_debug_timeout_probe(10 ** 6)
