"""The Python binding's own checks, which run before any library call: tensors
must be CUDA tensors of the documented dtype, required arguments present, and
the segment table packs into the C struct as given."""
import ctypes

import pytest
import torch

from w8a8_gemm_b200 import binding as B


def test_cpu_tensors_and_missing_arguments_are_rejected():
    x = torch.zeros(4, 32, dtype=torch.bfloat16)
    s = torch.zeros(1, 1, 2)
    planes = torch.zeros(1, 2, 4, 32, dtype=torch.int8)
    with pytest.raises(ValueError, match="CUDA"):
        B.sq_quantize_act(x, None, s, B.Segments(), planes)
    with pytest.raises(ValueError, match="required"):
        B._need(None, torch.float32, "s_act")
    B._need(None, torch.float32, "bias", optional=True)   # optional may be absent
    wq = torch.zeros(8, 32, dtype=torch.int8)
    with pytest.raises(ValueError, match="CUDA"):
        B.sq_dualscale_seglinear_gemm_gelu_quant(planes, wq, torch.zeros(1, 8), s, None,
                                                 B.Segments(), torch.zeros(2),
                                                 torch.zeros(1, 2, 4, 8, dtype=torch.int8))


def test_segment_table_packing():
    seg = B.Segments(B.SQ_SEG_INPUT, [0, 32, 96], 1, B.SQ_FLAG_SINGLE_SCALE)
    assert seg.P == 1
    c, keep = seg._c()
    assert (c.mode, c.n_seg, c.n_groups, c.flags) == (B.SQ_SEG_INPUT, 2, 1,
                                                       B.SQ_FLAG_SINGLE_SCALE)
    offs = ctypes.cast(c.offsets, ctypes.POINTER(ctypes.c_int32))
    assert [offs[i] for i in range(3)] == [0, 32, 96]
    assert B.Segments().P == 2 and B.Segments()._c()[0].n_seg == 1


def test_every_exported_name_has_a_wrapper_or_is_internal():
    wrapped = {n for n in B.EXPORTED if hasattr(B, n)}
    internal = {"sq_status_string", "sq_host_pipeline_workspace_bytes",
                "sq_host_pipeline_create", "sq_host_pipeline_destroy",
                # reached through sq_dualscale_seglinear_gemm / sq_debug_gemm_s32
                # with workspace=, and through gemm_workspace()
                "sq_dualscale_seglinear_gemm_ws", "sq_debug_gemm_s32_ws",
                "sq_gemm_workspace_bytes",
                # reached through sq_quantize_act(..., plan=)
                "sq_quantize_act_planned"}
    assert set(B.EXPORTED) - wrapped <= internal
