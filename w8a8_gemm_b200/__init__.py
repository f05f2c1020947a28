"""SegQuant DualScale + SegLinear W8A8 linear layer for NVIDIA B200 (sm_100a).

The computation lives in libsegquant.so (C ABI: include/segquant.h); this
package holds its build script, a thin ctypes binding with the same entry-point
names, a layer-level convenience wrapper, and the seeded synthetic workloads.
Importing the package never loads CUDA; the first library call does, and fails
loudly if the library has not been built.
"""
from .binding import (SQ_FLAG_FP8, SQ_FLAG_SINGLE_SCALE, SQ_FLAG_W4, SQ_OUT_BF16, SQ_OUT_F32,
                      SQ_SEG_INPUT, SQ_SEG_NONE, SQ_SEG_OUTPUT, HostPipeline, SegQuantError,
                      Segments, sq_calibrate_act, sq_choose_single_scale, sq_debug_gemm_s32, sq_dualscale_seglinear_gemm,
                      sq_dualscale_seglinear_gemm_gelu_quant, sq_dualscale_seglinear_host,
                      sq_dualscale_seglinear_host_noalloc, sq_get_device_status, sq_quantize_act,
                      sq_quantize_weight_seg, sq_quantize_weight_w4, sq_unpack_weight_w4,
                      sq_version)

__all__ = ["SQ_FLAG_FP8", "SQ_FLAG_SINGLE_SCALE", "SQ_FLAG_W4", "SQ_OUT_BF16", "SQ_OUT_F32",
           "SQ_SEG_INPUT", "SQ_SEG_NONE", "SQ_SEG_OUTPUT", "HostPipeline", "SegQuantError",
           "Segments", "sq_calibrate_act", "sq_choose_single_scale", "sq_debug_gemm_s32", "sq_dualscale_seglinear_gemm",
           "sq_dualscale_seglinear_gemm_gelu_quant", "sq_dualscale_seglinear_host",
           "sq_dualscale_seglinear_host_noalloc", "sq_get_device_status", "sq_quantize_act",
           "sq_quantize_weight_seg", "sq_quantize_weight_w4", "sq_unpack_weight_w4",
           "sq_version"]
