"""Thin Python binding of libsegquant.so: the same entry points as
include/segquant.h, taking torch tensors.  Argument marshalling only -- every
step of the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback.  A missing library raises at the first call.

All tensors must be CUDA tensors on the current device; calls are enqueued on
torch's current CUDA stream.  Every call raises SegQuantError unless the
library returned SQ_OK.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

# The library: the release build, or another build of it named by the
# environment variable SQ_LIBRARY (the test suite runs some cases against the
# bounds-checked debug build, libsegquant_debug.so).
LIB_PATH = os.environ.get("SQ_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libsegquant.so")

SQ_OK = 0
SQ_ERR_UNSUPPORTED = -2
SQ_SEG_NONE, SQ_SEG_OUTPUT, SQ_SEG_INPUT = 0, 1, 2
SQ_OUT_BF16, SQ_OUT_F32 = 0, 1
SQ_MAX_SEGMENTS = 64
SQ_FLAG_SINGLE_SCALE = 1
SQ_FLAG_W4 = 2
SQ_FLAG_FP8 = 4

EXPORTED = ("sq_calibrate_act", "sq_quantize_act", "sq_quantize_weight_seg",
            "sq_quantize_weight_w4", "sq_unpack_weight_w4",
            "sq_dualscale_seglinear_gemm", "sq_dualscale_seglinear_gemm_gelu_quant",
            "sq_debug_gemm_s32", "sq_get_device_status",
            "sq_status_string", "sq_version", "sq_debug_timeout_probe",
            "sq_host_pipeline_workspace_bytes", "sq_host_pipeline_create",
            "sq_host_pipeline_destroy", "sq_dualscale_seglinear_host",
            "sq_dualscale_seglinear_host_noalloc", "sq_choose_single_scale",
            "sq_dualscale_seglinear_gemm_ws", "sq_gemm_workspace_bytes", "sq_debug_gemm_s32_ws",
            "sq_debug_bounds_checks", "sq_debug_bounds_probe",
            "sq_quantize_act_plan", "sq_quantize_act_planned")
SQ_ERR_DEVICE_BOUNDS = -9
SQ_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class SegQuantError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


class _Segments(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("n_seg", ctypes.c_int32),
                ("offsets", ctypes.POINTER(ctypes.c_int32)), ("n_groups", ctypes.c_int32),
                ("flags", ctypes.c_int32)]


@dataclass
class Segments:
    """SegLinear segment table: mode, boundaries (over N for output mode, over
    K for input mode), the number of activation groups G, and flags
    (SQ_FLAG_SINGLE_SCALE for the single-scale path, SQ_FLAG_W4 for a GEMM whose
    weight operand comes from sq_unpack_weight_w4, SQ_FLAG_FP8 for E4M3 codes in
    the int8 buffers)."""
    mode: int = SQ_SEG_NONE
    offsets: Optional[Sequence[int]] = None
    n_groups: int = 1
    flags: int = 0

    @property
    def P(self) -> int:
        """Activation planes per group: 2 (X^+, X^-), or 1 in single-scale mode."""
        return 1 if self.flags & SQ_FLAG_SINGLE_SCALE else 2

    @property
    def n_seg(self) -> int:
        return 1 if self.offsets is None else len(self.offsets) - 1

    @property
    def S(self) -> int:
        return self.n_seg if self.mode == SQ_SEG_INPUT else 1

    def _c(self):
        if self.offsets is None:
            arr = None
            ptr = ctypes.POINTER(ctypes.c_int32)()
        else:
            arr = (ctypes.c_int32 * len(self.offsets))(*[int(v) for v in self.offsets])
            ptr = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
        s = _Segments(self.mode, self.n_seg, ptr, self.n_groups, self.flags)
        return s, arr  # keep the array alive for the call


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsegquant.so (built in-tree by w8a8_gemm_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m w8a8_gemm_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        p, i64 = ctypes.c_void_p, ctypes.c_int64
        seg = ctypes.POINTER(_Segments)
        L.sq_calibrate_act.argtypes = [p, i64, i64, i64, p, seg, p, p]
        L.sq_quantize_act.argtypes = [p, i64, i64, i64, p, p, seg, p, p]
        L.sq_quantize_act_plan.argtypes = [p, i64, p, seg, p, p]
        L.sq_quantize_act_planned.argtypes = [p, i64, i64, i64, p, p, seg, p, p, p]
        L.sq_quantize_weight_seg.argtypes = [p, i64, i64, p, seg, p, p, p]
        L.sq_quantize_weight_w4.argtypes = [p, i64, i64, p, seg, p, p, p]
        L.sq_unpack_weight_w4.argtypes = [p, i64, i64, p, p]
        L.sq_dualscale_seglinear_gemm.argtypes = [p, p, p, p, p, p, ctypes.c_int, i64, i64, i64,
                                                  i64, seg, p]
        L.sq_dualscale_seglinear_gemm_gelu_quant.argtypes = [p, p, p, p, p, i64, i64, i64, seg,
                                                             p, ctypes.c_int32, p, p]
        L.sq_debug_gemm_s32.argtypes = [p, p, i64, i64, i64, seg, p, p]
        L.sq_debug_gemm_s32_ws.argtypes = [p, p, i64, i64, i64, seg, p, p, ctypes.c_size_t, p]
        L.sq_dualscale_seglinear_gemm_ws.argtypes = [p, p, p, p, p, p, ctypes.c_int, i64, i64,
                                                     i64, i64, seg, p, ctypes.c_size_t, p]
        L.sq_gemm_workspace_bytes.argtypes = []
        L.sq_gemm_workspace_bytes.restype = ctypes.c_size_t
        L.sq_get_device_status.argtypes = [p]
        L.sq_choose_single_scale.argtypes = [p, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                             ctypes.POINTER(ctypes.c_int32)]
        L.sq_debug_timeout_probe.argtypes = [ctypes.c_uint32, p]
        L.sq_debug_bounds_checks.argtypes = []
        L.sq_debug_bounds_probe.argtypes = [p, i64, p]
        L.sq_host_pipeline_workspace_bytes.argtypes = [i64, i64, i64, ctypes.c_int32,
                                                       ctypes.c_int32]
        L.sq_host_pipeline_workspace_bytes.restype = ctypes.c_size_t
        L.sq_host_pipeline_create.argtypes = [i64, i64, i64, ctypes.c_int32, ctypes.c_int32, p,
                                              ctypes.c_size_t, ctypes.POINTER(p)]
        L.sq_host_pipeline_destroy.argtypes = [p]
        L.sq_dualscale_seglinear_host.argtypes = [p, p, i64, i64, i64, p, p, p, p, p, p,
                                                  ctypes.c_int, i64, i64, seg, p]
        L.sq_dualscale_seglinear_host_noalloc.argtypes = [p, i64, i64, i64, p, p, p, p, p, p,
                                                          ctypes.c_int, i64, i64, seg, p]
        L.sq_status_string.argtypes = [ctypes.c_int]
        L.sq_status_string.restype = ctypes.c_char_p
        L.sq_version.argtypes = []
        for f in (L.sq_calibrate_act, L.sq_quantize_act, L.sq_quantize_weight_seg,
                  L.sq_quantize_weight_w4, L.sq_unpack_weight_w4, L.sq_host_pipeline_create,
                  L.sq_host_pipeline_destroy, L.sq_dualscale_seglinear_host,
                  L.sq_dualscale_seglinear_host_noalloc,
                  L.sq_dualscale_seglinear_gemm, L.sq_dualscale_seglinear_gemm_gelu_quant,
                  L.sq_debug_gemm_s32, L.sq_get_device_status, L.sq_choose_single_scale,
                  L.sq_dualscale_seglinear_gemm_ws, L.sq_debug_gemm_s32_ws,
                  L.sq_version, L.sq_debug_timeout_probe, L.sq_debug_bounds_checks,
                  L.sq_debug_bounds_probe, L.sq_quantize_act_plan, L.sq_quantize_act_planned):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().sq_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != SQ_OK:
        raise SegQuantError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: Optional[torch.Tensor], dtype, name: str, optional=False):
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _rows(x: torch.Tensor):
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return x.shape[0], x.shape[1], x.stride(0)


# --------------------------------------------------------------------- calls
def sq_calibrate_act(x: torch.Tensor, d: Optional[torch.Tensor], seg: Segments,
                     s_act: torch.Tensor) -> torch.Tensor:
    """AMax calibration into s_act fp32 [G][S][2]."""
    _need(x, torch.bfloat16, "x")
    _need(d, torch.float32, "d", optional=True)
    _need(s_act, torch.float32, "s_act")
    M, K, ldx = _rows(x)
    cs, keep = seg._c()
    _check(lib().sq_calibrate_act(_ptr(x), M, K, ldx, _ptr(d), ctypes.byref(cs), _ptr(s_act),
                                  _stream()), "sq_calibrate_act")
    return s_act


def sq_quantize_act(x: torch.Tensor, d: Optional[torch.Tensor], s_act: torch.Tensor,
                    seg: Segments, planes: torch.Tensor,
                    plan: Optional[torch.Tensor] = None) -> torch.Tensor:
    """DualScale quantization of X / d into planes int8 [G][P][M][K]; with a
    plan from sq_quantize_act_plan (same d, s_act, seg), sq_quantize_act_planned."""
    _need(x, torch.bfloat16, "x")
    _need(d, torch.float32, "d", optional=True)
    _need(s_act, torch.float32, "s_act")
    _need(planes, torch.int8, "planes")
    _need(plan, torch.int32, "plan", optional=True)
    M, K, ldx = _rows(x)
    if tuple(planes.shape) != (seg.n_groups, seg.P, M, K) or not planes.is_contiguous():
        raise ValueError(f"planes must be contiguous [{seg.n_groups}, {seg.P}, {M}, {K}]")
    cs, keep = seg._c()
    if plan is None:
        _check(lib().sq_quantize_act(_ptr(x), M, K, ldx, _ptr(d), _ptr(s_act), ctypes.byref(cs),
                                     _ptr(planes), _stream()), "sq_quantize_act")
    else:
        _check(lib().sq_quantize_act_planned(_ptr(x), M, K, ldx, _ptr(d), _ptr(s_act),
                                             ctypes.byref(cs), _ptr(plan), _ptr(planes),
                                             _stream()), "sq_quantize_act_planned")
    return planes


def sq_quantize_act_plan(d: torch.Tensor, s_act: torch.Tensor, seg: Segments,
                         plan: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per (group, channel) bits [G][ceil(K/32)] (int32 storage of the uint32
    words): channels whose codes may skip both quotient corrections."""
    _need(d, torch.float32, "d")
    _need(s_act, torch.float32, "s_act")
    K = d.shape[-1]
    words = (K + 31) // 32
    if plan is None:
        plan = torch.empty(seg.n_groups, words, dtype=torch.int32, device=d.device)
    _need(plan, torch.int32, "plan")
    if tuple(plan.shape) != (seg.n_groups, words) or not plan.is_contiguous():
        raise ValueError(f"plan must be contiguous int32 [{seg.n_groups}, {words}]")
    cs, keep = seg._c()
    _check(lib().sq_quantize_act_plan(_ptr(d), K, _ptr(s_act), ctypes.byref(cs), _ptr(plan),
                                      _stream()), "sq_quantize_act_plan")
    return plan


def sq_quantize_weight_seg(w: torch.Tensor, d: Optional[torch.Tensor], seg: Segments,
                           wq: torch.Tensor, s_w: torch.Tensor):
    """Segment-wise AMax weight quantization: wq int8 [N][K], s_w fp32 [S][N]."""
    _need(w, torch.bfloat16, "w")
    _need(d, torch.float32, "d", optional=True)
    _need(wq, torch.int8, "wq")
    _need(s_w, torch.float32, "s_w")
    if not (w.is_contiguous() and wq.is_contiguous() and s_w.is_contiguous()):
        raise ValueError("w, wq and s_w must be contiguous")
    N, K = w.shape
    cs, keep = seg._c()
    _check(lib().sq_quantize_weight_seg(_ptr(w), N, K, _ptr(d), ctypes.byref(cs), _ptr(wq),
                                        _ptr(s_w), _stream()), "sq_quantize_weight_seg")
    return wq, s_w


def sq_quantize_weight_w4(w: torch.Tensor, d: Optional[torch.Tensor], seg: Segments,
                          wq4: torch.Tensor, s_w: torch.Tensor):
    """W4A8 weight quantization: packed codes wq4 uint8 [N][K/2], s_w fp32 [S][N]."""
    _need(w, torch.bfloat16, "w")
    _need(d, torch.float32, "d", optional=True)
    _need(wq4, torch.uint8, "wq4")
    _need(s_w, torch.float32, "s_w")
    N, K = w.shape
    if not (w.is_contiguous() and wq4.is_contiguous() and s_w.is_contiguous()):
        raise ValueError("w, wq4 and s_w must be contiguous")
    if tuple(wq4.shape) != (N, K // 2):
        raise ValueError(f"wq4 must be [{N}, {K // 2}]")
    cs, keep = seg._c()
    _check(lib().sq_quantize_weight_w4(_ptr(w), N, K, _ptr(d), ctypes.byref(cs), _ptr(wq4),
                                       _ptr(s_w), _stream()), "sq_quantize_weight_w4")
    return wq4, s_w


def sq_unpack_weight_w4(wq4: torch.Tensor, wq: torch.Tensor) -> torch.Tensor:
    """Packed W4 codes -> the int8 GEMM operand wq [N][K] = 16 q."""
    _need(wq4, torch.uint8, "wq4")
    _need(wq, torch.int8, "wq")
    N, K = wq.shape
    if tuple(wq4.shape) != (N, K // 2) or not (wq4.is_contiguous() and wq.is_contiguous()):
        raise ValueError(f"wq4 must be contiguous [{N}, {K // 2}] and wq contiguous [{N}, {K}]")
    _check(lib().sq_unpack_weight_w4(_ptr(wq4), N, K, _ptr(wq), _stream()),
           "sq_unpack_weight_w4")
    return wq


def gemm_workspace(device=None) -> torch.Tensor:
    """A zero-filled workspace for sq_dualscale_seglinear_gemm_ws /
    sq_debug_gemm_s32_ws on the current device (reuse it for every call on one
    stream)."""
    nbytes = lib().sq_gemm_workspace_bytes()
    if nbytes == 0:
        raise SegQuantError(-7, "sq_gemm_workspace_bytes")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or torch.device("cuda"))


def sq_dualscale_seglinear_gemm(planes: torch.Tensor, wq: torch.Tensor, s_w: torch.Tensor,
                                s_act: torch.Tensor, bias: Optional[torch.Tensor],
                                y: torch.Tensor, seg: Segments,
                                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = sum_i s_w (s+ X^+_i W^_i + s- X^-_i W^_i) + bias into y (bf16 or fp32 [M][N]).
    With `workspace` (gemm_workspace()), the _ws entry point balances the last
    wave of tiles; the result is the same bit for bit."""
    _need(planes, torch.int8, "planes")
    _need(wq, torch.int8, "wq")
    _need(s_w, torch.float32, "s_w")
    _need(s_act, torch.float32, "s_act")
    _need(bias, torch.bfloat16, "bias", optional=True)
    if y.dtype not in (torch.bfloat16, torch.float32) or not y.is_cuda:
        raise ValueError("y must be a CUDA bf16 or fp32 tensor")
    G, P, M, K = planes.shape
    N = wq.shape[0]
    if P != seg.P or wq.shape[1] != K or y.shape[0] != M or y.shape[1] != N or y.stride(1) != 1:
        raise ValueError("shape mismatch between planes [G,P,M,K], wq [N,K] and y [M,N]")
    out = SQ_OUT_BF16 if y.dtype == torch.bfloat16 else SQ_OUT_F32
    cs, keep = seg._c()
    if workspace is None:
        _check(lib().sq_dualscale_seglinear_gemm(_ptr(planes), _ptr(wq), _ptr(s_w), _ptr(s_act),
                                                 _ptr(bias), _ptr(y), out, M, N, K, y.stride(0),
                                                 ctypes.byref(cs), _stream()),
               "sq_dualscale_seglinear_gemm")
    else:
        _need(workspace, torch.uint8, "workspace")
        _check(lib().sq_dualscale_seglinear_gemm_ws(_ptr(planes), _ptr(wq), _ptr(s_w),
                                                    _ptr(s_act), _ptr(bias), _ptr(y), out, M, N,
                                                    K, y.stride(0), ctypes.byref(cs),
                                                    _ptr(workspace), workspace.numel(),
                                                    _stream()),
               "sq_dualscale_seglinear_gemm_ws")
    return y


def sq_dualscale_seglinear_gemm_gelu_quant(planes: torch.Tensor, wq: torch.Tensor,
                                           s_w: torch.Tensor, s_act: torch.Tensor,
                                           bias: Optional[torch.Tensor], seg: Segments,
                                           s_act_next: torch.Tensor, planes_next: torch.Tensor,
                                           single_next: bool = False) -> torch.Tensor:
    """The fused producer: the next layer's planes of bf16(gelu(bf16(y))) into
    planes_next (int8 [1][P'][M][N], P' = 2, or 1 with single_next), with its
    steps s_act_next (fp32 [2] = {s+, s-}).  This layer: one K-segment."""
    _need(planes, torch.int8, "planes")
    _need(wq, torch.int8, "wq")
    _need(s_w, torch.float32, "s_w")
    _need(s_act, torch.float32, "s_act")
    _need(bias, torch.bfloat16, "bias", optional=True)
    _need(s_act_next, torch.float32, "s_act_next")
    _need(planes_next, torch.int8, "planes_next")
    G, P, M, K = planes.shape
    N = wq.shape[0]
    pn = 1 if single_next else 2
    if (P != seg.P or wq.shape[1] != K or s_act_next.numel() != 2
            or tuple(planes_next.shape) != (1, pn, M, N) or not planes_next.is_contiguous()):
        raise ValueError("shape mismatch between planes [G,P,M,K], wq [N,K] and "
                         "planes_next [1,P',M,N]")
    cs, keep = seg._c()
    _check(lib().sq_dualscale_seglinear_gemm_gelu_quant(
        _ptr(planes), _ptr(wq), _ptr(s_w), _ptr(s_act), _ptr(bias), M, N, K, ctypes.byref(cs),
        _ptr(s_act_next), SQ_FLAG_SINGLE_SCALE if single_next else 0, _ptr(planes_next),
        _stream()), "sq_dualscale_seglinear_gemm_gelu_quant")
    return planes_next


def sq_debug_gemm_s32(planes: torch.Tensor, wq: torch.Tensor, seg: Segments,
                      acc: torch.Tensor, workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Raw int32 accumulators [S][P][M][N] of the same tensor-core kernel (with
    `workspace`: the balanced last wave of sq_debug_gemm_s32_ws)."""
    _need(planes, torch.int8, "planes")
    _need(wq, torch.int8, "wq")
    _need(acc, torch.int32, "acc")
    G, P, M, K = planes.shape
    N = wq.shape[0]
    if tuple(acc.shape) != (seg.S, seg.P, M, N) or not acc.is_contiguous():
        raise ValueError(f"acc must be contiguous [{seg.S}, {seg.P}, {M}, {N}]")
    cs, keep = seg._c()
    if workspace is None:
        _check(lib().sq_debug_gemm_s32(_ptr(planes), _ptr(wq), M, N, K, ctypes.byref(cs),
                                       _ptr(acc), _stream()), "sq_debug_gemm_s32")
    else:
        _need(workspace, torch.uint8, "workspace")
        _check(lib().sq_debug_gemm_s32_ws(_ptr(planes), _ptr(wq), M, N, K, ctypes.byref(cs),
                                          _ptr(acc), _ptr(workspace), workspace.numel(),
                                          _stream()), "sq_debug_gemm_s32_ws")
    return acc


class HostPipeline:
    """Streams, events and a device workspace (a torch tensor this object owns)
    for sq_dualscale_seglinear_host: layers with K <= max_K, N <= max_N,
    G <= max_G, P <= max_P, in chunks of chunk_rows rows."""

    def __init__(self, chunk_rows: int, max_K: int, max_N: int, max_G: int = 1, max_P: int = 2,
                 device=None):
        L = lib()
        nbytes = L.sq_host_pipeline_workspace_bytes(chunk_rows, max_K, max_N, max_G, max_P)
        if nbytes == 0:
            raise ValueError("invalid pipeline sizes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8,
                                     device=device or torch.device("cuda"))
        self._h = ctypes.c_void_p()
        _check(L.sq_host_pipeline_create(chunk_rows, max_K, max_N, max_G, max_P,
                                         _ptr(self.workspace), nbytes, ctypes.byref(self._h)),
               "sq_host_pipeline_create")

    def close(self):
        if self._h:
            _check(lib().sq_host_pipeline_destroy(self._h), "sq_host_pipeline_destroy")
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def sq_dualscale_seglinear_host(pl: HostPipeline, x_host: torch.Tensor, d: Optional[torch.Tensor],
                                s_act: torch.Tensor, wq: torch.Tensor, s_w: torch.Tensor,
                                bias: Optional[torch.Tensor], y_host: torch.Tensor,
                                seg: Segments) -> torch.Tensor:
    """One layer from host rows x_host (bf16 [M][K], CPU, pinned for overlap)
    to host rows y_host (bf16 or fp32 [M][N], CPU) through the pipeline; the
    weights and scales are CUDA tensors.  Ordered on torch's current stream."""
    if x_host.is_cuda or y_host.is_cuda:
        raise ValueError("x_host and y_host must be CPU tensors")
    if x_host.dtype != torch.bfloat16 or y_host.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("x_host must be bf16 and y_host bf16 or fp32")
    _need(d, torch.float32, "d", optional=True)
    _need(s_act, torch.float32, "s_act")
    _need(wq, torch.int8, "wq")
    _need(s_w, torch.float32, "s_w")
    _need(bias, torch.bfloat16, "bias", optional=True)
    M, K, ldx = _rows(x_host)
    N = wq.shape[0]
    if wq.shape[1] != K or y_host.shape[0] != M or y_host.shape[1] != N or y_host.stride(1) != 1:
        raise ValueError("shape mismatch between x_host [M,K], wq [N,K] and y_host [M,N]")
    out = SQ_OUT_BF16 if y_host.dtype == torch.bfloat16 else SQ_OUT_F32
    cs, keep = seg._c()
    _check(lib().sq_dualscale_seglinear_host(pl._h, _ptr(x_host), M, K, ldx, _ptr(d), _ptr(s_act),
                                             _ptr(wq), _ptr(s_w), _ptr(bias), _ptr(y_host), out,
                                             N, y_host.stride(0), ctypes.byref(cs), _stream()),
           "sq_dualscale_seglinear_host")
    return y_host


def sq_dualscale_seglinear_host_noalloc(x_host: torch.Tensor, d: Optional[torch.Tensor],
                                        s_act: torch.Tensor, wq: torch.Tensor,
                                        s_w: torch.Tensor, bias: Optional[torch.Tensor],
                                        y_host: torch.Tensor, seg: Segments) -> torch.Tensor:
    """The layer of sq_dualscale_seglinear_host without a pipeline or a
    workspace: for callers that may not allocate device memory.  The library's
    fixed device scratch (SQ_NOALLOC_SCRATCH_BYTES) holds the chunks; every
    call on a device shares it, so calls must not overlap on the GPU.  Ordered
    on torch's current stream."""
    if x_host.is_cuda or y_host.is_cuda:
        raise ValueError("x_host and y_host must be CPU tensors")
    if x_host.dtype != torch.bfloat16 or y_host.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("x_host must be bf16 and y_host bf16 or fp32")
    _need(d, torch.float32, "d", optional=True)
    _need(s_act, torch.float32, "s_act")
    _need(wq, torch.int8, "wq")
    _need(s_w, torch.float32, "s_w")
    _need(bias, torch.bfloat16, "bias", optional=True)
    M, K, ldx = _rows(x_host)
    N = wq.shape[0]
    if wq.shape[1] != K or y_host.shape[0] != M or y_host.shape[1] != N or y_host.stride(1) != 1:
        raise ValueError("shape mismatch between x_host [M,K], wq [N,K] and y_host [M,N]")
    out = SQ_OUT_BF16 if y_host.dtype == torch.bfloat16 else SQ_OUT_F32
    cs, keep = seg._c()
    _check(lib().sq_dualscale_seglinear_host_noalloc(_ptr(x_host), M, K, ldx, _ptr(d),
                                                     _ptr(s_act), _ptr(wq), _ptr(s_w), _ptr(bias),
                                                     _ptr(y_host), out, N, y_host.stride(0),
                                                     ctypes.byref(cs), _stream()),
           "sq_dualscale_seglinear_host_noalloc")
    return y_host


def sq_get_device_status() -> int:
    """Wait for torch's current stream, then return (and clear) the device
    error word (one per device, shared by all streams and callers)."""
    return lib().sq_get_device_status(_stream())


def sq_choose_single_scale(s_act: torch.Tensor, fp8: bool = False,
                           threshold: float = 2.0) -> bool:
    """The adaptive DualScale policy on a layer's calibrated DualScale steps
    (fp32 [G][S][2], any device; copied to the host): True where every group
    and K-segment has its larger side below threshold times the smaller."""
    s = s_act.detach().to("cpu", torch.float32).contiguous()
    if s.dim() < 1 or s.shape[-1] != 2:
        raise ValueError("s_act must end in a dimension of 2 ({s+, s-})")
    out = ctypes.c_int32(0)
    _check(lib().sq_choose_single_scale(ctypes.c_void_p(s.data_ptr()), s.numel() // 2,
                                        SQ_FLAG_FP8 if fp8 else 0, float(threshold),
                                        ctypes.byref(out)), "sq_choose_single_scale")
    return bool(out.value)


def sq_debug_timeout_probe(limit_us: int) -> None:
    """Test only: a kernel whose bounded barrier wait runs out after limit_us;
    the timeout lands in the device error word (see sq_get_device_status)."""
    _check(lib().sq_debug_timeout_probe(int(limit_us), _stream()), "sq_debug_timeout_probe")


def sq_debug_bounds_checks() -> bool:
    """True if the loaded library is the bounds-checked debug build."""
    return lib().sq_debug_bounds_checks() == 1


def sq_debug_bounds_probe(buf: torch.Tensor, n: int) -> None:
    """Test only (debug build): one checked store to buf[n] while the check is
    told the buffer holds n elements; buf must hold n + 1 int32 (a guard).
    The debug build skips the store and records SQ_ERR_DEVICE_BOUNDS."""
    _need(buf, torch.int32, "buf")
    if buf.numel() < n + 1:
        raise ValueError("buf must hold n + 1 elements")
    _check(lib().sq_debug_bounds_probe(_ptr(buf), int(n), _stream()), "sq_debug_bounds_probe")


def sq_version() -> int:
    return lib().sq_version()
