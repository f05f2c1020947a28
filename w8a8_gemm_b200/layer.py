"""Layer-level use of the library: one DualScale + SegLinear quantized linear.

Offline (once): quantize the weight segment-wise and calibrate s+ / s- on a
calibration slice -- both on the GPU through the C ABI.  Online (per call):
quantize the activation into the stacked planes, then run the fused GEMM.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class DualScaleSegLinear:
    """W8A8 DualScale linear with SegLinear segments.

    w      bf16 [N][K] nn.Linear weight (CUDA)
    bias   bf16 [N] or None
    d      fp32 [G][K] SmoothQuant divisor or None
    seg    binding.Segments
    x_cal  bf16 [rows][K] calibration activations
    weight_bits  8 (W8A8) or 4 (W4A8: weights kept packed, two codes per byte,
           and expanded into the int8 GEMM operand before every GEMM; several
           layers may share one operand buffer, `w_operand`, int8 [>= N*K])
    fp8    FP8 E4M3 codes for activations and weights (SQ_FLAG_FP8) instead of int8
    workspace  optional uint8 CUDA tensor from binding.gemm_workspace(): the GEMM
           then balances its last wave of tiles over all SMs (same results); layers
           run one after another on one stream may share one
    """

    def __init__(self, w: torch.Tensor, bias: Optional[torch.Tensor], d: Optional[torch.Tensor],
                 seg: B.Segments, x_cal: torch.Tensor, out_dtype=torch.bfloat16,
                 adaptive: bool = False, asymmetry_threshold: float = 2.0,
                 weight_bits: int = 8, w_operand: Optional[torch.Tensor] = None,
                 fp8: bool = False, workspace: Optional[torch.Tensor] = None):
        if weight_bits not in (8, 4):
            raise ValueError("weight_bits must be 8 or 4")
        if fp8 and weight_bits == 4:
            raise ValueError("FP8 codes and W4 weights do not combine")
        self.N, self.K = w.shape
        self.weight_bits = weight_bits
        self.workspace = workspace
        self.fp8 = fp8
        if weight_bits == 4:
            seg = B.Segments(seg.mode, seg.offsets, seg.n_groups, seg.flags | B.SQ_FLAG_W4)
        if fp8:
            seg = B.Segments(seg.mode, seg.offsets, seg.n_groups, seg.flags | B.SQ_FLAG_FP8)
        self.seg = seg
        self.G, self.S = seg.n_groups, seg.S
        self.d = d
        self.bias = bias
        self.out_dtype = out_dtype
        dev = w.device
        self.s_w = torch.empty(self.S, self.N, dtype=torch.float32, device=dev)
        if weight_bits == 4:
            self.wq4 = torch.empty(self.N, self.K // 2, dtype=torch.uint8, device=dev)
            B.sq_quantize_weight_w4(w, d, seg, self.wq4, self.s_w)
            if w_operand is None:
                w_operand = torch.empty(self.N * self.K, dtype=torch.int8, device=dev)
            if w_operand.numel() < self.N * self.K or w_operand.dtype != torch.int8:
                raise ValueError("w_operand must be int8 with at least N*K elements")
            self.wq = w_operand.view(-1)[: self.N * self.K].view(self.N, self.K)
        else:
            self.wq4 = None
            self.wq = torch.empty(self.N, self.K, dtype=torch.int8, device=dev)
            B.sq_quantize_weight_seg(w, d, seg, self.wq, self.s_w)
        self.s_act = torch.empty(self.G, self.S, 2, dtype=torch.float32, device=dev)
        B.sq_calibrate_act(x_cal, d, seg, self.s_act)
        if adaptive and not seg.flags & B.SQ_FLAG_SINGLE_SCALE:
            # Adaptive DualScale (the library's policy call): keep the two steps
            # only where the calibrated sides differ by at least
            # `asymmetry_threshold` in some group and K-segment; otherwise
            # switch the layer to one symmetric step.
            if B.sq_choose_single_scale(self.s_act, fp8=fp8, threshold=asymmetry_threshold):
                self.seg = B.Segments(seg.mode, seg.offsets, seg.n_groups,
                                      seg.flags | B.SQ_FLAG_SINGLE_SCALE)
                B.sq_calibrate_act(x_cal, d, self.seg, self.s_act)
        self.single_scale = bool(self.seg.flags & B.SQ_FLAG_SINGLE_SCALE)
        # With SmoothQuant divisors: the channels whose codes may skip both
        # quotient corrections (same codes; sq_quantize_act_plan).
        self.plan = (B.sq_quantize_act_plan(d, self.s_act, self.seg)
                     if d is not None and not fp8 else None)
        self._planes = None

    def planes_for(self, M: int, device) -> torch.Tensor:
        if self._planes is None or self._planes.shape[2] != M:
            self._planes = torch.empty(self.G, self.seg.P, M, self.K, dtype=torch.int8,
                                       device=device)
        return self._planes

    def quantize(self, x: torch.Tensor, planes: Optional[torch.Tensor] = None) -> torch.Tensor:
        if planes is None:
            planes = self.planes_for(x.shape[0], x.device)
        return B.sq_quantize_act(x, self.d, self.s_act, self.seg, planes, plan=self.plan)

    def gemm(self, planes: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        M = planes.shape[2]
        if y is None:
            y = torch.empty(M, self.N, dtype=self.out_dtype, device=planes.device)
        if self.wq4 is not None:
            B.sq_unpack_weight_w4(self.wq4, self.wq)
        return B.sq_dualscale_seglinear_gemm(planes, self.wq, self.s_w, self.s_act, self.bias,
                                             y, self.seg, workspace=self.workspace)

    def gemm_gelu_quant(self, planes: torch.Tensor, nxt: "DualScaleSegLinear",
                        planes_next: Optional[torch.Tensor] = None) -> torch.Tensor:
        """This layer's GEMM fused with the next layer's input: returns nxt's
        activation planes of bf16(gelu(bf16(y))) (an FFN's fc1 feeding fc2),
        computed in this GEMM's epilogue with nxt's calibrated steps.  This
        layer: one K-segment; nxt: one group and K-segment, no divisor."""
        if nxt.d is not None or nxt.seg.mode != B.SQ_SEG_NONE:
            raise ValueError("the next layer must have one segment and no SmoothQuant divisor")
        M = planes.shape[2]
        if planes_next is None:
            planes_next = torch.empty(1, nxt.seg.P, M, nxt.K, dtype=torch.int8,
                                      device=planes.device)
        if self.wq4 is not None:
            B.sq_unpack_weight_w4(self.wq4, self.wq)
        return B.sq_dualscale_seglinear_gemm_gelu_quant(planes, self.wq, self.s_w, self.s_act,
                                                        self.bias, self.seg,
                                                        nxt.s_act.reshape(2), planes_next,
                                                        single_next=nxt.seg.P == 1)

    def __call__(self, x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        return self.gemm(self.quantize(x), y)
