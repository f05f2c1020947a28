"""Shared helpers of the parity tests: run one synthetic layer through the CUDA
path (C ABI via the binding) and through the CPU oracle, on the same seeded
inputs, and compare."""
import numpy as np
import torch

import oracle
from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import workloads as wl


def segments(layer: wl.Layer, single=False, weight_bits=8, fp8=False) -> B.Segments:
    flags = ((B.SQ_FLAG_SINGLE_SCALE if single else 0) | (B.SQ_FLAG_W4 if weight_bits == 4 else 0)
             | (B.SQ_FLAG_FP8 if fp8 else 0))
    if layer.mode == wl.MODE_NONE:
        return B.Segments(B.SQ_SEG_NONE, None, 1, flags)
    return B.Segments(layer.mode, list(layer.offsets), layer.G, flags)


def oracle_offsets(layer: wl.Layer):
    return None if layer.mode == wl.MODE_NONE else list(layer.offsets)


def gpu_run(layer: wl.Layer, out_dtype=torch.float32, with_bias=True, s32=False,
            single=False, weight_bits=8, fp8=False):
    """CUDA path: weight quantization, calibration, activation quantization and
    the fused GEMM, all through the library.  weight_bits=4: W4A8 weights,
    packed, then expanded into the GEMM operand (16 q); out["wq"] is then the
    packed uint8 [N][K/2] and out["wq16"] the operand.  fp8=True: E4M3 codes
    in the int8 buffers, and out["acc"] holds the fp32 sums' bit patterns."""
    dev = torch.device("cuda")
    seg = segments(layer, single, weight_bits, fp8)
    x = layer.x.to(dev)
    w = layer.w.to(dev)
    xc = layer.x_cal.to(dev)
    d = None if layer.d is None else layer.d.to(dev)
    bias = layer.bias.to(dev) if (with_bias and layer.bias is not None) else None
    M, K, N, G, S = layer.M, layer.K, layer.N, layer.G, layer.S
    s_w = torch.empty(S, N, dtype=torch.float32, device=dev)
    extra = {}
    if weight_bits == 4:
        wq4 = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
        B.sq_quantize_weight_w4(w, d, seg, wq4, s_w)
        wq = torch.empty(N, K, dtype=torch.int8, device=dev)
        B.sq_unpack_weight_w4(wq4, wq)
        extra = dict(wq=wq4, wq16=wq)
    else:
        wq = torch.empty(N, K, dtype=torch.int8, device=dev)
        B.sq_quantize_weight_seg(w, d, seg, wq, s_w)
    s_act = torch.empty(G, S, 2, dtype=torch.float32, device=dev)
    B.sq_calibrate_act(xc, d, seg, s_act)
    planes = torch.empty(G, seg.P, M, K, dtype=torch.int8, device=dev)
    B.sq_quantize_act(x, d, s_act, seg, planes)
    ldy = (N + 7) // 8 * 8   # rows start 16-byte aligned for either dtype
    y = torch.empty(M, ldy, dtype=out_dtype, device=dev)[:, :N]
    B.sq_dualscale_seglinear_gemm(planes, wq, s_w, s_act, bias, y, seg)
    out = dict(wq=wq, s_w=s_w, s_act=s_act, planes=planes, y=y)
    out.update(extra)
    if s32:
        acc = torch.empty(S, seg.P, M, N, dtype=torch.int32, device=dev)
        B.sq_debug_gemm_s32(planes, wq, seg, acc)
        out["acc"] = acc
    torch.cuda.synchronize()
    assert B.sq_get_device_status() == 0
    return out


def oracle_prep(layer: wl.Layer, single=False, weight_bits=8, fp8=False):
    """Oracle calibration and quantization of both operands (weight_bits=4:
    W4A8 codes in [-7, 7] in "wq" and their packed storage in "wq4"; fp8:
    E4M3 codes as uint8)."""
    off = oracle_offsets(layer)
    d = None if layer.d is None else layer.d.numpy()
    if fp8:
        s_act = oracle.calibrate_act_fp8(wl.bits(layer.x_cal), d, layer.mode, off, layer.G,
                                         layer.N, single)
        planes = oracle.quantize_act_fp8(wl.bits(layer.x), s_act, d, layer.mode, off, layer.G,
                                         layer.N, single)
        wq, s_w = oracle.quantize_weight_fp8(wl.bits(layer.w), d, layer.mode, off, layer.G)
        return dict(s_act=s_act, planes=planes, wq=wq, s_w=s_w, fp8=True)
    s_act = oracle.calibrate_act(wl.bits(layer.x_cal), d, layer.mode, off, layer.G, layer.N,
                                 single)
    planes = oracle.quantize_act(wl.bits(layer.x), s_act, d, layer.mode, off, layer.G, layer.N,
                                 single)
    wq, s_w = oracle.quantize_weight(wl.bits(layer.w), d, layer.mode, off, layer.G,
                                     bits=weight_bits)
    out = dict(s_act=s_act, planes=planes, wq=wq, s_w=s_w)
    if weight_bits == 4:
        out["wq4"] = oracle.pack_w4(wq)
    return out


def oracle_y(layer, prep, rows=None, with_bias=True, threads=None):
    bias = wl.bits(layer.bias) if (with_bias and layer.bias is not None) else None
    if prep.get("fp8"):
        return oracle.gemm_fp8(prep["planes"], prep["wq"], prep["s_w"], prep["s_act"], bias,
                               layer.mode, oracle_offsets(layer), rows=rows,
                               threads=threads or oracle.num_threads())
    return oracle.gemm(prep["planes"], prep["wq"], prep["s_w"], prep["s_act"], bias, layer.mode,
                       oracle_offsets(layer), rows=rows,
                       threads=threads or oracle.num_threads())


def oracle_acc(layer, prep, rows=None, threads=None):
    return oracle.gemm_s32(prep["planes"], prep["wq"], layer.mode, oracle_offsets(layer),
                           rows=rows, threads=threads or oracle.num_threads())


def rel_err_floor(y: np.ndarray, r: np.ndarray) -> float:
    """max |y - r| / (|r| + 1e-3 rms(r)): relative error with a floor near 0."""
    r = r.astype(np.float64)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    den = np.abs(r) + 1e-3 * rms + 1e-30
    return float(np.max(np.abs(y.astype(np.float64) - r) / den)) if r.size else 0.0


def bf16_ulp_diff(y_bf16: torch.Tensor, r_f32: np.ndarray) -> int:
    """Largest distance, in bf16 ulps, between y and RNE_bf16(r)."""
    ref = torch.from_numpy(np.ascontiguousarray(r_f32)).to(torch.bfloat16)
    a = y_bf16.cpu().view(torch.int16).to(torch.int32)
    b = ref.view(torch.int16).to(torch.int32)
    # map sign-magnitude bf16 bit patterns onto a monotone integer line
    a = torch.where(a < 0, -(a & 0x7FFF), a)
    b = torch.where(b < 0, -(b & 0x7FFF), b)
    return int((a - b).abs().max()) if a.numel() else 0


def bf16_close(y_bf16: torch.Tensor, r_f32: np.ndarray, tol: float = 1e-3) -> bool:
    """bf16 output check where the fp32 accumulation order is the tensor
    core's (FP8 products summed in fp32 inside the MMA): |y - r| <= ulp_bf16(r)
    + tol * (|r| + 1e-3 rms(r)), the fp32 criterion widened by one bf16 ulp."""
    r = r_f32.astype(np.float64)
    y = y_bf16.float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(r), 1e-38))) - 7)
    return bool(np.all(np.abs(y - r) <= ulp + tol * (np.abs(r) + 1e-3 * rms)))


def sample_rows(M: int, bm: int = 128, stride: int = 97):
    """Every row of the first and last 128-row tile plus a strided subsample."""
    rows = set(range(min(bm, M)))
    rows |= set(range(max(0, M - bm), M))
    rows |= set(range(0, M, stride))
    return np.array(sorted(rows), dtype=np.int64)


def oracle_acc_fp8(layer, prep, rows=None, threads=None, absolute=False):
    """FP8: the exact sums of E4M3 products rounded once to fp32; with
    absolute=True the sums of |products| (sign bits cleared), which bound the
    rounding error of any fp32 summation order."""
    planes, wq = prep["planes"], prep["wq"]
    if absolute:
        planes, wq = planes & 0x7F, wq & 0x7F
    return oracle.gemm_fp8_acc(planes, wq, layer.mode, oracle_offsets(layer), rows=rows,
                               threads=threads or oracle.num_threads())
