"""CPU oracle for the SegQuant DualScale + SegLinear W8A8 linear layer.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg; never by the library's product path.  It shares
no code with the CUDA path.  The arithmetic lives in oracle.c (plain C, one
obvious loop per formula); this module only marshals numpy arrays into it.

Definitions followed (see oracle.c for the full list of readings):
  "SegQuant" (papernotes.org), section DualScale: X+ = max(X,0), X- = min(X,0),
  s+ = max/q_max, s- = |min|/|q_min|, Y = s+ s_w (X^+ W^) + s- s_w (X^- W^);
  section SegLinear: output-segmented concatenation, input-segmented sum.
  "SegQuant" author page, section 3: the case-wise quantizer Q_dual.

Conventions: bf16 tensors travel as uint16 bit patterns; the segment table is
(mode, offsets, G) with mode 0 = none, 1 = output-segmented, 2 = input-
segmented.
"""
import ctypes

import numpy as np

from . import build as _build

MODE_NONE, MODE_OUTPUT, MODE_INPUT = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.orc_calibrate_act.argtypes = [p, i64, i64, i64, p, i32, i32, p, i32, i64, i32, p]
        L.orc_quantize_act.argtypes = [p, i64, i64, i64, p, p, i32, i32, p, i32, i64, i32, p]
        L.orc_quantize_weight.argtypes = [p, i64, i64, p, i32, i32, p, i32, p, p]
        L.orc_quantize_weight_q.argtypes = [p, i64, i64, p, i32, i32, p, i32, i32, p, p]
        L.orc_pack_w4.argtypes = [p, i64, i64, p]
        L.orc_gemm_s32.argtypes = [p, p, i64, i64, i64, i32, i32, p, i32, i32, p, i64, p, i32]
        L.orc_gemm.argtypes = [p, p, p, p, p, i64, i64, i64, i32, i32, p, i32, i32, p, i64, p,
                               i32]
        L.orc_num_threads.argtypes = []
        L.orc_e4m3_encode.argtypes = [p, i64, p]
        L.orc_e4m3_decode.argtypes = [p, i64, p]
        L.orc_calibrate_act_fp8.argtypes = [p, i64, i64, i64, p, i32, i32, p, i32, i64, i32, p]
        L.orc_quantize_act_fp8.argtypes = [p, i64, i64, i64, p, p, i32, i32, p, i32, i64, i32,
                                           p]
        L.orc_quantize_weight_fp8.argtypes = [p, i64, i64, p, i32, i32, p, i32, p, p]
        L.orc_gemm_fp8_acc.argtypes = [p, p, i64, i64, i64, i32, i32, p, i32, i32, p, i64, p,
                                       i32]
        L.orc_gelu_bf16.argtypes = [p, i64, p]
        L.orc_gelu_parts.argtypes = [p, i64, p, p, p, p]
        L.orc_gemm_fp8.argtypes = [p, p, p, p, p, i64, i64, i64, i32, i32, p, i32, i32, p, i64,
                                   p, i32]
        for f in (L.orc_calibrate_act, L.orc_quantize_act, L.orc_quantize_weight,
                  L.orc_quantize_weight_q, L.orc_pack_w4,
                  L.orc_gemm_s32, L.orc_gemm, L.orc_num_threads, L.orc_e4m3_encode,
                  L.orc_e4m3_decode, L.orc_calibrate_act_fp8, L.orc_quantize_act_fp8,
                  L.orc_quantize_weight_fp8, L.orc_gemm_fp8_acc, L.orc_gemm_fp8):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _seg(mode, offsets, G, N, K):
    if offsets is None:
        offsets = [0, K if mode != MODE_OUTPUT else N]
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int32))
    n_seg = len(off) - 1
    S = n_seg if mode == MODE_INPUT else 1
    return off, n_seg, S


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


def num_threads():
    return lib().orc_num_threads()


def calibrate_act(x_bits, d=None, mode=MODE_NONE, offsets=None, G=1, N=0, single=False):
    """AMax calibration: returns s_act float32 [G][S][2] = {s+, s-} (equal in
    single-scale mode)."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    d = _c(d, np.float32)
    out = np.zeros((G, S, 2), np.float32)
    _check(lib().orc_calibrate_act(_ptr(x), M, K, K, _ptr(d), mode, n_seg,
                                   _ptr(off), G, N, int(single), _ptr(out)), "calibrate_act")
    return out


def quantize_act(x_bits, s_act, d=None, mode=MODE_NONE, offsets=None, G=1, N=0,
                 single=False):
    """Q_dual of X / d: returns planes int8 [G][2][M][K] (0 = X^+, 1 = X^-), or
    [G][1][M][K] holding X^+ + X^- in single-scale mode."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    s = _c(s_act, np.float32)
    assert s.size == G * S * 2
    d = _c(d, np.float32)
    planes = np.zeros((G, 1 if single else 2, M, K), np.int8)
    _check(lib().orc_quantize_act(_ptr(x), M, K, K, _ptr(d), _ptr(s), mode,
                                  n_seg, _ptr(off), G, N, int(single), _ptr(planes)),
           "quantize_act")
    return planes


def quantize_weight(w_bits, d=None, mode=MODE_NONE, offsets=None, G=1, bits=8):
    """Segment-wise AMax weight quantization: returns (wq int8 [N][K], s_w f32 [S][N]).
    bits=8: codes in [-127, 127]; bits=4 (W4A8): codes in [-7, 7]."""
    w = _c(w_bits, np.uint16)
    N, K = w.shape
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    d = _c(d, np.float32)
    wq = np.zeros((N, K), np.int8)
    s_w = np.zeros((S, N), np.float32)
    qmax = {8: 127, 4: 7}[bits]
    _check(lib().orc_quantize_weight_q(_ptr(w), N, K, _ptr(d), mode, n_seg,
                                       _ptr(off), G, qmax, _ptr(wq), _ptr(s_w)),
           "quantize_weight")
    return wq, s_w


def pack_w4(wq):
    """4-bit storage of codes in [-8, 7]: uint8 [N][K/2], channel 2j in the low
    nibble and 2j + 1 in the high nibble (two's complement)."""
    wq = _c(wq, np.int8)
    N, K = wq.shape
    out = np.zeros((N, K // 2), np.uint8)
    _check(lib().orc_pack_w4(_ptr(wq), N, K, _ptr(out)), "pack_w4")
    return out


def _rows(rows, M):
    if rows is None:
        return None, M
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    assert r.ndim == 1 and (r.size == 0 or (r.min() >= 0 and r.max() < M))
    return r, r.size


def gemm_s32(planes, wq, mode=MODE_NONE, offsets=None, rows=None, threads=1):
    """Raw int32 accumulators [S][P][rows][N] (P = planes per group)."""
    planes = _c(planes, np.int8)
    wq = _c(wq, np.int8)
    G, P, M, K = planes.shape
    N = wq.shape[0]
    assert P in (1, 2) and wq.shape[1] == K
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    r, nr = _rows(rows, M)
    acc = np.zeros((S, P, nr, N), np.int32)
    _check(lib().orc_gemm_s32(_ptr(planes), _ptr(wq), M, N, K, mode, n_seg,
                              _ptr(off), G, P, _ptr(r), nr, _ptr(acc), threads),
           "gemm_s32")
    return acc


def gemm(planes, wq, s_w, s_act, bias_bits=None, mode=MODE_NONE, offsets=None,
         rows=None, threads=1):
    """Layer output, fp32 epilogue: float32 [rows][N]."""
    planes = _c(planes, np.int8)
    wq = _c(wq, np.int8)
    G, P, M, K = planes.shape
    N = wq.shape[0]
    assert P in (1, 2) and wq.shape[1] == K
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    s_w = _c(s_w, np.float32)
    s_act = _c(s_act, np.float32)
    assert s_w.size == S * N and s_act.size == G * S * 2
    b = _c(bias_bits, np.uint16)
    r, nr = _rows(rows, M)
    y = np.zeros((nr, N), np.float32)
    _check(lib().orc_gemm(_ptr(planes), _ptr(wq), _ptr(s_w), _ptr(s_act),
                          _ptr(b), M, N, K, mode, n_seg, _ptr(off), G, P, _ptr(r),
                          nr, _ptr(y), threads), "gemm")
    return y


def layer(x_bits, w_bits, x_cal_bits, d=None, bias_bits=None, mode=MODE_NONE,
          offsets=None, G=1, rows=None, threads=1, single=False, weight_bits=8):
    """Whole static pipeline on the CPU: calibrate, quantize both sides, GEMM.

    Returns a dict with s_act, planes, wq, s_w and y (fp32 rows)."""
    w = _c(w_bits, np.uint16)
    N = w.shape[0]
    s_act = calibrate_act(x_cal_bits, d, mode, offsets, G, N, single)
    planes = quantize_act(x_bits, s_act, d, mode, offsets, G, N, single)
    wq, s_w = quantize_weight(w, d, mode, offsets, G, bits=weight_bits)
    y = gemm(planes, wq, s_w, s_act, bias_bits, mode, offsets, rows, threads)
    return dict(s_act=s_act, planes=planes, wq=wq, s_w=s_w, y=y)


# ------------------------------------------------------------------ FP8 (E4M3)
def e4m3_encode(v):
    """fp32 -> E4M3 codes (uint8): round half to even, finite saturation to +-448,
    NaN -> 0x7F."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    out = np.zeros(v.shape, np.uint8)
    _check(lib().orc_e4m3_encode(_ptr(v), v.size, _ptr(out)), "e4m3_encode")
    return out


def e4m3_decode(b):
    """E4M3 codes (uint8) -> their fp32 values (NaN for 0x7F / 0xFF)."""
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint8))
    out = np.zeros(b.shape, np.float32)
    _check(lib().orc_e4m3_decode(_ptr(b), b.size, _ptr(out)), "e4m3_decode")
    return out


def calibrate_act_fp8(x_bits, d=None, mode=MODE_NONE, offsets=None, G=1, N=0, single=False):
    """AMax calibration of the FP8 path: s+ = max/448, s- = |min|/448."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    d = _c(d, np.float32)
    out = np.zeros((G, S, 2), np.float32)
    _check(lib().orc_calibrate_act_fp8(_ptr(x), M, K, K, _ptr(d), mode, n_seg, _ptr(off), G, N,
                                       int(single), _ptr(out)), "calibrate_act_fp8")
    return out


def quantize_act_fp8(x_bits, s_act, d=None, mode=MODE_NONE, offsets=None, G=1, N=0,
                     single=False):
    """DualScale planes of E4M3 codes: uint8 [G][2][M][K] ([G][1][M][K] single scale)."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    s = _c(s_act, np.float32)
    d = _c(d, np.float32)
    planes = np.zeros((G, 1 if single else 2, M, K), np.uint8)
    _check(lib().orc_quantize_act_fp8(_ptr(x), M, K, K, _ptr(d), _ptr(s), mode, n_seg, _ptr(off),
                                      G, N, int(single), _ptr(planes)), "quantize_act_fp8")
    return planes


def quantize_weight_fp8(w_bits, d=None, mode=MODE_NONE, offsets=None, G=1):
    """E4M3 weights: (wq uint8 [N][K], s_w f32 [S][N]) with s_w = amax/448."""
    w = _c(w_bits, np.uint16)
    N, K = w.shape
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    d = _c(d, np.float32)
    wq = np.zeros((N, K), np.uint8)
    s_w = np.zeros((S, N), np.float32)
    _check(lib().orc_quantize_weight_fp8(_ptr(w), N, K, _ptr(d), mode, n_seg, _ptr(off), G,
                                         _ptr(wq), _ptr(s_w)), "quantize_weight_fp8")
    return wq, s_w


def gemm_fp8_acc(planes, wq, mode=MODE_NONE, offsets=None, rows=None, threads=1):
    """Exact sums of E4M3 products rounded once to fp32: [S][P][rows][N]."""
    planes = _c(planes, np.uint8)
    wq = _c(wq, np.uint8)
    G, P, M, K = planes.shape
    N = wq.shape[0]
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    r, n_rows = _rows(rows, M)
    acc = np.zeros((S, P, n_rows, N), np.float32)
    _check(lib().orc_gemm_fp8_acc(_ptr(planes), _ptr(wq), M, N, K, mode, n_seg, _ptr(off), G, P,
                                  _ptr(r), n_rows, _ptr(acc), threads), "gemm_fp8_acc")
    return acc


def gemm_fp8(planes, wq, s_w, s_act, bias_bits=None, mode=MODE_NONE, offsets=None, rows=None,
             threads=1):
    """FP8 layer output fp32 [rows][N]: the W8A8 epilogue on the fp32 sums."""
    planes = _c(planes, np.uint8)
    wq = _c(wq, np.uint8)
    G, P, M, K = planes.shape
    N = wq.shape[0]
    off, n_seg, S = _seg(mode, offsets, G, N, K)
    r, n_rows = _rows(rows, M)
    y = np.zeros((n_rows, N), np.float32)
    _check(lib().orc_gemm_fp8(_ptr(planes), _ptr(wq), _ptr(_c(s_w, np.float32)),
                              _ptr(_c(s_act, np.float32)), _ptr(_c(bias_bits, np.uint16)), M, N,
                              K, mode, n_seg, _ptr(off), G, P, _ptr(r), n_rows, _ptr(y),
                              threads), "gemm_fp8")
    return y


def layer_fp8(x_bits, w_bits, x_cal_bits, d=None, bias_bits=None, mode=MODE_NONE, offsets=None,
              G=1, rows=None, threads=1, single=False):
    """Whole FP8 pipeline on the CPU: calibrate, quantize both sides, GEMM."""
    w = _c(w_bits, np.uint16)
    N = w.shape[0]
    s_act = calibrate_act_fp8(x_cal_bits, d, mode, offsets, G, N, single)
    planes = quantize_act_fp8(x_bits, s_act, d, mode, offsets, G, N, single)
    wq, s_w = quantize_weight_fp8(w, d, mode, offsets, G)
    y = gemm_fp8(planes, wq, s_w, s_act, bias_bits, mode, offsets, rows, threads)
    return dict(s_act=s_act, planes=planes, wq=wq, s_w=s_w, y=y)


def gelu_bf16(y):
    """bf16(gelu(bf16(y))) of fp32 values, as bf16 bit patterns (uint16): the
    FFN activation between fc1 and fc2, tanh approximation, for the fused
    producer."""
    y = _c(y, np.float32)
    out = np.empty(y.shape, np.uint16)
    _check(lib().orc_gelu_bf16(_ptr(y), y.size, _ptr(out)), "gelu_bf16")
    return out


def gelu_parts(x):
    """The pieces of gelu_bf16 on fp32 inputs: e^x (for 0 <= x <= 18), tanh,
    gelu, and bf16 rounding (bit patterns)."""
    x = _c(x, np.float32)
    e, t, g = (np.empty(x.shape, np.float32) for _ in range(3))
    b = np.empty(x.shape, np.uint16)
    _check(lib().orc_gelu_parts(_ptr(x), x.size, _ptr(e), _ptr(t), _ptr(g), _ptr(b)),
           "gelu_parts")
    return dict(exp=e, tanh=t, gelu=g, bf16=b)


__all__ = ["MODE_NONE", "MODE_OUTPUT", "MODE_INPUT", "calibrate_act",
           "quantize_act", "quantize_weight", "pack_w4", "gemm_s32", "gemm", "layer",
           "num_threads", "lib", "e4m3_encode", "e4m3_decode", "calibrate_act_fp8",
           "quantize_act_fp8", "quantize_weight_fp8", "gemm_fp8_acc", "gemm_fp8", "layer_fp8",
           "gelu_bf16", "gelu_parts"]
