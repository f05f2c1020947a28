"""Host-side checks that need no GPU: the C-ABI library loads, exports every
entry point include/segquant.h declares, and rejects invalid arguments on the
host before touching CUDA (so these calls are safe without a device)."""
import ctypes
import os
import re

import numpy as np

import pytest

from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import build as sqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "segquant.h")

SQ_ERR_INVALID_ARG, SQ_ERR_UNSUPPORTED, SQ_ERR_ALIGNMENT, SQ_ERR_OVERFLOW = -1, -2, -3, -4


@pytest.fixture(scope="module")
def L():
    sqbuild.build()
    return B.lib()


def declared_entry_points():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SQ_API\s+[\w\s\*]+?\b(sq_\w+)\s*\(", text)))


def test_header_declares_expected_calls():
    names = declared_entry_points()
    for n in ("sq_quantize_act", "sq_quantize_weight_seg", "sq_dualscale_seglinear_gemm"):
        assert n in names
    assert set(names) == set(B.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_entry_points():
        assert hasattr(L, name), name


def test_status_strings(L):
    assert B.status_string(0) == "SQ_OK"
    for code in range(-9, 0):
        assert B.status_string(code).startswith("SQ_ERR_")
    assert B.lib().sq_version() == 201


def _seg(mode, offsets, groups=1):
    s = B.Segments(mode, offsets, groups)
    c, keep = s._c()
    return c, keep


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def test_quantize_act_rejects_bad_shapes(L):
    p = ctypes.c_void_p
    c, keep = _seg(B.SQ_SEG_NONE, None)
    # K not a multiple of 16
    assert L.sq_quantize_act(p(FAKE), 4, 24, 24, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG
    # ldx < K
    assert L.sq_quantize_act(p(FAKE), 4, 32, 16, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG
    # misaligned x
    assert L.sq_quantize_act(p(FAKE + 2), 4, 32, 32, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_ALIGNMENT
    # ldx not a multiple of 8 elements
    assert L.sq_quantize_act(p(FAKE), 4, 32, 36, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_ALIGNMENT
    # an input of more than 2^44 elements (including a huge row stride)
    assert L.sq_quantize_act(p(FAKE), 2**31 - 1, 2**20, 2**20, None, p(FAKE), ctypes.byref(c),
                             p(FAKE), None) == SQ_ERR_INVALID_ARG
    assert L.sq_quantize_act(p(FAKE), 2**20, 32, 2**62, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG


def test_segment_table_validation(L):
    p = ctypes.c_void_p
    # input segments must end at K and be multiples of 32 wide
    c, keep = _seg(B.SQ_SEG_INPUT, [0, 32, 48])
    assert L.sq_quantize_act(p(FAKE), 4, 48, 48, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_UNSUPPORTED
    c, keep = _seg(B.SQ_SEG_INPUT, [0, 32, 32, 64])
    assert L.sq_quantize_act(p(FAKE), 4, 64, 64, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG
    c, keep = _seg(B.SQ_SEG_INPUT, [0, 32, 64])
    assert L.sq_quantize_act(p(FAKE), 4, 96, 96, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG
    # input mode has one activation group
    c, keep = _seg(B.SQ_SEG_INPUT, [0, 32, 64], groups=2)
    assert L.sq_quantize_act(p(FAKE), 4, 64, 64, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG
    # output mode: G must be 1 or n_seg; with G > 1 widths are multiples of 128
    c, keep = _seg(B.SQ_SEG_OUTPUT, [0, 128, 256, 384], groups=2)
    assert L.sq_quantize_weight_seg(p(FAKE), 384, 64, None, ctypes.byref(c), p(FAKE), p(FAKE),
                                    None) == SQ_ERR_INVALID_ARG
    c, keep = _seg(B.SQ_SEG_OUTPUT, [0, 64, 192], groups=2)
    assert L.sq_quantize_weight_seg(p(FAKE), 192, 64, None, ctypes.byref(c), p(FAKE), p(FAKE),
                                    None) == SQ_ERR_UNSUPPORTED
    # output offsets must end at N
    c, keep = _seg(B.SQ_SEG_OUTPUT, [0, 128, 256], groups=1)
    assert L.sq_quantize_weight_seg(p(FAKE), 300, 64, None, ctypes.byref(c), p(FAKE), p(FAKE),
                                    None) == SQ_ERR_INVALID_ARG
    # too many segments
    offs = list(range(0, 32 * 66, 32))
    c, keep = _seg(B.SQ_SEG_INPUT, offs)
    K = offs[-1]
    assert L.sq_quantize_act(p(FAKE), 4, K, K, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG


def test_unknown_flags_rejected(L):
    p = ctypes.c_void_p
    s = B.Segments(B.SQ_SEG_NONE, None, 1, flags=8)
    c, keep = s._c()
    assert L.sq_quantize_act(p(FAKE), 4, 32, 32, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG
    # W4 weights and FP8 codes do not combine
    s = B.Segments(B.SQ_SEG_NONE, None, 1, flags=B.SQ_FLAG_W4 | B.SQ_FLAG_FP8)
    c, keep = s._c()
    assert L.sq_quantize_act(p(FAKE), 4, 32, 32, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == SQ_ERR_INVALID_ARG
    s = B.Segments(B.SQ_SEG_NONE, None, 1, flags=B.SQ_FLAG_SINGLE_SCALE)
    c, keep = s._c()
    # a valid single-scale table gets past validation (M == 0: no-op, no CUDA)
    assert L.sq_quantize_act(p(FAKE), 0, 32, 32, None, p(FAKE), ctypes.byref(c), p(FAKE),
                             None) == 0


def test_gemm_overflow_and_layout_checks(L):
    p = ctypes.c_void_p
    c, keep = _seg(B.SQ_SEG_NONE, None)
    # one K-segment wider than 132104 could overflow int32
    K = 132112
    assert L.sq_dualscale_seglinear_gemm(p(FAKE), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), 0,
                                         8, 8, K, 8, ctypes.byref(c), None) == SQ_ERR_OVERFLOW
    # ldy < N
    assert L.sq_dualscale_seglinear_gemm(p(FAKE), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), 0,
                                         8, 16, 64, 8, ctypes.byref(c), None) == SQ_ERR_INVALID_ARG
    # an output of more than 2^44 elements (M, N each within int32)
    big = 2**31 - 1
    assert L.sq_dualscale_seglinear_gemm(p(FAKE), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), 0,
                                         big, big, 64, big + 1, ctypes.byref(c),
                                         None) == SQ_ERR_INVALID_ARG
    # bf16 output rows must start 16-byte aligned (ldy multiple of 8)
    assert L.sq_dualscale_seglinear_gemm(p(FAKE), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), 0,
                                         8, 20, 64, 20, ctypes.byref(c), None) == SQ_ERR_ALIGNMENT
    # bad output dtype
    assert L.sq_dualscale_seglinear_gemm(p(FAKE), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), 7,
                                         8, 16, 64, 16, ctypes.byref(c), None) == SQ_ERR_INVALID_ARG
    # misaligned planes
    assert L.sq_dualscale_seglinear_gemm(p(FAKE + 8), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), 0,
                                         8, 16, 64, 16, ctypes.byref(c), None) == SQ_ERR_ALIGNMENT
    # null scales
    assert L.sq_dualscale_seglinear_gemm(p(FAKE), p(FAKE), None, p(FAKE), None, p(FAKE), 0,
                                         8, 16, 64, 16, ctypes.byref(c), None) == SQ_ERR_INVALID_ARG
    # M == 0 is a valid no-op that never touches CUDA
    assert L.sq_dualscale_seglinear_gemm(None, None, None, None, None, None, 0,
                                         0, 16, 64, 16, ctypes.byref(c), None) == 0


def test_binding_without_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        B.lib()


def test_w4_calls_validate_on_host(L):
    p = ctypes.c_void_p
    c, keep = _seg(B.SQ_SEG_NONE, None)
    # K not a multiple of 16
    assert L.sq_quantize_weight_w4(p(FAKE), 8, 24, None, ctypes.byref(c), p(FAKE), p(FAKE),
                                   None) == SQ_ERR_INVALID_ARG
    # misaligned packed output
    assert L.sq_quantize_weight_w4(p(FAKE), 8, 32, None, ctypes.byref(c), p(FAKE + 8), p(FAKE),
                                   None) == SQ_ERR_ALIGNMENT
    assert L.sq_unpack_weight_w4(p(FAKE), 0, 32, p(FAKE), None) == SQ_ERR_INVALID_ARG
    assert L.sq_unpack_weight_w4(p(FAKE), 8, 40, p(FAKE), None) == SQ_ERR_INVALID_ARG
    assert L.sq_unpack_weight_w4(p(FAKE + 4), 8, 32, p(FAKE), None) == SQ_ERR_ALIGNMENT
    # the W4 flag is a valid segment-table flag, alone or with single scale
    for flags in (B.SQ_FLAG_W4, B.SQ_FLAG_W4 | B.SQ_FLAG_SINGLE_SCALE):
        cs, keep = B.Segments(B.SQ_SEG_NONE, None, 1, flags=flags)._c()
        assert L.sq_dualscale_seglinear_gemm(None, None, None, None, None, None, 0,
                                             0, 16, 64, 16, ctypes.byref(cs), None) == 0


def test_host_pipeline_validates_on_host(L):
    p = ctypes.c_void_p
    assert L.sq_host_pipeline_workspace_bytes(0, 64, 64, 1, 2) == 0
    assert L.sq_host_pipeline_workspace_bytes(128, 24, 64, 1, 2) == 0      # K % 16 != 0
    assert L.sq_host_pipeline_workspace_bytes(128, 64, 64, 1, 3) == 0      # P must be 1 or 2
    # sizes whose byte counts would not fit 64 bits are rejected, not wrapped
    assert L.sq_host_pipeline_workspace_bytes(2**31 - 1, 2**31 - 16, 2**31 - 1, 64, 2) == 0
    assert L.sq_host_pipeline_workspace_bytes(2**31 - 1, 2**20, 64, 1, 2) == 0
    need = L.sq_host_pipeline_workspace_bytes(128, 64, 64, 1, 2)
    # two slots of x (128*64*2) + planes (2*128*64) + y (128*64*4), 256-byte rounded
    assert need == 2 * (16384 + 16384 + 32768)
    h = p()
    assert L.sq_host_pipeline_create(128, 64, 64, 1, 2, None, need, ctypes.byref(h)) == \
        SQ_ERR_INVALID_ARG
    assert L.sq_host_pipeline_create(128, 64, 64, 1, 2, p(FAKE), need - 1, ctypes.byref(h)) == \
        SQ_ERR_INVALID_ARG
    assert L.sq_host_pipeline_create(128, 64, 64, 1, 2, p(FAKE + 16), need, ctypes.byref(h)) == \
        SQ_ERR_ALIGNMENT
    assert L.sq_host_pipeline_destroy(None) == 0
    c, keep = _seg(B.SQ_SEG_NONE, None)
    assert L.sq_dualscale_seglinear_host(None, p(FAKE), 8, 64, 64, None, p(FAKE), p(FAKE),
                                         p(FAKE), None, p(FAKE), 0, 64, 64, ctypes.byref(c),
                                         None) == SQ_ERR_INVALID_ARG


def test_gelu_quant_validation(L):
    """The fused producer's host checks, before any launch."""
    p = ctypes.c_void_p
    none, keep0 = _seg(B.SQ_SEG_NONE, None)
    inp, keep1 = _seg(B.SQ_SEG_INPUT, [0, 32, 64])
    f = L.sq_dualscale_seglinear_gemm_gelu_quant
    args = lambda seg, N=64, s_next=FAKE, flags=0: (p(FAKE), p(FAKE), p(FAKE), p(FAKE), None,
                                                    8, N, 64, ctypes.byref(seg), p(s_next),
                                                    flags, p(FAKE), None)
    assert f(*args(inp)) == SQ_ERR_UNSUPPORTED            # this layer: one K-segment only
    assert f(*args(none, flags=B.SQ_FLAG_W4)) == SQ_ERR_INVALID_ARG   # next: 0 or single scale
    assert f(*args(none, N=40)) == SQ_ERR_ALIGNMENT       # N is the next layer's K: % 16
    assert f(*args(none, s_next=0)) == SQ_ERR_INVALID_ARG  # the next layer's steps
    fp8, keep2 = B.Segments(B.SQ_SEG_NONE, None, 1, B.SQ_FLAG_FP8)._c()
    assert f(*args(fp8)) == SQ_ERR_UNSUPPORTED
    # M == 0 is a valid no-op that never touches CUDA
    assert f(p(FAKE), p(FAKE), p(FAKE), p(FAKE), None, 0, 64, 64, ctypes.byref(none), p(FAKE), 0,
             p(FAKE), None) == 0



def _choose(L, steps, flags=0, threshold=2.0):
    arr = np.ascontiguousarray(np.asarray(steps, np.float32).reshape(-1, 2))
    out = ctypes.c_int32(-1)
    rc = L.sq_choose_single_scale(arr.ctypes.data_as(ctypes.c_void_p), arr.shape[0], flags,
                                  ctypes.c_float(threshold), ctypes.byref(out))
    return rc, out.value


def test_choose_single_scale_policy(L):
    """The adaptive policy on the host: max = s+ * 127 and |min| = s- * 128
    (448 for FP8); single scale only where every group and K-segment has
    max(max, |min|) < threshold * min(max, |min|)."""
    # max 1.0, |min| 0.9: close -> single
    assert _choose(L, [[1.0 / 127, 0.9 / 128]]) == (0, 1)
    # max 1.0, |min| 0.3: ratio 3.3 -> keep DualScale
    assert _choose(L, [[1.0 / 127, 0.3 / 128]]) == (0, 0)
    # one asymmetric (group, segment) among symmetric ones keeps the layer DualScale
    steps = [[1.0 / 127, 1.0 / 128]] * 23 + [[4.0 / 127, 1.0 / 128]]
    assert _choose(L, steps) == (0, 0)
    assert _choose(L, steps[:23]) == (0, 1)
    # the threshold is strict, and it is the caller's
    assert _choose(L, [[2.0 / 127, 1.0 / 128]], threshold=2.0) == (0, 0)
    assert _choose(L, [[2.0 / 127, 1.0 / 128]], threshold=2.5) == (0, 1)
    # an empty side has step 1 and counts as large: a one-sided layer keeps DualScale
    assert _choose(L, [[0.5 / 127, 1.0]]) == (0, 0)
    # FP8 steps are max / 448 on both sides
    assert _choose(L, [[1.0 / 448, 0.6 / 448]], flags=B.SQ_FLAG_FP8) == (0, 1)
    assert _choose(L, [[1.0 / 448, 0.4 / 448]], flags=B.SQ_FLAG_FP8) == (0, 0)


def test_choose_single_scale_rejects_bad_arguments(L):
    INVALID = -1
    assert _choose(L, [[0.0, 0.01]])[0] == INVALID          # a step of 0
    assert _choose(L, [[-0.01, 0.01]])[0] == INVALID        # negative
    assert _choose(L, [[float("nan"), 0.01]])[0] == INVALID
    assert _choose(L, [[float("inf"), 0.01]])[0] == INVALID
    assert _choose(L, [[0.01, 0.01]], threshold=1.0)[0] == INVALID
    assert _choose(L, [[0.01, 0.01]], flags=B.SQ_FLAG_W4)[0] == INVALID
    out = ctypes.c_int32(0)
    arr = np.ones(2, np.float32)
    assert L.sq_choose_single_scale(arr.ctypes.data_as(ctypes.c_void_p), 0, 0,
                                    ctypes.c_float(2.0), ctypes.byref(out)) == INVALID
    assert L.sq_choose_single_scale(None, 1, 0, ctypes.c_float(2.0), ctypes.byref(out)) == INVALID


def test_binding_choose_single_scale_takes_any_device_tensor():
    import torch
    s = torch.tensor([[[1.0 / 127, 0.9 / 128]], [[1.0 / 127, 0.95 / 128]]])
    assert B.sq_choose_single_scale(s) is True
    assert B.sq_choose_single_scale(s, threshold=1.05) is False


def test_debug_build_exports_the_same_calls_and_reports_its_checks(L):
    """The bounds-checked debug build is a second build of the same sources:
    it exports every declared call, and sq_debug_bounds_checks() tells the two
    builds apart (no device is touched)."""
    debug = ctypes.CDLL(sqbuild.build(debug=True))
    for name in declared_entry_points():
        assert hasattr(debug, name), name
    debug.sq_debug_bounds_checks.restype = ctypes.c_int32
    L.sq_debug_bounds_checks.restype = ctypes.c_int32
    assert debug.sq_debug_bounds_checks() == 1
    assert L.sq_debug_bounds_checks() == 0
    debug.sq_version.restype = ctypes.c_int32
    assert debug.sq_version() == L.sq_version()


def test_bounds_probe_rejects_bad_arguments_on_the_host(L):
    f = L.sq_debug_bounds_probe
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    f.restype = ctypes.c_int
    assert f(None, 8, None) == SQ_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(256), 0, None) == SQ_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(258), 8, None) == SQ_ERR_ALIGNMENT
    # the release build launches nothing for a valid request
    assert f(ctypes.c_void_p(256), 8, None) == SQ_ERR_UNSUPPORTED


def test_quantize_plan_rejects_bad_arguments_on_the_host(L):
    """The plan and the planned quantize check their arguments before touching
    a device: a plan needs divisors, covers int8 codes only, and is 4-byte
    aligned."""
    plan_f = L.sq_quantize_act_plan
    plan_f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                       ctypes.c_void_p, ctypes.c_void_p]
    plan_f.restype = ctypes.c_int
    seg = B.Segments()
    cs, keep = seg._c()
    ok = ctypes.c_void_p(256)
    assert plan_f(None, 256, ok, ctypes.byref(cs), ok, None) == SQ_ERR_INVALID_ARG
    assert plan_f(ok, 256, ok, ctypes.byref(cs), None, None) == SQ_ERR_INVALID_ARG
    assert plan_f(ok, 256, ok, ctypes.byref(cs), ctypes.c_void_p(258), None) == SQ_ERR_ALIGNMENT
    assert plan_f(ok, 100, ok, ctypes.byref(cs), ok, None) != 0     # K must be a multiple of 16
    cs8, keep8 = B.Segments(flags=B.SQ_FLAG_FP8)._c()
    assert plan_f(ok, 256, ok, ctypes.byref(cs8), ok, None) == SQ_ERR_UNSUPPORTED
    q = L.sq_quantize_act_planned
    q.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p]
    q.restype = ctypes.c_int
    # a plan without divisors
    assert q(ok, 4, 256, 256, None, ok, ctypes.byref(cs), ok, ok, None) == SQ_ERR_INVALID_ARG
    assert q(ok, 4, 256, 256, ok, ok, ctypes.byref(cs8), ok, ok, None) == SQ_ERR_UNSUPPORTED
