"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle's own formula retyped.

  * hand-derived worked examples (tests/golden/*.txt, each citing its passage);
  * brute force over every bf16 bit pattern with exact rational arithmetic;
  * closed forms (single-scale reduction, identity weight);
  * structural identities of SegLinear (output concatenation, input sum);
  * dequantize-then-float64-matmul on tiny shapes with ragged tails;
  * error bounds of round-to-nearest;
  * the qualitative claim that DualScale beats one scale on SiLU/GELU data.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import MODE_INPUT, MODE_NONE, MODE_OUTPUT
from w8a8_gemm_b200 import workloads as wl


# ----------------------------------------------------------------- helpers
def bf16_bits(vals):
    t = torch.tensor(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def parse_floats(s):
    return [float(v) for v in s.split()]


def read_fixture(golden_dir, name):
    lines = []
    with open(os.path.join(golden_dir, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                key, _, val = ln.partition(":")
                lines.append((key.strip(), val.strip()))
    return lines


def rne_fraction(v: Fraction) -> int:
    return round(v)  # Fraction.__round__ rounds half to even


# ----------------------------------------------------------- worked examples
def test_worked_dualscale_quantizer(golden_dir):
    fx = read_fixture(golden_dir, "dualscale_quant_worked.txt")
    kv = dict((k, v) for k, v in fx if k != "case")
    calib = np.array(parse_floats(kv["calib"]), np.float32)[None]
    s_act = oracle.calibrate_act(bf16_bits(calib))
    assert s_act[0, 0, 0] == np.float32(kv["s_plus"])
    assert s_act[0, 0, 1] == np.float32(kv["s_minus"])
    cases = [v.split() for k, v in fx if k == "case"]
    xs = np.array([float(c[0]) for c in cases], np.float32)[None]
    planes = oracle.quantize_act(bf16_bits(xs), s_act)
    for j, c in enumerate(cases):
        assert planes[0, 0, 0, j] == int(c[1]), c
        assert planes[0, 1, 0, j] == int(c[2]), c


def test_worked_smoothquant_fold(golden_dir):
    fx = read_fixture(golden_dir, "smoothquant_fold_worked.txt")
    d = np.array([parse_floats(v) for k, v in fx if k == "d"], np.float32)
    calib = np.array([parse_floats(v) for k, v in fx if k == "calib_row"], np.float32)
    kv = dict(fx)
    s_act = oracle.calibrate_act(bf16_bits(calib), d=d)
    assert s_act[0, 0, 0] == np.float32(kv["s_plus"])
    assert s_act[0, 0, 1] == np.float32(kv["s_minus"])
    for k, v in fx:
        if k != "row":
            continue
        xs, qp, qm = (parse_floats(p) for p in v.split("|"))
        planes = oracle.quantize_act(bf16_bits(np.array([xs], np.float32)), s_act, d=d)
        assert planes[0, 0, 0].tolist() == [int(q) for q in qp]
        assert planes[0, 1, 0].tolist() == [int(q) for q in qm]


def test_worked_weight_quant(golden_dir):
    fx = read_fixture(golden_dir, "weight_quant_worked.txt")
    rows, sws, qs = [], [], []
    for k, v in fx:
        w, sw, q = v.split("|")
        rows.append(parse_floats(w))
        sws.append(float(sw.split()[1]))
        qs.append([int(float(t)) for t in q.split()[1:]])
    wq, s_w = oracle.quantize_weight(bf16_bits(np.array(rows, np.float32)))
    assert s_w[0].tolist() == sws
    assert wq.tolist() == qs


def test_worked_weight_quant_w4(golden_dir):
    fx = read_fixture(golden_dir, "weight_quant_w4_worked.txt")
    rows, sws, qs, packed = [], [], [], []
    for k, v in fx:
        w, sw, q, pk = v.split("|")
        rows.append(parse_floats(w))
        sws.append(float(sw.split()[1]))
        qs.append([int(t) for t in q.split()[1:]])
        packed.append([int(t) for t in pk.split()[1:]])
    wq, s_w = oracle.quantize_weight(bf16_bits(np.array(rows, np.float32)), bits=4)
    assert s_w[0].tolist() == sws
    assert wq.tolist() == qs
    assert oracle.pack_w4(wq).tolist() == packed


def test_w4_codes_bounds_and_half_step():
    """W4 codes lie in [-7, 7], the largest |w| of each channel maps to +-7, and
    every weight is within half a step of its reconstruction s_w q."""
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((16, 96)) * rng.uniform(0.01, 1.0, (16, 1))).astype(np.float32)
    wb = bf16_bits(w)
    wf = (wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wq, s_w = oracle.quantize_weight(wb, bits=4)
    assert wq.min() >= -7 and wq.max() <= 7
    arg = np.abs(wf).argmax(axis=1)
    assert np.all(np.abs(wq[np.arange(16), arg]) == 7)
    err = np.abs(wf - s_w[0][:, None].astype(np.float64) * wq)
    assert np.all(err <= s_w[0][:, None] * (0.5 + 1e-6))


def test_w4_input_segments_use_their_own_amax():
    """With input segments every (channel, segment) pair has its own step."""
    w = np.zeros((2, 64), np.float32)
    w[:, :32] = 0.875      # segment 0: amax 7/8 -> s_w 1/8, codes 7
    w[:, 32:] = -0.109375  # segment 1: amax 7/64 -> s_w 1/64, codes -7
    wq, s_w = oracle.quantize_weight(bf16_bits(w), mode=oracle.MODE_INPUT, offsets=[0, 32, 64],
                                     bits=4)
    assert s_w.tolist() == [[0.125, 0.125], [0.015625, 0.015625]]
    assert np.all(wq[:, :32] == 7) and np.all(wq[:, 32:] == -7)


def test_w4_pack_nibble_order_and_range():
    wq = np.array([[-8, 7, 1, -1, 0, -8]], np.int8)
    assert oracle.pack_w4(wq).tolist() == [[0x78, 0xF1, 0x80]]
    with pytest.raises(Exception):
        oracle.pack_w4(np.array([[8, 0]], np.int8))


def test_w4_layer_equals_brute_force_dequantized_product():
    """W4A8 layer: the oracle's fp32 result against the dequantized operands
    multiplied in float64 (the DualScale factorisation with 4-bit weights)."""
    rng = np.random.default_rng(3)
    M, K, N = 7, 96, 9
    x = (rng.standard_normal((M, K)) * 2).astype(np.float32)
    xc = (rng.standard_normal((32, K)) * 2).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    r = oracle.layer(bf16_bits(x), bf16_bits(w), bf16_bits(xc), weight_bits=4)
    s = r["s_act"][0, 0]
    xt = s[0] * r["planes"][0, 0].astype(np.float64) + s[1] * r["planes"][0, 1]
    wt = r["s_w"][0][:, None].astype(np.float64) * r["wq"]
    assert r["wq"].min() >= -7 and r["wq"].max() <= 7
    ref = xt @ wt.T
    assert np.max(np.abs(r["y"] - ref)) <= 1e-5 * (np.abs(ref).max() + 1e-30)


def _ints(s):
    return [int(v) for v in s.split()]


def test_worked_gemm_all_modes(golden_dir):
    kv = dict(read_fixture(golden_dir, "gemm_worked.txt"))
    f = lambda k: np.array(parse_floats(kv[k]), np.float32)
    # one segment
    planes = np.array([[[_ints(kv["none.qplus"])], [_ints(kv["none.qminus"])]]], np.int8)
    wq = np.array([_ints(kv["none.w"])], np.int8)
    acc = oracle.gemm_s32(planes, wq)
    assert acc[0, :, 0, 0].tolist() == _ints(kv["none.acc"])
    y = oracle.gemm(planes, wq, f("none.s_w")[None], f("none.s_act"),
                    bf16_bits(f("none.bias")))
    assert y[0, 0] == np.float32(kv["none.y"])
    # input-segmented
    offs = _ints(kv["input.offsets"])
    planes = np.array([[[_ints(kv["input.qplus"])], [_ints(kv["input.qminus"])]]], np.int8)
    wq = np.array([_ints(kv["input.w"])], np.int8)
    acc = oracle.gemm_s32(planes, wq, MODE_INPUT, offs)
    assert acc[:, :, 0, 0].reshape(-1).tolist() == _ints(kv["input.acc"])
    y = oracle.gemm(planes, wq, f("input.s_w")[:, None], f("input.s_act"), None,
                    MODE_INPUT, offs)
    assert y[0, 0] == np.float32(kv["input.y"])
    # output-segmented, one activation group per segment
    offs = _ints(kv["output.offsets"])
    planes = np.array([[[_ints(kv["output.g0.qplus"])], [_ints(kv["output.g0.qminus"])]],
                       [[_ints(kv["output.g1.qplus"])], [_ints(kv["output.g1.qminus"])]]],
                      np.int8)
    wq = np.array([_ints(kv["output.w0"]), _ints(kv["output.w1"])], np.int8)
    acc = oracle.gemm_s32(planes, wq, MODE_OUTPUT, offs)
    assert acc[0, 0, 0].tolist() == _ints(kv["output.acc_plus"])
    assert acc[0, 1, 0].tolist() == _ints(kv["output.acc_minus"])
    y = oracle.gemm(planes, wq, f("output.s_w")[None], f("output.s_act"), None,
                    MODE_OUTPUT, offs)
    assert y[0].tolist() == parse_floats(kv["output.y"])


# ------------------------------------------------------ brute force, all bf16
def _expected_q(x: float, mult: int):
    """Exact-rational Q_dual with power-of-two step 1/mult."""
    if math.isnan(x):
        return 0, 0
    if x < 0:
        if math.isinf(x):
            return 0, -128
        return 0, max(-128, rne_fraction(Fraction(x) * mult))
    if math.isinf(x):
        return 127, 0
    return min(127, rne_fraction(Fraction(x) * mult)), 0


def test_bruteforce_every_bf16_value():
    """Every one of the 65536 bf16 patterns through Q_dual with s+ = 1/64 and
    s- = 1/512 (powers of two, so x / s is exact and only the rounding rule,
    the sign split and the saturation decide the code)."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    s_act = np.array([[[1 / 64, 1 / 512]]], np.float32)
    planes = oracle.quantize_act(allbits, s_act)
    xs = bits_to_f32(allbits.reshape(-1))
    qp = planes[0, 0].reshape(-1)
    qm = planes[0, 1].reshape(-1)
    exp = [_expected_q(float(x), 64 if not (x < 0) else 512) for x in xs]
    assert qp.tolist() == [e[0] for e in exp]
    assert qm.tolist() == [e[1] for e in exp]


def test_bruteforce_weight_power_of_two_scale():
    """Rows whose amax is 127 * 2^-e: s_w = 2^-e, so w / s_w is exact and the
    code must equal the exact round-half-even of w * 2^e."""
    rng = np.random.default_rng(0)
    for e in (3, 7, 10):
        vals = bits_to_f32(rng.integers(0, 65536, size=(8, 40), dtype=np.uint32)
                           .astype(np.uint16))
        vals = np.where(np.isfinite(vals), vals, 0).astype(np.float32)
        vals = np.clip(vals, -127 * 2.0 ** -e, 127 * 2.0 ** -e)
        vals[:, 0] = 127 * 2.0 ** -e  # fixes amax
        w = bf16_bits(vals)
        wf = bits_to_f32(w)
        wq, s_w = oracle.quantize_weight(w)
        assert np.all(s_w == np.float32(2.0 ** -e))
        for n in range(wf.shape[0]):
            for k in range(wf.shape[1]):
                assert wq[n, k] == rne_fraction(Fraction(float(wf[n, k])) * 2 ** e)


# -------------------------------------------------------------- invariants
def _c1_like(M=96, K=160, N=72, seed=0):
    return wl.gelu_layer("t", M, K, N, seed, bias=True)


def test_split_identity_and_rounding_bound():
    """X = X+ + X-: every element lands in exactly one plane with its own sign,
    and |s q - x/d| <= s/2 (the round-to-nearest half step) inside the range."""
    L = wl.adanorm_layer("t", 64, 128, 96, 3, seed=1, G=3)
    xb = wl.bits(L.x)
    d = L.d.numpy()
    s_act = oracle.calibrate_act(wl.bits(L.x_cal), d, MODE_OUTPUT, L.offsets, 3, L.N)
    planes = oracle.quantize_act(xb, s_act, d, MODE_OUTPUT, L.offsets, 3, L.N)
    x = bits_to_f32(xb).astype(np.float64)
    for g in range(3):
        qp, qm = planes[g, 0].astype(np.int64), planes[g, 1].astype(np.int64)
        assert np.all((qp == 0) | (qm == 0))
        assert np.all(qp >= 0) and np.all(qm <= 0)
        assert np.all(qp[x < 0] == 0) and np.all(qm[x >= 0] == 0)
        sp, sm = float(s_act[g, 0, 0]), float(s_act[g, 0, 1])
        u = x / d[g].astype(np.float64)[None]
        inr_p = (u >= 0) & (u / sp <= 127)
        inr_m = (u < 0) & (u / sm >= -128)
        tol = 0.5 + 1e-4
        assert np.all(np.abs(qp[inr_p] - u[inr_p] / sp) <= tol)
        assert np.all(np.abs(qm[inr_m] - u[inr_m] / sm) <= tol)
        # out-of-range values saturate
        assert np.all(qp[(u >= 0) & (u / sp > 127.5 + 1e-4)] == 127)
        assert np.all(qm[(u < 0) & (u / sm < -128.5 - 1e-4)] == -128)


def test_calibration_extremes_map_to_code_limits():
    """Quantizing the calibration slice with its own AMax scales sends the max
    to +127 and the min to -128 (q_max = 127, |q_min| = 128)."""
    L = _c1_like()
    xb = wl.bits(L.x_cal)
    s = oracle.calibrate_act(xb)
    planes = oracle.quantize_act(xb, s)
    x = bits_to_f32(xb)
    assert planes[0, 0].reshape(-1)[np.argmax(x)] == 127
    assert planes[0, 1].reshape(-1)[np.argmin(x)] == -128
    assert planes[0, 0].max() == 127 and planes[0, 1].min() == -128


def test_calibration_degenerate_and_nan():
    pos = bf16_bits(np.array([[0.5, 1.0, 0.0]], np.float32))
    neg = bf16_bits(np.array([[-0.5, -1.0, -0.0]], np.float32))
    zero = bf16_bits(np.zeros((1, 3), np.float32))
    assert oracle.calibrate_act(pos)[0, 0, 1] == 1.0   # no negatives -> s- = 1
    assert oracle.calibrate_act(neg)[0, 0, 0] == 1.0   # no positives -> s+ = 1
    assert oracle.calibrate_act(zero)[0, 0].tolist() == [1.0, 1.0]
    withnan = bf16_bits(np.array([[np.nan, 1.984375, -0.25]], np.float32))
    assert oracle.calibrate_act(withnan)[0, 0].tolist() == [1 / 64, 1 / 512]


def test_calibration_segments_independent():
    L = wl.outproj_layer("t", 64, 128, 32, 32, seed=2)
    xb = wl.bits(L.x_cal).copy()
    s0 = oracle.calibrate_act(xb, L.d.numpy(), MODE_INPUT, L.offsets, 1, L.N)
    xb[:, 40] = bf16_bits(np.full(xb.shape[0], 1000.0, np.float32))  # segment 1 only
    s1 = oracle.calibrate_act(xb, L.d.numpy(), MODE_INPUT, L.offsets, 1, L.N)
    assert np.array_equal(s0[0, [0, 2, 3]], s1[0, [0, 2, 3]])
    assert s1[0, 1, 0] > s0[0, 1, 0]


def test_weight_quant_invariants_per_segment():
    L = wl.outproj_layer("t", 16, 192, 40, 64, seed=3)
    d = L.d.numpy()
    w = wl.bits(L.w)
    wq, s_w = oracle.quantize_weight(w, d, MODE_INPUT, L.offsets)
    wf = bits_to_f32(w).astype(np.float64) * d[0].astype(np.float64)[None]
    for i in range(3):
        k0, k1 = L.offsets[i], L.offsets[i + 1]
        q = wq[:, k0:k1].astype(np.int64)
        assert np.all(np.abs(q).max(1) == 127)           # AMax element maps to 127
        s = s_w[i].astype(np.float64)[:, None]
        assert np.all(np.abs(s * q - wf[:, k0:k1]) <= s * (0.5 + 1e-5))
    # segment independence: scaling segment 2 leaves segments 0, 1 untouched
    w2 = w.copy()
    w2[:, 128:] = bf16_bits(bits_to_f32(w[:, 128:]) * 4)
    wq2, s_w2 = oracle.quantize_weight(w2, d, MODE_INPUT, L.offsets)
    assert np.array_equal(wq2[:, :128], wq[:, :128])
    assert np.array_equal(s_w2[:2], s_w[:2])


def test_weight_quant_output_groups_use_their_divisor():
    L = wl.adanorm_layer("t", 8, 64, 48, 3, seed=4, G=3)
    d = L.d.numpy().copy()
    wq, s_w = oracle.quantize_weight(wl.bits(L.w), d, MODE_OUTPUT, L.offsets, 3)
    d[1] *= 2.0   # only group 1's divisor changes -> only columns 16..31 move
    wq2, s_w2 = oracle.quantize_weight(wl.bits(L.w), d, MODE_OUTPUT, L.offsets, 3)
    assert np.array_equal(wq2[:16], wq[:16]) and np.array_equal(wq2[32:], wq[32:])
    assert np.array_equal(s_w2[0, 16:32], s_w[0, 16:32] * 2)


def test_zero_weight_column():
    w = np.zeros((3, 32), np.uint16)
    w[1] = bf16_bits(np.linspace(-1, 1, 32, dtype=np.float32))
    wq, s_w = oracle.quantize_weight(w)
    assert s_w[0, 0] == 1.0 and s_w[0, 2] == 1.0 and np.all(wq[[0, 2]] == 0)


# -------------------------------------------------------------- closed forms
def test_single_scale_reduction():
    """s+ = s- = s gives ordinary per-tensor quantization: q+ + q- equals
    sat(rne(x / s)), and acc+ + acc- equals the int GEMM of (q+ + q-)."""
    L = _c1_like(M=70, K=96, N=50, seed=5)
    xb = wl.bits(L.x)
    s = 2.0 ** -5
    s_act = np.array([[[s, s]]], np.float32)
    planes = oracle.quantize_act(xb, s_act)
    x = bits_to_f32(xb).astype(np.float64)
    q_single = np.clip(np.rint(x / s), -128, 127).astype(np.int64)
    q_sum = planes[0, 0].astype(np.int64) + planes[0, 1].astype(np.int64)
    assert np.array_equal(q_sum, q_single)
    wq, s_w = oracle.quantize_weight(wl.bits(L.w))
    acc = oracle.gemm_s32(planes, wq)
    ref = q_single @ wq.astype(np.int64).T
    assert np.array_equal(acc[0, 0].astype(np.int64) + acc[0, 1], ref)
    y = oracle.gemm(planes, wq, s_w, s_act)
    y_ref = s * s_w[0].astype(np.float64)[None] * ref
    assert np.allclose(y, y_ref, rtol=1e-6, atol=1e-6 * np.abs(y_ref).max())


def test_identity_weight_gives_dequantized_planes():
    L = _c1_like(M=33, K=48, N=48, seed=6)
    xb = wl.bits(L.x)
    s_act = oracle.calibrate_act(wl.bits(L.x_cal))
    planes = oracle.quantize_act(xb, s_act)
    wq = np.eye(48, dtype=np.int8)
    y = oracle.gemm(planes, wq, np.ones((1, 48), np.float32), s_act)
    sp, sm = float(s_act[0, 0, 0]), float(s_act[0, 0, 1])
    deq = (sp * planes[0, 0].astype(np.float64) + sm * planes[0, 1].astype(np.float64))
    assert np.array_equal(y, deq.astype(np.float32))


# ------------------------------------------------------ SegLinear identities
def test_output_segments_equal_concatenation():
    """Output-segmented Y = [X^W^_1, ..., X^W^_N] (bitwise): each segment with
    its own activation group equals a standalone one-segment layer."""
    L = wl.adanorm_layer("t", 40, 96, 3 * 48, 3, seed=7, G=3)
    d = L.d.numpy()
    xb, wb, bb = wl.bits(L.x), wl.bits(L.w), wl.bits(L.bias)
    full = oracle.layer(xb, wb, wl.bits(L.x_cal), d, bb, MODE_OUTPUT, L.offsets, 3)
    for j in range(3):
        n0, n1 = L.offsets[j], L.offsets[j + 1]
        part = oracle.layer(xb, wb[n0:n1], wl.bits(L.x_cal), d[j:j + 1], bb[n0:n1])
        assert np.array_equal(full["planes"][j], part["planes"][0])
        assert np.array_equal(full["s_act"][j], part["s_act"][0])
        assert np.array_equal(full["wq"][n0:n1], part["wq"])
        assert np.array_equal(full["y"][:, n0:n1], part["y"])


def rn_f32(v: Fraction) -> float:
    """Round an exact rational to the nearest fp32 value, ties to even
    (normal and subnormal range), written from the IEEE definition."""
    if v == 0:
        return 0.0
    sign = -1 if v < 0 else 1
    a = abs(v)
    m, e = math.frexp(float(a))          # float(a) is within one ulp: adjust
    e -= 1                               # a in [2^e, 2^(e+1)) after the fix-up
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (max(e, -126) - 23)
    return sign * float(round(a / q) * q)   # Fraction.__round__: half to even


def fma_f32(a: float, b: float, c: float) -> float:
    return rn_f32(Fraction(a) * Fraction(b) + Fraction(c))


def test_rn_f32_matches_numpy_rounding():
    rng = np.random.default_rng(0)
    for v in rng.standard_normal(2000) * np.exp2(rng.integers(-140, 100, 2000)):
        assert rn_f32(Fraction(float(v))) == float(np.float32(v))


@pytest.mark.parametrize("single", [False, True])
def test_one_segment_epilogue_order(single):
    """One K-segment: y = fma(c-, f(A-), fl(c+ f(A+))) + bias with
    c+- = fl(s_w s+-) (single scale: y = fl(c f(A)) + bias), recomputed in exact
    rational arithmetic from the oracle's own accumulators and scales."""
    L = _c1_like(M=6, K=96, N=7, seed=12)
    xb, wb = wl.bits(L.x), wl.bits(L.w)
    bias = (np.random.default_rng(4).standard_normal(7) * 0.1).astype(np.float32)
    bb = bf16_bits(bias)
    r = oracle.layer(xb, wb, wl.bits(L.x_cal), None, bb, single=single)
    acc = oracle.gemm_s32(r["planes"], r["wq"])
    b32 = bits_to_f32(bb)
    for m in range(6):
        for n in range(7):
            cp = float(np.float32(r["s_w"][0, n]) * np.float32(r["s_act"][0, 0, 0]))
            y = fma_f32(cp, float(np.float32(acc[0, 0, m, n])), 0.0)
            if not single:
                cm = float(np.float32(r["s_w"][0, n]) * np.float32(r["s_act"][0, 0, 1]))
                y = fma_f32(cm, float(np.float32(acc[0, 1, m, n])), y)
            y = rn_f32(Fraction(y) + Fraction(float(b32[n])))
            assert r["y"][m, n] == np.float32(y)


@pytest.mark.parametrize("single", [False, True])
def test_input_segments_equal_sum(single):
    """Input-segmented Y = sum_i X^_i W^_i: the int32 partials equal those of
    standalone per-segment products, and Y is the sum of the per-segment terms
    c+_i f(A+_i) + c-_i f(A-_i), c+-_i = fl(s_w[i] s+-_i), accumulated with one
    exactly rounded fused multiply-add per term, segments in ascending order,
    and the bias added last (recomputed here in exact rational arithmetic)."""
    L = wl.outproj_layer("t", 9, 128, 11, 32, seed=8)
    d = L.d.numpy()
    xb, wb, bb = wl.bits(L.x), wl.bits(L.w), wl.bits(L.bias)
    full = oracle.layer(xb, wb, wl.bits(L.x_cal), d, bb, MODE_INPUT, L.offsets, single=single)
    acc = oracle.gemm_s32(full["planes"], full["wq"], MODE_INPUT, L.offsets)
    for i in range(4):
        k0, k1 = L.offsets[i], L.offsets[i + 1]
        part = oracle.layer(np.ascontiguousarray(xb[:, k0:k1]),
                            np.ascontiguousarray(wb[:, k0:k1]),
                            np.ascontiguousarray(wl.bits(L.x_cal)[:, k0:k1]),
                            d[:, k0:k1], single=single)
        assert np.array_equal(part["planes"][0], full["planes"][0][:, :, k0:k1])
        assert np.array_equal(part["s_w"][0], full["s_w"][i])
        pacc = oracle.gemm_s32(part["planes"], part["wq"])
        assert np.array_equal(pacc[0], acc[i])
    bias = bits_to_f32(bb)
    s_act, s_w = full["s_act"], full["s_w"]
    for m in range(L.M):
        for n in range(L.N):
            y = 0.0
            for i in range(4):
                cp = float(np.float32(s_w[i, n]) * np.float32(s_act[0, i, 0]))
                cm = float(np.float32(s_w[i, n]) * np.float32(s_act[0, i, 1]))
                y = fma_f32(cp, float(np.float32(acc[i, 0, m, n])), y)
                if not single:
                    y = fma_f32(cm, float(np.float32(acc[i, 1, m, n])), y)
            y = rn_f32(Fraction(y) + Fraction(float(bias[n])))
            assert full["y"][m, n] == np.float32(y)


# ------------------------------------------- brute-force float64 reconstruction
# Three output groups need N >= 3 columns, so (MODE_OUTPUT, G = 3) leaves out N = 1.
_BF_GRID = [(mode, G, M, K, N)
            for mode, G in ((MODE_NONE, 1), (MODE_INPUT, 1), (MODE_OUTPUT, 1), (MODE_OUTPUT, 3))
            for M, K, N in ((1, 32, 1), (5, 96, 17), (17, 64, 9), (13, 96, 15))
            if not (G > 1 and N < G)]


@pytest.mark.parametrize("mode,G,M,K,N", _BF_GRID)
def test_bruteforce_dequantized_matmul(mode, G, M, K, N):
    """Y equals (s+ q+ + s- q-) (s_w q_w)^T + b evaluated in float64, within
    the fp32 rounding of the epilogue's few operations."""
    rng = np.random.default_rng(M * 1000 + K * 10 + N + mode)
    if mode == MODE_INPUT:
        offsets = [0, 32, K] if K > 32 else [0, K]
        if K == 96:
            offsets = [0, 32, 64, 96]
    elif mode == MODE_OUTPUT:
        cut = sorted(set([0, N // 3, (2 * N) // 3, N]))
        offsets = cut if G > 1 or len(cut) > 1 else [0, N]
        assert G == 1 or len(offsets) - 1 == G
    else:
        offsets = None
    n_seg = len(offsets) - 1 if offsets else 1
    S = n_seg if mode == MODE_INPUT else 1
    x = (rng.standard_normal((M, K)) * rng.uniform(0.1, 3, K)).astype(np.float32)
    x = np.where(rng.random((M, K)) < 0.5, np.minimum(x, 0) * 0.1, x).astype(np.float32)
    xb = bf16_bits(x)
    wb = bf16_bits((rng.standard_normal((N, K)) * 0.05).astype(np.float32))
    bb = bf16_bits((rng.standard_normal(N) * 0.1).astype(np.float32))
    d = rng.uniform(0.5, 2.0, (G, K)).astype(np.float32)
    out = oracle.layer(xb, wb, xb, d, bb, mode, offsets, G)
    planes, wq, s_w, s_act = out["planes"], out["wq"], out["s_w"], out["s_act"]
    koff = offsets if mode == MODE_INPUT else [0, K]
    noff = offsets if (mode == MODE_OUTPUT and G > 1) else [0, N]
    y_bf = np.zeros((M, N))
    mag = np.zeros((M, N))
    for gi in range(len(noff) - 1):
        n0, n1 = noff[gi], noff[gi + 1]
        for i in range(S):
            k0, k1 = koff[i], koff[i + 1]
            sp, sm = s_act[gi, i].astype(np.float64)
            xp = sp * planes[gi, 0][:, k0:k1].astype(np.float64)
            xm = sm * planes[gi, 1][:, k0:k1].astype(np.float64)
            wt = s_w[i, n0:n1].astype(np.float64)[:, None] * wq[n0:n1, k0:k1].astype(np.float64)
            y_bf[:, n0:n1] += xp @ wt.T + xm @ wt.T
            mag[:, n0:n1] += np.abs(xp @ wt.T) + np.abs(xm @ wt.T)
    b = bits_to_f32(bb).astype(np.float64)[None]
    y_bf += b
    mag += np.abs(b) + 1e-30
    assert np.all(np.abs(out["y"] - y_bf) <= 1e-6 * mag)


# ---------------------------------------------------------- qualitative claim
def test_dualscale_beats_single_scale_on_gelu_data():
    """DualScale lowers the output error on GELU-skewed activations compared
    with one symmetric per-tensor scale ("SegQuant" papernotes.org, section
    DualScale; author page section 3)."""
    L = wl.gelu_layer("t", 128, 256, 64, seed=9)
    xb, wb = wl.bits(L.x), wl.bits(L.w)
    x = bits_to_f32(xb).astype(np.float64)
    w = bits_to_f32(wb).astype(np.float64)
    y_true = x @ w.T
    dual = oracle.layer(xb, wb, wl.bits(L.x_cal))
    xc = bits_to_f32(wl.bits(L.x_cal))
    s = max(xc.max(), -xc.min()) / 127.0
    single_s = np.array([[[s, s]]], np.float32)
    planes = oracle.quantize_act(xb, single_s)
    y_single = oracle.gemm(planes, dual["wq"], dual["s_w"], single_s)
    e_dual = np.linalg.norm(dual["y"] - y_true) / np.linalg.norm(y_true)
    e_single = np.linalg.norm(y_single - y_true) / np.linalg.norm(y_true)
    assert e_dual < e_single


def test_row_subset_matches_full():
    L = _c1_like(M=50, K=64, N=20, seed=10)
    out = oracle.layer(wl.bits(L.x), wl.bits(L.w), wl.bits(L.x_cal), threads=2)
    rows = [0, 7, 49, 13]
    y = oracle.gemm(out["planes"], out["wq"], out["s_w"], out["s_act"], rows=rows, threads=3)
    assert np.array_equal(y, out["y"][rows])
    acc = oracle.gemm_s32(out["planes"], out["wq"], rows=rows)
    assert np.array_equal(acc, oracle.gemm_s32(out["planes"], out["wq"])[:, :, rows])


def test_invalid_segments_rejected():
    x = bf16_bits(np.ones((2, 64), np.float32))
    with pytest.raises(ValueError):
        oracle.calibrate_act(x, None, MODE_INPUT, [0, 40, 30, 64])
    with pytest.raises(ValueError):
        oracle.calibrate_act(x, None, MODE_INPUT, [0, 32, 60])


# ------------------------------------------------ single-scale (adaptive) mode
def test_worked_single_scale(golden_dir):
    fx = read_fixture(golden_dir, "single_scale_worked.txt")
    kv = dict((k, v) for k, v in fx if k != "case")
    s = oracle.calibrate_act(bf16_bits(np.array([parse_floats(kv["calib"])], np.float32)),
                             single=True)
    assert s[0, 0].tolist() == [float(kv["s"])] * 2
    s2 = oracle.calibrate_act(bf16_bits(np.array([parse_floats(kv["calib2"])], np.float32)),
                              single=True)
    assert s2[0, 0].tolist() == [float(kv["s2"])] * 2
    cases = [v.split() for k, v in fx if k == "case"]
    xs = np.array([float(c[0]) for c in cases], np.float32)[None]
    planes = oracle.quantize_act(bf16_bits(xs), s, single=True)
    assert planes.shape[1] == 1
    assert planes[0, 0, 0].tolist() == [int(c[1]) for c in cases]


def test_single_scale_every_bf16_value():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    s_act = np.array([[[1 / 64, 1 / 64]]], np.float32)
    planes = oracle.quantize_act(allbits, s_act, single=True)
    xs = bits_to_f32(allbits.reshape(-1))
    exp = []
    for x in xs:
        x = float(x)
        if math.isnan(x):
            exp.append(0)
        elif math.isinf(x):
            exp.append(127 if x > 0 else -128)
        else:
            exp.append(max(-128, min(127, rne_fraction(Fraction(x) * 64))))
    assert planes[0, 0].reshape(-1).tolist() == exp


def test_single_scale_is_dualscale_with_equal_steps():
    """Single-scale planes are X^+ + X^- of the DualScale quantizer run with
    s+ = s- = s, and its accumulator is A+ + A- (bit-exact)."""
    L = wl.outproj_layer("t", 57, 192, 70, 64, seed=21)
    d = L.d.numpy()
    xb, wb = wl.bits(L.x), wl.bits(L.w)
    s1 = oracle.calibrate_act(wl.bits(L.x_cal), d, MODE_INPUT, L.offsets, single=True)
    assert np.array_equal(s1[..., 0], s1[..., 1])
    p1 = oracle.quantize_act(xb, s1, d, MODE_INPUT, L.offsets, single=True)
    p2 = oracle.quantize_act(xb, s1, d, MODE_INPUT, L.offsets)
    assert np.array_equal(p1[:, 0].astype(np.int16), p2[:, 0].astype(np.int16) + p2[:, 1])
    wq, _ = oracle.quantize_weight(wb, d, MODE_INPUT, L.offsets)
    a1 = oracle.gemm_s32(p1, wq, MODE_INPUT, L.offsets)
    a2 = oracle.gemm_s32(p2, wq, MODE_INPUT, L.offsets)
    assert np.array_equal(a1[:, 0].astype(np.int64), a2[:, 0].astype(np.int64) + a2[:, 1])


@pytest.mark.parametrize("mode,G", [(MODE_NONE, 1), (MODE_INPUT, 1), (MODE_OUTPUT, 3)])
def test_single_scale_dequantized_matmul(mode, G):
    rng = np.random.default_rng(31 + mode)
    M, K, N = 13, 96, 15
    offsets = {MODE_NONE: None, MODE_INPUT: [0, 32, 64, 96], MODE_OUTPUT: [0, 5, 10, 15]}[mode]
    x = (rng.standard_normal((M, K)) * rng.uniform(0.1, 3, K)).astype(np.float32)
    xb = bf16_bits(x)
    wb = bf16_bits((rng.standard_normal((N, K)) * 0.05).astype(np.float32))
    bb = bf16_bits((rng.standard_normal(N) * 0.1).astype(np.float32))
    d = rng.uniform(0.5, 2.0, (G, K)).astype(np.float32)
    out = oracle.layer(xb, wb, xb, d, bb, mode, offsets, G, single=True)
    planes, wq, s_w, s_act = out["planes"], out["wq"], out["s_w"], out["s_act"]
    assert planes.shape[1] == 1
    koff = offsets if mode == MODE_INPUT else [0, K]
    noff = offsets if mode == MODE_OUTPUT else [0, N]
    S = len(koff) - 1
    y_bf = np.zeros((M, N))
    mag = np.zeros((M, N))
    for gi in range(len(noff) - 1):
        n0, n1 = noff[gi], noff[gi + 1]
        gg = gi if G > 1 else 0
        for i in range(S):
            k0, k1 = koff[i], koff[i + 1]
            xq = float(s_act[gg, i, 0]) * planes[gg, 0][:, k0:k1].astype(np.float64)
            wt = s_w[i, n0:n1].astype(np.float64)[:, None] * wq[n0:n1, k0:k1].astype(np.float64)
            y_bf[:, n0:n1] += xq @ wt.T
            mag[:, n0:n1] += np.abs(xq @ wt.T)
    b = bits_to_f32(bb).astype(np.float64)[None]
    y_bf += b
    mag += np.abs(b) + 1e-30
    assert np.all(np.abs(out["y"] - y_bf) <= 1e-6 * mag)
