"""Pins of the FP8 (E4M3) oracle: the code format against torch's float8_e4m3fn
(an independent library implementation of the same format) on every code and
every in-range bf16 value, a hand-derived worked example of the DualScale FP8
quantizer, exact rational accumulation of E4M3 products, and a float64
dequantize-then-multiply of a whole FP8 layer."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from test_oracle import bf16_bits, parse_floats, read_fixture


def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.isnan(ours).sum() == 2          # 0x7F and 0xFF
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert ours[0x7E] == 448.0 and ours[0x08] == 2.0 ** -6 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_matches_torch_on_every_bf16_in_range():
    b = np.arange(65536, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    ok = np.isfinite(f) & (np.abs(f) <= 448)
    ref = torch.from_numpy(f[ok].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(f[ok]), ref)


def test_e4m3_encode_matches_torch_on_random_fp32():
    rng = np.random.default_rng(5)
    mag = np.exp2(rng.uniform(-14, 8.8, 200000)).astype(np.float32)
    v = (mag * rng.choice([-1, 1], mag.size)).astype(np.float32)
    v = v[np.abs(v) <= 448]
    ref = torch.from_numpy(v.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


def test_e4m3_saturation_nan_and_signed_zero():
    v = np.array([448.0, 463.9, 464.0, 1e30, np.inf, -500.0, -np.inf, np.nan, 0.0, -0.0,
                  -1e-30], np.float32)
    assert oracle.e4m3_encode(v).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F,
                                              0x00, 0x80, 0x80]


def test_fp8_worked_example(golden_dir):
    kv = dict(read_fixture(golden_dir, "fp8_quant_worked.txt"))
    cal_part, sp_part, sm_part = kv["calib"].split("|")
    cal = np.array(parse_floats(cal_part), np.float32)[None]
    s = oracle.calibrate_act_fp8(bf16_bits(cal))
    assert s[0, 0].tolist() == [float(sp_part.split()[1]), float(sm_part.split()[1])]
    x = np.array(parse_floats(kv["x"]), np.float32)[None]
    planes = oracle.quantize_act_fp8(bf16_bits(x), s)
    assert planes[0, 0, 0].tolist() == [int(t, 16) for t in kv["plus"].split()]
    assert planes[0, 1, 0].tolist() == [int(t, 16) for t in kv["minus"].split()]


def test_fp8_single_scale_plane_takes_the_branch_code():
    x = np.array([[3.0, -2.0, 0.0, -0.0, np.nan]], np.float32)
    s = oracle.calibrate_act_fp8(bf16_bits(np.array([[4.0, -2.0]], np.float32)), single=True)
    assert s[0, 0].tolist() == [float(np.float32(4.0) / np.float32(448.0))] * 2
    p1 = oracle.quantize_act_fp8(bf16_bits(x), s, single=True)
    p2 = oracle.quantize_act_fp8(bf16_bits(x), s)
    assert p1[0, 0, 0].tolist() == [int(v) for v in np.where(x[0] < 0, p2[0, 1, 0], p2[0, 0, 0])]
    assert p1[0, 0, 0, 4] == 0 and p2[0, 0, 0, 4] == 0 and p2[0, 1, 0, 4] == 0  # NaN


def test_fp8_accumulators_are_exact_sums():
    rng = np.random.default_rng(11)
    planes = rng.integers(0, 256, (1, 2, 3, 40)).astype(np.uint8)
    planes[planes & 0x7F == 0x7F] = 0                  # no NaN codes
    wq = rng.integers(0, 256, (5, 40)).astype(np.uint8)
    wq[wq & 0x7F == 0x7F] = 0
    acc = oracle.gemm_fp8_acc(planes, wq)
    dec = lambda c: Fraction(float(oracle.e4m3_decode(np.array([c], np.uint8))[0]))
    for pl in range(2):
        for m in range(3):
            for n in range(5):
                exact = sum(dec(planes[0, pl, m, k]) * dec(wq[n, k]) for k in range(40))
                assert acc[0, pl, m, n] == np.float32(float(exact))


def test_fp8_layer_equals_float64_dequantized_product():
    rng = np.random.default_rng(3)
    M, K, N = 6, 64, 7
    x = (rng.standard_normal((M, K)) * 2).astype(np.float32)
    xc = (rng.standard_normal((32, K)) * 2).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    r = oracle.layer_fp8(bf16_bits(x), bf16_bits(w), bf16_bits(xc))
    s = r["s_act"][0, 0].astype(np.float64)
    xt = s[0] * oracle.e4m3_decode(r["planes"][0, 0]) + s[1] * oracle.e4m3_decode(r["planes"][0, 1])
    wt = r["s_w"][0][:, None].astype(np.float64) * oracle.e4m3_decode(r["wq"])
    ref = xt @ wt.T
    assert np.max(np.abs(r["y"] - ref)) <= 1e-5 * (np.abs(ref).max() + 1e-30)
    # and close to the unquantized product (FP8 keeps 3 mantissa bits)
    xb = (bf16_bits(x).astype(np.uint32) << 16).view(np.float32)
    wb = (bf16_bits(w).astype(np.uint32) << 16).view(np.float32)
    full = xb.astype(np.float64) @ wb.T.astype(np.float64)
    assert np.linalg.norm(r["y"] - full) <= 0.1 * np.linalg.norm(full)


def test_fp8_weights_hit_448_and_stay_within_half_a_quantum():
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((12, 80)) * 0.03).astype(np.float32)
    wq, s_w = oracle.quantize_weight_fp8(bf16_bits(w))
    vals = oracle.e4m3_decode(wq)
    wf = (bf16_bits(w).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(vals).max(axis=1) == 448.0)
    u = wf / s_w[0][:, None]
    quantum = np.exp2(np.floor(np.log2(np.maximum(np.abs(u), 2.0 ** -6))) - 3)
    assert np.all(np.abs(vals - u) <= quantum / 2 * (1 + 1e-6))


def test_fp8_weight_step_is_amax_over_448():
    """s_w = amax / 448 exactly: amax = 7/8 gives s_w = 2^-9, and the codes of
    w = 7/8, 7/16, -7/32, 1/64 are then e4m3 of 448, 224, -112, 8 (all exact)."""
    w = np.array([[0.875, 0.4375, -0.21875, 0.015625] + [0.0] * 12], np.float32)
    wq, s_w = oracle.quantize_weight_fp8(bf16_bits(w))
    assert s_w.tolist() == [[2.0 ** -9]]
    assert oracle.e4m3_decode(wq[0, :4]).tolist() == [448.0, 224.0, -112.0, 8.0]
