"""Parity of the CUDA path against the CPU oracle on the same seeded inputs.

Bar (as fixed for this method): int8 planes, int8 weights, the scales that
come out of calibration and the int32 accumulators are bit-exact; fp32 output
within max |y - r| / (|r| + 1e-3 rms(r)) <= 1e-3.  The epilogue runs the
oracle's fp32 operations in the oracle's order (a fused multiply-add per term,
from the bias) for one and for several K-segments, so the fp32 output is
bit-exact and the bf16 output equals RNE_bf16(oracle fp32) as well.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import workloads as wl

from parity import (bf16_ulp_diff, gpu_run, oracle_acc, oracle_prep, oracle_y, rel_err_floor, sample_rows, segments)

pytestmark = pytest.mark.gpu
FP32_TOL = 1e-3


def _input_layer_mixed():
    L = wl.outproj_layer("mixed", 300, 416, 264, 32, seed=11)
    L.offsets = [0, 64, 96, 224, 416]   # widths 64, 32, 128, 192
    return L


SMALL = {
    "none_tails": lambda: wl.gelu_layer("none", 300, 416, 520, seed=1, bias=True),
    "none_tiny": lambda: wl.gelu_layer("tiny", 1, 16, 8, seed=2, bias=True),
    "none_ragged": lambda: wl.gelu_layer("rag", 5, 48, 13, seed=3, bias=True),
    "none_k_tail": lambda: wl.gelu_layer("ktail", 129, 144, 300, seed=4, bias=True),
    "input_heads": lambda: wl.outproj_layer("heads", 300, 448, 264, 64, seed=5),
    "input_mixed": _input_layer_mixed,
    "input_wide": lambda: wl.outproj_layer("wide", 130, 1024, 136, 512, seed=6),
    # N = 261: the last 8-column store of a row crosses N (element-wise tail)
    "input_odd_n": lambda: wl.outproj_layer("oddn", 150, 256, 261, 64, seed=14),
    # the most segments a table may hold (SQ_MAX_SEGMENTS = 64)
    "input_max_segments": lambda: wl.outproj_layer("maxin", 130, 2048, 136, 32, seed=12),
    "output_max_segments": lambda: wl.adanorm_layer("maxout", 130, 256, 64 * 9, 64, seed=13, G=1),
    "output_g1": lambda: wl.adanorm_layer("o1", 200, 256, 768, 3, seed=7, G=1),
    "output_g3": lambda: wl.adanorm_layer("o3", 200, 256, 768, 3, seed=8, G=3),
    "output_g2_bn128": lambda: wl.adanorm_layer("o2", 130, 128, 256, 2, seed=9, G=2),
    "qkv_g3": lambda: wl.qkv_layer("qkv", 257, 192, 384, 3, seed=10, G=3),
}


def _check_layer(L, full_rows=True):
    prep = oracle_prep(L)
    g = gpu_run(L, out_dtype=torch.float32, s32=True)
    assert np.array_equal(g["s_act"].cpu().numpy(), prep["s_act"])
    assert np.array_equal(g["wq"].cpu().numpy(), prep["wq"])
    assert np.array_equal(g["s_w"].cpu().numpy(), prep["s_w"])
    assert np.array_equal(g["planes"].cpu().numpy(), prep["planes"])
    acc = oracle_acc(L, prep)
    assert np.array_equal(g["acc"].cpu().numpy(), acc)
    r = oracle_y(L, prep)
    y = g["y"].cpu().numpy()
    assert rel_err_floor(y, r) <= FP32_TOL
    assert np.array_equal(y, r)              # same fp32 operations, same order
    gb = gpu_run(L, out_dtype=torch.bfloat16)
    assert bf16_ulp_diff(gb["y"], r) == 0    # RNE of the same fp32 value


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_layers_bitexact(name):
    _check_layer(SMALL[name]())


def test_every_bf16_value_quantizes_like_oracle():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    s_act = np.array([[[1 / 64, 1 / 512]]], np.float32)
    ref = oracle.quantize_act(allbits, s_act)
    x = torch.from_numpy(allbits.view(np.int16)).view(torch.bfloat16).cuda()
    planes = torch.empty(1, 2, 256, 256, dtype=torch.int8, device="cuda")
    B.sq_quantize_act(x, None, torch.from_numpy(s_act).cuda(), B.Segments(), planes)
    assert np.array_equal(planes.cpu().numpy(), ref)


_NP2_STEPS = [(float.fromhex("0x1.fd0eb8p-8"), float.fromhex("0x1.0adc5p-7")),
              (float.fromhex("0x1.945622p-6"), float.fromhex("0x1.0624dcp-8")),
              (float.fromhex("0x1.1cf06ap-8"), float.fromhex("0x1.fffffep-6")),
              (0.0123457, 0.000731), (0.2718, 0.0031416), (0.00057, 0.0419)]


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("with_d", [False, True])
def test_every_bf16_value_at_non_power_of_two_steps(with_d, single, fp8):
    """Every bf16 pattern at steps that are not powers of two, where the form of
    the quotient decides the code: the kernel's corrected reciprocal must give
    the oracle's rne(fl(fl(x/d)/s)) (FP8: e4m3(fl(fl(x/d)/s))) bit for bit.
    With a divisor, every one of the 256 channels has its own d."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    x = torch.from_numpy(allbits.view(np.int16)).view(torch.bfloat16).cuda()
    d = None
    if with_d:
        d = np.exp(np.random.default_rng(5).uniform(-4, 4, (1, 256))).astype(np.float32)
        d[0, :4] = [3.0, 2.5, 0.7071068, 1.0]
    P = 1 if single else 2
    flags = (B.SQ_FLAG_SINGLE_SCALE if single else 0) | (B.SQ_FLAG_FP8 if fp8 else 0)
    for sp, sm in _NP2_STEPS:
        if single:
            sm = sp
        s_act = np.array([[[sp, sm]]], np.float32)
        if fp8:
            ref = oracle.quantize_act_fp8(allbits, s_act, d=d, single=single).view(np.int8)
        else:
            ref = oracle.quantize_act(allbits, s_act, d=d, single=single)
        planes = torch.empty(1, P, 256, 256, dtype=torch.int8, device="cuda")
        B.sq_quantize_act(x, None if d is None else torch.from_numpy(d).cuda(),
                          torch.from_numpy(s_act).cuda(), B.Segments(flags=flags), planes)
        assert np.array_equal(planes.cpu().numpy(), ref), (sp, sm)


@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("layout", ["wide", "narrow"])
def test_uncorrected_codes_only_where_exact(layout, single):
    """The quantizer skips the quotient's correction for a 256-channel column
    block only after a block-wide test of the step pair of every K-segment in
    it.  Every segment holds every bf16 value; some step pairs are ones under
    which the uncorrected codes would differ from rne(fl(x/s)) for some input
    (constructed by a search), beside ordinary ones.  "wide": four 256-wide
    segments (one per column block, segments 0 and 2 with such steps);
    "narrow": eight 64-wide segments, the first column block with one such
    step among four, the second with none.  Every plane equals the oracle's."""
    from correction_free import forms_agree_everywhere, steps_where_forms_differ
    bad = steps_where_forms_differ(2, seed=11)
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    if layout == "wide":
        pairs = [(bad[0], 1 / 512), (1 / 64, 1 / 128), (0.0123457, bad[1]), (0.2718, 0.0031416)]
        xb = np.tile(allbits.reshape(256, 256), (1, 4))
        offsets = [0, 256, 512, 768, 1024]
    else:
        pairs = [(1 / 64, 1 / 128), (0.0123457, bad[1]), (0.2718, 0.0031416), (1 / 32, 0.75),
                 (0.00057, 0.0419), (1 / 64, 1 / 512), (0.5, 0.25), (0.0123457, 0.000731)]
        xb = np.tile(allbits.reshape(1024, 64), (1, 8))
        offsets = list(range(0, 513, 64))
    if single:
        pairs = [(a, a) for a, _ in pairs]
        if layout == "narrow":
            pairs[1] = (bad[1], bad[1])
    dangerous = [(a, b) for a, b in pairs if a in bad or b in bad]
    assert dangerous
    assert not any(forms_agree_everywhere(np.float32(a), np.float32(b)) for a, b in dangerous)
    xb = np.ascontiguousarray(xb)
    M, K = xb.shape
    s_act = np.array([pairs], np.float32)
    ref = oracle.quantize_act(xb, s_act, mode=oracle.MODE_INPUT, offsets=offsets, G=1,
                              single=single)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    flags = B.SQ_FLAG_SINGLE_SCALE if single else 0
    seg = B.Segments(B.SQ_SEG_INPUT, offsets, 1, flags=flags)
    planes = torch.empty(1, seg.P, M, K, dtype=torch.int8, device="cuda")
    B.sq_quantize_act(x, None, torch.from_numpy(s_act).cuda(), seg, planes)
    assert np.array_equal(planes.cpu().numpy(), ref)


@pytest.mark.parametrize("kind", ["positive", "negative", "zero", "nan_and_inf", "mixed"])
def test_calibration_degenerate_slices_on_gpu(kind):
    """AMax calibration on the GPU equals the oracle's, bit for bit, including
    one-sided, all-zero and NaN/Inf slices (R5, R6)."""
    rng = np.random.default_rng(17)
    x = rng.standard_normal((5, 64)).astype(np.float32)
    if kind == "positive":
        x = np.abs(x)
    elif kind == "negative":
        x = -np.abs(x)
    elif kind == "zero":
        x = np.zeros_like(x)
    elif kind == "nan_and_inf":
        x[0, 3] = np.nan
        x[2, 7] = np.inf
        x[4, 9] = -np.inf
    xt = torch.from_numpy(x).to(torch.bfloat16)
    bits = xt.view(torch.int16).numpy().view(np.uint16)
    d = rng.uniform(0.5, 2.0, (1, 64)).astype(np.float32)
    for seg, mode, off in ((B.Segments(), oracle.MODE_NONE, None),
                           (B.Segments(B.SQ_SEG_INPUT, [0, 32, 64], 1), oracle.MODE_INPUT,
                            [0, 32, 64])):
        ref = oracle.calibrate_act(bits, d, mode, off, 1, 0)
        s_act = torch.empty(1, seg.S, 2, device="cuda")
        B.sq_calibrate_act(xt.cuda(), torch.from_numpy(d).cuda(), seg, s_act)
        assert np.array_equal(s_act.cpu().numpy(), ref)


def test_strided_activation_rows():
    """ldx > K: the activation is a column slice of a wider tensor."""
    L = wl.gelu_layer("ld", 70, 96, 40, seed=12, bias=True)
    wide = torch.zeros(70, 160, dtype=torch.bfloat16)
    wide[:, 32:128] = L.x
    xg = wide.cuda()[:, 32:128]
    s_act = oracle.calibrate_act(wl.bits(L.x_cal))
    ref = oracle.quantize_act(wl.bits(L.x), s_act)
    planes = torch.empty(1, 2, 70, 96, dtype=torch.int8, device="cuda")
    B.sq_quantize_act(xg, None, torch.from_numpy(s_act).cuda(), B.Segments(), planes)
    assert np.array_equal(planes.cpu().numpy(), ref)


def test_empty_batch_is_noop():
    L = wl.gelu_layer("e", 4, 32, 16, seed=13)
    seg = B.Segments()
    planes = torch.empty(1, 2, 0, 32, dtype=torch.int8, device="cuda")
    x = torch.empty(0, 32, dtype=torch.bfloat16, device="cuda")
    s_act = torch.ones(1, 1, 2, device="cuda")
    B.sq_quantize_act(x, None, s_act, seg, planes)
    y = torch.empty(0, 16, dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros(16, 32, dtype=torch.int8, device="cuda")
    B.sq_dualscale_seglinear_gemm(planes, wq, torch.ones(1, 16, device="cuda"), s_act, None, y,
                                  seg)
    torch.cuda.synchronize()


def test_output_segments_equal_separate_calls_on_gpu():
    """SegLinear output identity on the device: one G = 3 call equals three
    single-segment calls on the same planes and weights, bit for bit."""
    L = wl.adanorm_layer("o3", 260, 256, 768, 3, seed=14, G=3)
    g = gpu_run(L, out_dtype=torch.float32)
    for j in range(3):
        n0, n1 = L.offsets[j], L.offsets[j + 1]
        y = torch.empty(L.M, n1 - n0, dtype=torch.float32, device="cuda")
        B.sq_dualscale_seglinear_gemm(g["planes"][j:j + 1].contiguous(),
                                      g["wq"][n0:n1].contiguous(),
                                      g["s_w"][:, n0:n1].contiguous(),
                                      g["s_act"][j:j + 1].contiguous(),
                                      L.bias[n0:n1].cuda(), y, B.Segments())
        assert torch.equal(y, g["y"][:, n0:n1])


def test_input_segments_sum_on_gpu():
    """SegLinear input identity on the device: the int32 partials of each
    K-segment equal a standalone one-segment call on that slice."""
    L = wl.outproj_layer("heads", 200, 256, 136, 64, seed=15)
    g = gpu_run(L, out_dtype=torch.float32, s32=True)
    for i in range(4):
        k0, k1 = L.offsets[i], L.offsets[i + 1]
        acc = torch.empty(1, 2, L.M, L.N, dtype=torch.int32, device="cuda")
        B.sq_debug_gemm_s32(g["planes"][:, :, :, k0:k1].contiguous(),
                            g["wq"][:, k0:k1].contiguous(), B.Segments(), acc)
        assert torch.equal(acc[0], g["acc"][i])


FULL = ["c1_tiny_dualscale", "c2_sd35_adanorm", "c3_sd35_attn_out", "c4_sd35_ffn",
        "c5_flux_block", "c5_flux_adanorm_m2"]


@pytest.mark.parametrize("cfg", FULL)
def test_full_size_configs_sampled_rows(cfg):
    """Full-size workload layers: planes, weights and scales compared in full,
    outputs on every row of the first and last M tile plus a strided sample."""
    for L in wl.config_layers(cfg, seed=0):
        prep = oracle_prep(L)
        g = gpu_run(L, out_dtype=torch.bfloat16)
        assert np.array_equal(g["s_act"].cpu().numpy(), prep["s_act"])
        assert np.array_equal(g["wq"].cpu().numpy(), prep["wq"])
        assert np.array_equal(g["s_w"].cpu().numpy(), prep["s_w"])
        assert np.array_equal(g["planes"].cpu().numpy(), prep["planes"])
        rows = sample_rows(L.M)
        r = oracle_y(L, prep, rows=rows)
        yb = g["y"][torch.from_numpy(rows).cuda()]
        assert bf16_ulp_diff(yb, r) == 0
        gf = gpu_run(L, out_dtype=torch.float32)
        assert np.array_equal(gf["y"][torch.from_numpy(rows).cuda()].cpu().numpy(), r)
        del g, gf
        torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", ["c2_sd35_adanorm", "c5_flux_block", "c5_flux_adanorm_m2"])
def test_full_size_shared_activation_group(cfg):
    """The output-segmented layers with one shared activation group (G = 1,
    one X^ for every output segment, the pages' output-segmented formula) at
    full size: planes in full, int32 accumulators and outputs on the sampled
    rows."""
    for L in wl.config_layers(cfg, seed=0, G_output=1):
        if L.mode != wl.MODE_OUTPUT:
            continue
        assert L.G == 1
        prep = oracle_prep(L)
        g = gpu_run(L, out_dtype=torch.float32, s32=True)
        assert np.array_equal(g["s_act"].cpu().numpy(), prep["s_act"])
        assert np.array_equal(g["wq"].cpu().numpy(), prep["wq"])
        assert np.array_equal(g["planes"].cpu().numpy(), prep["planes"])
        rows = sample_rows(L.M)
        idx = torch.from_numpy(rows).cuda()
        assert np.array_equal(g["acc"][:, :, idx].cpu().numpy(), oracle_acc(L, prep, rows=rows))
        assert np.array_equal(g["y"][idx].cpu().numpy(), oracle_y(L, prep, rows=rows))
        del g
        torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", FULL)
def test_full_size_int32_accumulators_sampled_rows(cfg):
    """The raw int32 accumulators of every full-size workload layer, per
    K-segment and polarity, against the oracle's int32 products on the sampled
    rows: above 2^24 the fp32 output rounds the accumulator, so an off-by-one
    there could hide behind an output that still matches (K = 6144 allows
    |A| up to 128 * 127 * 6144, about 10^8)."""
    for L in wl.config_layers(cfg, seed=0):
        prep = oracle_prep(L)
        g = gpu_run(L, out_dtype=torch.float32, s32=True)
        assert np.array_equal(g["planes"].cpu().numpy(), prep["planes"])
        rows = sample_rows(L.M)
        ref = oracle_acc(L, prep, rows=rows)
        got = g["acc"][:, :, torch.from_numpy(rows).cuda()].cpu().numpy()
        assert got.shape == ref.shape
        assert np.array_equal(got, ref), L.name
        del g
        torch.cuda.empty_cache()


def _integer_layer(widths, seed, single):
    """Input-segmented layer whose quantization is the identity: integer
    activations in [-128, 127]; every segment's calibration slice spans
    [-128, 127] (s+ = 127/127, s- = 128/128), or [-127, 127] for the single
    step (s = 127/127); integer weights whose rows reach 127 in every segment
    (s_w = 1).  Rows 0 and 1 are all 127 and all -128, weight rows 0 and 1 all
    127 and all -127: their products are the largest accumulators a segment
    of that width can hold.  Every fp32 sum stays below 2^24, so Y is the
    exact integer product in any summation order."""
    g = torch.Generator().manual_seed(seed)
    K = sum(widths)
    M, N = 130, 136
    offsets = [0] + [int(v) for v in np.cumsum(widths)]
    x = torch.randint(-128, 128, (M, K), generator=g).float()
    x[0] = 127.0
    x[1] = -128.0
    x_cal = x[:2].clone()
    if single:
        x_cal[1] = -127.0
    w = torch.randint(-127, 128, (N, K), generator=g).float()
    w[:, offsets[:-1]] = 127.0
    w[0] = 127.0
    w[1] = -127.0
    L = wl.Layer("int", x.to(torch.bfloat16), x_cal.to(torch.bfloat16), w.to(torch.bfloat16),
                 None, None, wl.MODE_INPUT, offsets, 1)
    exact = x.double().numpy() @ w.double().numpy().T
    return L, exact


@pytest.mark.parametrize("widths", [[256, 256], [256, 288], [32, 256, 96]])
@pytest.mark.parametrize("single", [False, True])
def test_input_segments_extreme_accumulators_exact(widths, single):
    """The per-segment drains at the largest accumulators a segment allows
    (|A| up to w * 128 * 127 for width w, beyond 2^22 for w = 288): with unit
    scales every step is exact, so Y must equal the integer product."""
    L, exact = _integer_layer(widths, sum(widths) + single, single)
    prep = oracle_prep(L, single)
    assert np.all(prep["s_act"] == 1.0) and np.all(prep["s_w"] == 1.0)
    g = gpu_run(L, out_dtype=torch.float32, s32=True, single=single)
    assert np.array_equal(g["acc"].cpu().numpy(), oracle_acc(L, prep))
    y = g["y"].cpu().numpy()
    assert np.array_equal(y.astype(np.float64), exact)
    assert np.array_equal(oracle_y(L, prep).astype(np.float64), exact)
