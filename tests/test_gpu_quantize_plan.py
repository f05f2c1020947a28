"""The quantize plan (sq_quantize_act_plan, sq_quantize_act_planned): for layers
with SmoothQuant divisors, a channel whose codes provably do not change may be
quantized without either quotient's correction.  The plan's bits must be the
verdicts of the numpy model of both forms (tests/correction_free.py), and the
planned planes must be the oracle's, bit for bit, for every bf16 input --
including channels whose divisors were constructed so that the uncorrected
forms would give a different code for some input (those a column block
patches, or keeps the corrections for)."""
import numpy as np
import pytest
import torch

import oracle
from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import workloads as wl

from correction_free import channel_passes_test_d, divisors_where_forms_differ
from parity import oracle_prep, segments

pytestmark = pytest.mark.gpu


def _plan_bits(plan, K):
    """[G][words] int32 words -> bool [G][K]."""
    w = plan.cpu().numpy().view(np.uint32)
    bits = (w[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(w.shape[0], -1)[:, :K].astype(bool)


def _steps_and_divisors(G, K, seed, dangerous_at=()):
    rng = np.random.default_rng(seed)
    s_act = np.exp2(rng.uniform(-9, 1, (G, 1, 2))).astype(np.float32)
    d = np.exp2(rng.uniform(-3, 3, (G, K))).astype(np.float32)
    for g, c in dangerous_at:
        s = float(s_act[g, 0, 0])
        d[g, c] = divisors_where_forms_differ(1, s, seed=seed + c)[0]
        s_act[g, 0, 1] = s_act[g, 0, 0]   # the constructed d fails on both sides
    return s_act, d


def test_plan_bits_equal_the_model():
    """Every channel's bit is the numpy model's verdict (both polarities, 768
    candidates), for random divisors and steps and for constructed ones."""
    G, K = 2, 320
    s_act, d = _steps_and_divisors(G, K, seed=5, dangerous_at=[(0, 3), (1, 300)])
    seg = B.Segments(B.SQ_SEG_NONE, None, 1) if G == 1 else B.Segments(
        B.SQ_SEG_OUTPUT, [0, 256, 512], G)
    plan = B.sq_quantize_act_plan(torch.from_numpy(d).cuda(), torch.from_numpy(s_act).cuda(), seg)
    got = _plan_bits(plan, K)
    want = np.array([[channel_passes_test_d(d[g, c], s_act[g, 0, 0], s_act[g, 0, 1])
                      for c in range(K)] for g in range(G)])
    assert not want[0, 3] and not want[1, 300]
    assert np.array_equal(got, want)
    words = plan.cpu().numpy().view(np.uint32)
    assert words[0, -1] >> (K % 32) == (1 << (32 - K % 32)) - 1   # padding channels set


FIX_MAX = 16   # left-out channels a 256-channel column block may patch


def _left_out_layout(layout):
    """K and the channels whose divisors are constructed to fail the test:
    "blocks": column block 0 leaves out one channel, block 1 sixteen (the
    patch list's capacity; one lane's eight channels among them), block 2
    seventeen (one more: the block keeps the corrections), block 3 none;
    "ragged": K = 320, one channel in the first block and one in the
    64-channel tail block."""
    if layout == "blocks":
        bad = ([7] + list(range(256, 264)) + [300, 333, 400, 401, 450, 480, 500, 511]
               + [512 + 15 * i for i in range(17)])
        return 1024, bad
    return 320, [7, 300]


def _layout_divisors(K, bad, s, seed):
    """Divisors that pass the plan's test everywhere except at `bad`, where
    they are ones under which some bf16 input's uncorrected codes differ."""
    rng = np.random.default_rng(seed)
    d = np.empty(K, np.float32)
    for c in range(K):
        while True:
            d[c] = np.float32(np.exp2(rng.uniform(-3, 3)))
            if channel_passes_test_d(d[c], s, s):
                break
    failing = divisors_where_forms_differ(3, s, seed=seed)
    for i, c in enumerate(bad):
        d[c] = failing[i % 3]
    return d[None, :]


@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("layout", ["blocks", "ragged"])
def test_planned_planes_equal_the_oracle_for_every_bf16_input(layout, single):
    """M = 65536 rows hold every bf16 value in every channel.  Column blocks
    whose plan leaves out at most FIX_MAX channels take the uncorrected codes
    and patch the left-out channels with the exact ones; a block with more
    keeps the corrections.  Every plane equals the oracle's and the unplanned
    kernel's, bit for bit."""
    K, bad = _left_out_layout(layout)
    s = np.float32(float.fromhex("0x1.0adc5p-7"))
    d = _layout_divisors(K, bad, s, seed=21)
    s_act = np.array([[[s, s]]], np.float32)
    bits_want = np.array([channel_passes_test_d(d[0, c], s, s) for c in range(K)])
    assert sorted(np.flatnonzero(~bits_want).tolist()) == sorted(bad)
    if layout == "blocks":
        per_block = [(~bits_want[b * 256:(b + 1) * 256]).sum() for b in range(4)]
        assert per_block == [1, FIX_MAX, FIX_MAX + 1, 0]
    M = 65536
    flags = B.SQ_FLAG_SINGLE_SCALE if single else 0
    seg = B.Segments(flags=flags)
    xb = np.ascontiguousarray(np.repeat(np.arange(M, dtype=np.uint32).astype(np.uint16)[:, None],
                                        K, axis=1))
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    dt, st = torch.from_numpy(d).cuda(), torch.from_numpy(s_act).cuda()
    plan = B.sq_quantize_act_plan(dt, st, seg)
    assert np.array_equal(_plan_bits(plan, K)[0], bits_want)
    planned = torch.empty(1, seg.P, M, K, dtype=torch.int8, device="cuda")
    plain = torch.empty_like(planned)
    B.sq_quantize_act(x, dt, st, seg, planned, plan=plan)
    B.sq_quantize_act(x, dt, st, seg, plain)
    ref = oracle.quantize_act(xb, s_act, d=d, single=single)
    assert np.array_equal(plain.cpu().numpy(), ref)
    assert np.array_equal(planned.cpu().numpy(), ref)


@pytest.mark.parametrize("cfg", ["c3_sd35_attn_out", "c2_sd35_adanorm"])
def test_planned_full_size_layers(cfg):
    """The SD3.5 layers with divisors at full size (input segments; output
    groups): planned planes equal the unplanned kernel's everywhere and the
    oracle's on the sampled rows' planes."""
    for L in wl.config_layers(cfg, seed=0):
        assert L.d is not None
        seg = segments(L)
        dev = torch.device("cuda")
        x, d = L.x.to(dev), L.d.to(dev)
        s_act = torch.empty(seg.n_groups, seg.S, 2, device=dev)
        B.sq_calibrate_act(L.x_cal.to(dev), d, seg, s_act)
        plan = B.sq_quantize_act_plan(d, s_act, seg)
        planned = torch.empty(seg.n_groups, 2, L.M, L.K, dtype=torch.int8, device=dev)
        plain = torch.empty_like(planned)
        B.sq_quantize_act(x, d, s_act, seg, planned, plan=plan)
        B.sq_quantize_act(x, d, s_act, seg, plain)
        assert torch.equal(planned, plain), L.name
        assert np.array_equal(planned.cpu().numpy(), oracle_prep(L)["planes"]), L.name
