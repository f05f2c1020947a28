"""Pins of the FFN activation the fused producer applies between fc1 and fc2
(bf16(gelu(bf16(y))), tanh approximation): each piece against the mathematics
in float64 within a stated bound, and the whole against torch's own GELU."""
import math

import numpy as np
import torch

import oracle


def _grid(lo, hi, n):
    return np.linspace(lo, hi, n, dtype=np.float64).astype(np.float32)


def test_exp_reduction_and_series_bound():
    # Cody-Waite reduction + degree-7 Taylor series on [0, 18]: within 0.75
    # units of 2^-23 relative (the final rounding alone takes up to 0.5).
    # Dropping the 1/7! term adds up to one more unit, a missing ln2 tail far
    # more, so either fails.
    z = np.concatenate([_grid(0.0, 18.0, 400001),
                        (np.arange(0, 27) * np.float32(math.log(2) / 2)).astype(np.float32)])
    e = oracle.gelu_parts(z)["exp"].astype(np.float64)
    ref = np.exp(z.astype(np.float64))
    assert np.max(np.abs(e - ref) / ref) <= 0.75 * 2.0 ** -23
    assert oracle.gelu_parts(np.float32([0.0]))["exp"][0] == 1.0


def test_tanh_bound_symmetry_and_saturation():
    u = _grid(-12.0, 12.0, 240001)
    t = oracle.gelu_parts(u)["tanh"]
    assert np.max(np.abs(t.astype(np.float64) - np.tanh(u.astype(np.float64)))) <= 2.0 ** -22
    assert np.array_equal(oracle.gelu_parts(-u)["tanh"], -t)          # odd, exactly
    assert oracle.gelu_parts(np.float32([0.0]))["tanh"][0] == 0.0
    assert np.all(oracle.gelu_parts(_grid(9.0, 50.0, 1001))["tanh"] == 1.0)


def _gelu64(x):
    x = x.astype(np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def test_gelu_against_float64_definition():
    # every finite bf16 value in [-30, 30] plus a dense fp32 grid; the error
    # bound allows for the cancellation in 1 + tanh for large negative x
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    xb = (bits.astype(np.uint32) << 16).view(np.float32)
    xb = xb[np.isfinite(xb) & (np.abs(xb) <= 30)]
    x = np.concatenate([xb, _grid(-20.0, 20.0, 100001)])
    g = oracle.gelu_parts(x)["gelu"].astype(np.float64)
    ref = _gelu64(x)
    assert np.all(np.abs(g - ref) <= 2.0 ** -20 * np.abs(ref) + 2.0 ** -22 * np.abs(x))
    assert oracle.gelu_parts(np.float32([0.0]))["gelu"][0] == 0.0
    big = np.float32([100.0, 1e10, -100.0, -1e10])
    gb = oracle.gelu_parts(big)["gelu"]
    assert gb[0] == 100.0 and gb[1] == np.float32(1e10) and gb[2] == 0.0 and gb[3] == 0.0


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(5)
    v = rng.standard_normal(200000).astype(np.float32) * np.float32(10.0) ** rng.integers(-20, 20, 200000).astype(np.float32)
    # exact ties, odd and even kept halves
    ties = ((rng.integers(0, 1 << 15, 5000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    v = np.concatenate([v, ties, np.float32([0.0, -0.0, 3.0e38, -3.0e38])])
    ours = oracle.gelu_parts(v)["bf16"]
    theirs = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_gelu_bf16_close_to_torch():
    """The whole activation against torch's tanh GELU on the same bf16 inputs:
    the same bf16 value almost everywhere, and never further apart than one
    bf16 ulp or 2^-21 (below x ~ -5 torch's fp32 tanh is exactly -1 and its
    GELU 0, while the true value is ~1e-7, far below any quantization step)."""
    rng = np.random.default_rng(6)
    y = (rng.standard_normal(300000) * 3.0).astype(np.float32)
    ours = oracle.gelu_bf16(y)
    xb = torch.from_numpy(y).to(torch.bfloat16)
    ref = torch.nn.functional.gelu(xb.float(), approximate="tanh").to(torch.bfloat16)
    theirs = ref.view(torch.int16).numpy().view(np.uint16)
    a = (ours.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    b = (theirs.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126))) - 7)
    assert np.all(np.abs(a - b) <= np.maximum(ulp, 2.0 ** -21))
    assert np.mean(ours == theirs) >= 0.99


def test_identities_of_the_branch_free_form():
    """The arithmetic facts the GPU's form of the same operations rests on,
    checked in IEEE fp32 (numpy): 2/d == 2 RN(1/d) for the divisors e + 1 in
    [2, e^18 + 1] (whole binades exhaustively, the rest sampled), and the
    integer read from the bits of 1.5 * 2^23 + v is rne(v) on [-128, 127]."""
    two, one = np.float32(2.0), np.float32(1.0)
    for lo in (2.0, 4.0, float(2 ** 25)):
        d = np.arange(np.float32(lo).view(np.int32), np.float32(2 * lo).view(np.int32),
                      dtype=np.int32).view(np.float32)
        assert np.array_equal(two / d, two * (one / d))
    rng = np.random.default_rng(7)
    d = np.exp(rng.uniform(np.log(2.0), np.log(math.exp(18) + 1), 2_000_000)).astype(np.float32)
    assert np.array_equal(two / d, two * (one / d))
    # rne on [-128, 127] by the bits of 1.5 * 2^23 + v: every half and a dense grid
    v = np.concatenate([np.arange(-256, 255, dtype=np.float32) / np.float32(2),
                        _grid(-128.0, 127.0, 1_000_001)])
    q = (v + np.float32(12582912.0)).view(np.int32) - 0x4B400000
    assert np.array_equal(q, np.rint(v).astype(np.int32))
    # the capped exponent and selected 1 give the same tanh as the branch
    u = _grid(-30.0, 30.0, 600001)
    a = np.abs(u)
    e = oracle.gelu_parts(np.float32(2.0) * np.minimum(a, np.float32(9.0)))["exp"]
    t = np.where(a < 9.0, one - two * (one / (e + one)), one).astype(np.float32)
    t = np.where(u < 0.0, -t, t)
    assert np.array_equal(t, oracle.gelu_parts(u)["tanh"])
