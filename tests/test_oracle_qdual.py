"""Pins for the oracle's DualScale quantizer at steps that are NOT powers of
two, where the way the quotient is formed decides the code.

The pages define Q_dual(x) = round(x/s-) for x < 0 and round(x/s+) for x >= 0
("SegQuant" author page, section 3; "SegQuant" papernotes.org notes, section
DualScale).  The reading pinned here: u = fl(x / d) (u = x without a
SmoothQuant divisor), v = fl(u / s) -- both fp32 IEEE divisions -- then round
half to even and saturate to the int8 code range.  A tie of v itself goes to
the even code (v is rounded twice: to fp32, then to an integer).

The expected codes never come from the oracle or from a floating-point
division: the quotient is rounded to fp32 here with exact integer arithmetic
(rn32_div below), which is itself checked against exact rational rounding.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
from test_oracle import bits_to_f32, read_fixture, rn_f32


# --------------------------------------------------------------- exact helper
def _decompose(a: np.ndarray):
    """Finite fp32 values as (sign, m, e) with |a| = m * 2^e, m an integer."""
    b = a.astype(np.float32).view(np.uint32).astype(np.int64)
    sign = (b >> 31) & 1
    E = (b >> 23) & 0xFF
    F = b & 0x7FFFFF
    m = np.where(E == 0, F, F | (1 << 23))
    e = np.where(E == 0, -149, E - 150)
    return sign, m, e


def rn32_div(a: np.ndarray, b: float) -> np.ndarray:
    """fl(a / b) for finite fp32 a and a positive normal fp32 b, computed with
    integers only: the quotient of the two significands, scaled by 2^39, is
    kept as integer part Q and remainder R; Q is rounded to 24 significant bits
    (ties to even, the remainder acting as sticky bit).  Quotients outside the
    normal range are returned as +-inf (overflow) or flagged by `tiny`."""
    a = np.asarray(a, np.float32)
    sa, ma, ea = _decompose(a)
    _, mb, eb = _decompose(np.array([b], np.float32))
    mb, eb = int(mb[0]), int(eb[0])
    num = ma << 39                       # ma < 2^24, so num < 2^63
    Q, R = num // mb, num % mb
    zero = ma == 0
    Qs = np.where(zero, 1, Q)
    L = np.frexp(Qs.astype(np.float64))[1].astype(np.int64)   # bit length, +-1
    L = np.where((Qs >> (L - 1)) == 0, L - 1, L)
    L = np.where((Qs >> L) != 0, L + 1, L)
    sh = L - 24                          # Q has >= 31 bits for every finite a != 0
    T = Qs >> sh
    rem = Qs & ((np.int64(1) << sh) - 1)
    half = np.int64(1) << (sh - 1)
    up = (rem > half) | ((rem == half) & ((R > 0) | ((T & 1) == 1)))
    T = T + up
    exp = sh + ea - eb - 39              # value = T * 2^exp, T <= 2^24
    top = exp + 23                       # binade exponent of the value
    mag = np.ldexp(T.astype(np.float64), exp.astype(np.int32))
    mag = np.where(zero, 0.0, mag)
    mag = np.where(top > 127, np.inf, mag)
    out = np.where(sa == 1, -mag, mag).astype(np.float32)
    tiny = (~zero) & (top < -126)
    return out, tiny


def test_rn32_div_agrees_with_exact_rational_rounding():
    rng = np.random.default_rng(7)
    nums = (rng.integers(0, 2 ** 32, 3000, dtype=np.uint64).astype(np.uint32)).view(np.float32)
    nums = nums[np.isfinite(nums)]
    for b in (np.float32(0.0078125), np.float32(3.0), np.float32(0.0116479),
              np.float32(float.fromhex("0x1.fffffep-3"))):
        got, tiny = rn32_div(nums, float(b))
        for a, g, t in zip(nums[:600], got[:600], tiny[:600]):
            q = Fraction(float(a)) / Fraction(float(b))
            if t or abs(q) > Fraction(float(np.finfo(np.float32).max)):
                continue
            assert float(g) == rn_f32(q), (float(a), float(b))


# ----------------------------------------------------------- expected codes
def expected_codes(x: np.ndarray, s_plus: float, s_minus: float, d: float = None):
    """X^+ and X^- codes of the reading, from rn32_div only."""
    x = np.asarray(x, np.float32)
    finite = np.isfinite(x)
    xf = np.where(finite, x, 0).astype(np.float32)
    if d is None:
        u = xf
    else:
        u, tiny_u = rn32_div(xf, d)
        assert not np.any(tiny_u & (xf != 0)), "inputs chosen so that x/d stays normal"
    vp, tiny_p = rn32_div(np.abs(u), s_plus)
    vm, tiny_m = rn32_div(np.abs(u), s_minus)
    # a quotient below the normal range is far below 1/2: code 0
    vp = np.where(tiny_p, 0, vp).astype(np.float64)
    vm = np.where(tiny_m, 0, vm).astype(np.float64)
    neg = x < 0
    pos = x >= 0            # NaN is neither; -0.0 is positive
    qp = np.where(pos, np.minimum(np.rint(vp), 127), 0)
    qm = np.where(neg, -np.minimum(np.rint(vm), 128), 0)
    qp = np.where(np.isposinf(x), 127, qp)
    qm = np.where(np.isneginf(x), -128, qm)
    return qp.astype(np.int64), qm.astype(np.int64)


# Steps that are not powers of two: the hand-derived ones, a significand of
# all ones, one just above a power of two, and random ones over the range of
# calibrated activation steps.
_rng = np.random.default_rng(2024)
STEPS = ([float.fromhex(h) for h in ("0x1.fd0eb8p-8", "0x1.0adc5p-7", "0x1.945622p-6",
                                     "0x1.0624dcp-8", "0x1.fffffep-6", "0x1.000002p-7")]
         + [float(np.float32(v)) for v in np.exp(_rng.uniform(np.log(2e-4), np.log(0.2), 26))])


def test_worked_qdual_division(golden_dir):
    for k, v in read_fixture(golden_dir, "qdual_division_worked.txt"):
        if k != "case":
            continue
        sh, dv, xh, code = v.split()
        s = np.float32(float.fromhex(sh))
        assert float(s) == float.fromhex(sh)
        x = float.fromhex(xh)
        xb = (np.array([[x]], np.float32).view(np.uint32) >> 16).astype(np.uint16)
        assert float(bits_to_f32(xb)[0, 0]) == x
        d = None if float(dv) == 1 else np.array([[float(dv)]], np.float32)
        planes = oracle.quantize_act(xb, np.array([[[s, s]]], np.float32), d=d)
        if x >= 0:
            assert (planes[0, 0, 0, 0], planes[0, 1, 0, 0]) == (int(code), 0), v
        else:
            assert (planes[0, 0, 0, 0], planes[0, 1, 0, 0]) == (0, int(code)), v


def test_worked_fp8_division(golden_dir):
    for k, v in read_fixture(golden_dir, "qdual_division_worked.txt"):
        if k != "fp8_case":
            continue
        sh, xh, code = v.split()
        s = np.float32(float.fromhex(sh))
        x = float.fromhex(xh)
        xb = (np.array([[x]], np.float32).view(np.uint32) >> 16).astype(np.uint16)
        assert float(bits_to_f32(xb)[0, 0]) == x
        planes = oracle.quantize_act_fp8(xb, np.array([[[s, s]]], np.float32))
        assert (planes[0, 0, 0, 0], planes[0, 1, 0, 0]) == (int(code, 16), 0), v
    # a reciprocal multiply would give the other code
    r = np.float32(1) / np.float32(float.fromhex("0x1.b8e39p-5"))
    v = np.float32(float.fromhex("0x1.74p-7")) * r
    assert float(v) == 27 / 128
    assert int(torch.tensor([float(v)]).to(torch.float8_e4m3fn).view(torch.uint8)) == 0x26


def test_every_bf16_value_at_non_power_of_two_steps():
    """All 65536 bf16 patterns (zeros, subnormals, infinities and NaNs
    included) at 32 step pairs that are not powers of two."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    x = bits_to_f32(allbits.reshape(-1))
    for j, sp in enumerate(STEPS):
        sm = STEPS[(j + 7) % len(STEPS)]
        planes = oracle.quantize_act(allbits, np.array([[[sp, sm]]], np.float32))
        qp, qm = expected_codes(x, sp, sm)
        assert np.array_equal(planes[0, 0].reshape(-1).astype(np.int64), qp), sp
        assert np.array_equal(planes[0, 1].reshape(-1).astype(np.int64), qm), sm


def test_every_bf16_value_with_a_smoothquant_divisor():
    """u = fl(x / d) first, then fl(u / s): all bf16 values at six (d, s)
    pairs with divisors that are not powers of two.  Values whose quotient by
    d would leave the normal fp32 range are excluded (a divisor and an input
    that far apart have no use)."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = bits_to_f32(allbits)
    keep = ~np.isfinite(x) | (x == 0) | ((np.abs(x) > 2.0 ** -100) & (np.abs(x) < 2.0 ** 100))
    allbits = allbits[keep]
    allbits = allbits[: allbits.size // 64 * 64].reshape(-1, 64)
    x = bits_to_f32(allbits.reshape(-1))
    for dv, sp, sm in ((3.0, STEPS[3], STEPS[0]), (1.5, STEPS[8], STEPS[9]),
                       (0.7071068, STEPS[10], STEPS[1]), (12.37, STEPS[2], STEPS[11]),
                       (0.0913, STEPS[12], STEPS[13]), (5.0, STEPS[4], STEPS[5])):
        d = np.full((1, 64), dv, np.float32)
        planes = oracle.quantize_act(allbits, np.array([[[sp, sm]]], np.float32), d=d)
        qp, qm = expected_codes(x, sp, sm, d=float(np.float32(dv)))
        assert np.array_equal(planes[0, 0].reshape(-1).astype(np.int64), qp), dv
        assert np.array_equal(planes[0, 1].reshape(-1).astype(np.int64), qm), dv


def test_single_scale_codes_are_the_sum_at_non_power_of_two_steps():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    x = bits_to_f32(allbits.reshape(-1))
    for s in STEPS[:8]:
        planes = oracle.quantize_act(allbits, np.array([[[s, s]]], np.float32), single=True)
        qp, qm = expected_codes(x, s, s)
        assert np.array_equal(planes[0, 0].reshape(-1).astype(np.int64), qp + qm), s


def test_fp8_codes_at_non_power_of_two_steps():
    """E4M3 codes of fl(x / s): the exact fp32 quotient (rn32_div), then
    torch's float8_e4m3fn conversion (round half to even) after saturation to
    +-448; NaN gives 0x00 in both planes, -0.0 the + plane's e4m3(-0.0)."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    x = bits_to_f32(allbits.reshape(-1))
    finite = np.isfinite(x)
    xf = np.where(finite, x, 0).astype(np.float32)
    for j in (0, 2, 5, 9, 17):
        sp, sm = STEPS[j], STEPS[j + 1]
        planes = oracle.quantize_act_fp8(allbits, np.array([[[sp, sm]]], np.float32))
        for plane, s, sel in ((0, sp, (x >= 0)), (1, sm, (x < 0))):
            v, tiny = rn32_div(xf, s)
            v = np.where(tiny, np.copysign(0.0, xf), v)
            v = np.where(np.isinf(x), np.copysign(np.inf, x), v)
            v = np.clip(v, -448.0, 448.0).astype(np.float32)
            codes = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            exp = np.where(sel, codes, 0).astype(np.uint8)
            got = planes[0, plane].reshape(-1)
            assert np.array_equal(got, exp), (plane, s)


def test_worked_cases_separate_the_three_readings(golden_dir):
    """The fixture tells the pinned reading apart from its two neighbours:
    case A from a rounded reciprocal, rne(fl(x * fl(1/s))) (44, not 43), and
    cases C and D from the round-half-even of the exact real quotient (83 and
    53, not 82 and 54).  So an oracle computing either would fail
    test_worked_qdual_division.  Case F tells it apart from folding the
    divisor into the step, rne(fl(x / fl(d * s))) (81, not 80)."""
    cases = [v.split() for k, v in read_fixture(golden_dir, "qdual_division_worked.txt")
             if k == "case"]
    by_x = {c[2]: c for c in cases}
    s = np.float32(float.fromhex("0x1.fd0eb8p-8"))
    x = np.float32(float.fromhex("0x1.5ap-2"))
    fold = int(np.rint(np.float64(x * (np.float32(1) / s))))
    assert fold == 44 and int(by_x["0x1.5ap-2"][3]) == 43
    for xh, exact in (("0x1.58p-1", 83), ("0x1.52p+0", 53)):
        sh = by_x[xh][0]
        q = Fraction(float.fromhex(xh)) / Fraction(float.fromhex(sh))
        assert round(q) == exact != int(by_x[xh][3])
    d, s, x = np.float32(2.5), np.float32(float.fromhex("0x1.1cf06ap-8")), np.float32(0.875)
    assert int(np.rint(np.float64(x / (d * s)))) == 81 and int(by_x["0x1.cp-1"][3]) == 80
