"""Numpy model of the activation quantizer's two ways of forming an int8 code
(no divisor), used to test the argument that lets the kernel skip the
quotient's correction for some step pairs.

  exact:         q = rne(min(fl(u / s), 128))          (IEEE division, then RNE)
  uncorrected:   q = rne(min(RN(u * fl(1 / s)), 128))  (reciprocal, one product)

The + plane takes u >= 0 with s+ (code lowered to 127), the - plane u < 0 with
s- (code -q).  numpy's float32 division, reciprocal and product are IEEE
round-to-nearest, like the kernel's explicit _rn operations.  The candidate
test mirrors the kernel's: for every rounding boundary b = h + 1/2 (h < 128),
the bf16 values around fl(b s) truncated to bf16."""
import numpy as np

ALL_BF16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def bf16_to_f32(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def _plane_codes(mag, s, uncorrected):
    """Codes rne(min(q, 128)) of non-negative finite-or-inf magnitudes (NaN -> 0)."""
    s = np.float32(s)
    with np.errstate(over="ignore", invalid="ignore"):
        if uncorrected:
            q = (mag * (np.float32(1) / s)).astype(np.float32)
        else:
            q = (mag / s).astype(np.float32)
    q = np.where(np.isnan(q), np.float32(0), q)
    return np.rint(np.minimum(q, np.float32(128))).astype(np.int32)


def codes(bits, s_plus, s_minus, uncorrected):
    """(+ plane, - plane) int8 codes of bf16 inputs."""
    x = bf16_to_f32(bits)
    neg = np.signbit(x) & ~np.isnan(x)
    mag = np.abs(x)
    qp = np.where(neg, 0, np.minimum(_plane_codes(mag, s_plus, uncorrected), 127))
    qm = np.where(neg, -_plane_codes(mag, s_minus, uncorrected), 0)
    return qp.astype(np.int8), qm.astype(np.int8)


def candidates(s):
    """bf16 magnitudes next to every boundary (h + 1/2) s, h = 0..127."""
    b = (np.arange(128, dtype=np.float32) + np.float32(0.5))
    t = (b * np.float32(s)).astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    c = np.concatenate([t - np.uint32(0x10000), t, t + np.uint32(0x10000)])
    return (c >> 16).astype(np.uint16)


def passes_candidate_test(s_plus, s_minus):
    """The kernel's block-wide test: both forms agree on the candidates."""
    cp = candidates(s_plus)
    cm = candidates(s_minus) | np.uint16(0x8000)
    for c in (cp, cm):
        a = codes(c, s_plus, s_minus, False)
        u = codes(c, s_plus, s_minus, True)
        if not (np.array_equal(a[0], u[0]) and np.array_equal(a[1], u[1])):
            return False
    return True


def forms_agree_everywhere(s_plus, s_minus):
    a = codes(ALL_BF16, s_plus, s_minus, False)
    u = codes(ALL_BF16, s_plus, s_minus, True)
    return np.array_equal(a[0], u[0]) and np.array_equal(a[1], u[1])


def steps_where_forms_differ(n, seed):
    """n float32 steps s for which some bf16 input gets different codes from
    the two forms (searched next to x / (h + 1/2) for random bf16 x and h)."""
    rng = np.random.default_rng(seed)
    found = []
    while len(found) < n:
        x = bf16_to_f32(rng.integers(0x3C00, 0x4400))   # x in [2^-7, 2^9)
        h = rng.integers(0, 127)
        s0 = np.float32(x / np.float32(h + 0.5))
        base = s0.view(np.int32)
        for k in range(-64, 65):
            s = np.int32(base + k).view(np.float32)
            if not forms_agree_everywhere(s, s):
                found.append(float(s))
                break
    return found


# ------------------------------------------------- with SmoothQuant divisors
# u = x / d first, then the code of u at step s.  The exact form takes both
# quotients as IEEE divisions; the uncorrected form multiplies by the rounded
# reciprocals: q = rne(min(RN(RN(x fl(1/d)) fl(1/s)), 128)).  Both lie within
# 2^-22 (relative) of x / (d s), so they can differ only for x next to a
# boundary (h + 1/2) s d; the per-channel test evaluates the bf16 neighbours of
# fl(fl((h + 1/2) s) d).

def _plane_codes_d(mag, d, s, uncorrected):
    d, s = np.float32(d), np.float32(s)
    with np.errstate(over="ignore", invalid="ignore"):
        if uncorrected:
            u = (mag * (np.float32(1) / d)).astype(np.float32)
            q = (u * (np.float32(1) / s)).astype(np.float32)
        else:
            u = (mag / d).astype(np.float32)
            q = (u / s).astype(np.float32)
    q = np.where(np.isnan(q), np.float32(0), q)
    return np.rint(np.minimum(q, np.float32(128))).astype(np.int32)


def codes_d(bits, d, s_plus, s_minus, uncorrected):
    """(+ plane, - plane) int8 codes of bf16 inputs divided by d first."""
    x = bf16_to_f32(bits)
    neg = np.signbit(x) & ~np.isnan(x)
    mag = np.abs(x)
    qp = np.where(neg, 0, np.minimum(_plane_codes_d(mag, d, s_plus, uncorrected), 127))
    qm = np.where(neg, -_plane_codes_d(mag, d, s_minus, uncorrected), 0)
    return qp.astype(np.int8), qm.astype(np.int8)


def candidates_d(d, s):
    b = (np.arange(128, dtype=np.float32) + np.float32(0.5))
    t = ((b * np.float32(s)).astype(np.float32) * np.float32(d)).astype(np.float32)
    t = t.view(np.uint32) & np.uint32(0xFFFF0000)
    c = np.concatenate([t - np.uint32(0x10000), t, t + np.uint32(0x10000)])
    return (c >> 16).astype(np.uint16)


def channel_passes_test_d(d, s_plus, s_minus):
    """The per-channel test of the plan: both forms agree on the candidates."""
    for c in (candidates_d(d, s_plus), candidates_d(d, s_minus) | np.uint16(0x8000)):
        a = codes_d(c, d, s_plus, s_minus, False)
        u = codes_d(c, d, s_plus, s_minus, True)
        if not (np.array_equal(a[0], u[0]) and np.array_equal(a[1], u[1])):
            return False
    return True


def channel_forms_agree_everywhere_d(d, s_plus, s_minus):
    a = codes_d(ALL_BF16, d, s_plus, s_minus, False)
    u = codes_d(ALL_BF16, d, s_plus, s_minus, True)
    return np.array_equal(a[0], u[0]) and np.array_equal(a[1], u[1])


def divisors_where_forms_differ(n, s, seed):
    """n float32 divisors d for which some bf16 input's codes at step s differ
    between the two forms (searched next to x / ((h + 1/2) s))."""
    rng = np.random.default_rng(seed)
    s = np.float32(s)
    found = []
    while len(found) < n:
        x = bf16_to_f32(rng.integers(0x3C00, 0x4400))
        h = rng.integers(0, 127)
        base = np.float32(x / ((np.float32(h) + np.float32(0.5)) * s)).view(np.int32)
        for k in range(-64, 65):
            d = np.int32(base + k).view(np.float32)
            if not channel_forms_agree_everywhere_d(d, s, s):
                found.append(float(d))
                break
    return found
