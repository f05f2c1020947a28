"""The activation quantizer forms int8 codes without the quotient's correction
(one product u * fl(1/s)) when a block-wide test on a few hundred inputs says
that this gives the exact codes rne(fl(u/s)) for every bf16 input.  These CPU
tests check that argument on a numpy model of both forms: the test passes
exactly when the forms agree on all 65,536 bf16 values, over random steps and
over steps constructed so that the forms differ."""
import numpy as np
import pytest

from correction_free import (codes, forms_agree_everywhere, passes_candidate_test,
                             steps_where_forms_differ)


def test_worked_counterexample_is_caught():
    """s = 0x1.fd0eb8p-8, x = 0x1.5ap-2: x/s = 43.4999980..., fl(x/s) rounds to
    43, fl(x * fl(1/s)) = 43.5 rounds to 44 (either polarity)."""
    s = np.float32(float.fromhex("0x1.fd0eb8p-8"))
    x = np.array([0x3EAD, 0xBEAD], np.uint16)          # +-0x1.5ap-2
    exact = codes(x, s, s, False)
    fast = codes(x, s, s, True)
    assert (exact[0][0], exact[1][1]) == (43, -43)
    assert (fast[0][0], fast[1][1]) == (44, -44)
    assert not passes_candidate_test(s, np.float32(1 / 64))
    assert not passes_candidate_test(np.float32(1 / 64), s)
    assert passes_candidate_test(np.float32(1 / 64), np.float32(1 / 512))


@pytest.mark.parametrize("seed", range(4))
def test_candidate_test_is_exact_on_random_steps(seed):
    """Log-uniform steps over 2^-30 .. 2^20: the candidate test passes iff the
    two forms agree on every bf16 input of both polarities."""
    rng = np.random.default_rng(100 + seed)
    n_fast = 0
    for _ in range(60):
        sp, sm = np.exp2(rng.uniform(-30, 20, 2)).astype(np.float32)
        ok = passes_candidate_test(sp, sm)
        assert ok == forms_agree_everywhere(sp, sm), (float(sp), float(sm))
        n_fast += ok
    assert n_fast > 40            # the uncorrected form is the common case


def test_candidate_test_rejects_every_constructed_step():
    """Steps where some bf16 input's codes differ between the forms, on either
    side: the test must reject each of them."""
    bad = steps_where_forms_differ(12, seed=7)
    one = np.float32(1 / 64)
    for s in bad:
        s = np.float32(s)
        assert not forms_agree_everywhere(s, one)
        assert not passes_candidate_test(s, one), float(s)
        assert not passes_candidate_test(one, s), float(s)


def test_powers_of_two_and_calibrated_steps_pass():
    """Steps that are powers of two make both forms exact; AMax steps m/127 and
    m/128 of bf16 maxima are the common case of calibrated layers."""
    for e in range(-20, 10):
        assert passes_candidate_test(np.float32(2.0 ** e), np.float32(2.0 ** (e - 3)))
    rng = np.random.default_rng(3)
    agree = [forms_agree_everywhere(np.float32(m) / np.float32(127), np.float32(m) / np.float32(128))
             == passes_candidate_test(np.float32(m) / np.float32(127), np.float32(m) / np.float32(128))
             for m in rng.uniform(0.1, 40, 40)]
    assert all(agree)


# ---------------------------------------------- with SmoothQuant divisors
from correction_free import (channel_forms_agree_everywhere_d, channel_passes_test_d,  # noqa: E402
                             codes_d, divisors_where_forms_differ)


@pytest.mark.parametrize("seed", range(3))
def test_channel_test_is_exact_with_divisors(seed):
    """With a divisor d, the per-channel test (the bf16 neighbours of
    fl(fl((h + 1/2) s) d)) passes iff the doubly uncorrected codes equal the
    exact ones on every bf16 input, over log-uniform d and steps."""
    rng = np.random.default_rng(300 + seed)
    n_fast = 0
    for _ in range(40):
        d = np.float32(np.exp2(rng.uniform(-6, 6)))
        sp, sm = np.exp2(rng.uniform(-20, 8, 2)).astype(np.float32)
        ok = channel_passes_test_d(d, sp, sm)
        assert ok == channel_forms_agree_everywhere_d(d, sp, sm), (float(d), float(sp), float(sm))
        n_fast += ok
    assert n_fast > 10


def test_channel_test_rejects_constructed_divisors():
    s = np.float32(float.fromhex("0x1.0adc5p-7"))
    for d in divisors_where_forms_differ(8, s, seed=17):
        d = np.float32(d)
        assert not channel_forms_agree_everywhere_d(d, s, s)
        assert not channel_passes_test_d(d, s, s), float(d)
        assert not channel_passes_test_d(d, s, np.float32(1 / 64)), float(d)


def test_divisor_one_reduces_to_the_plain_forms():
    s = np.float32(float.fromhex("0x1.fd0eb8p-8"))
    x = np.array([0x3EAD, 0xBEAD], np.uint16)
    exact = codes_d(x, np.float32(1), s, s, False)
    fast = codes_d(x, np.float32(1), s, s, True)
    assert (exact[0][0], exact[1][1]) == (43, -43)
    assert (fast[0][0], fast[1][1]) == (44, -44)


# ------------------------------------------- the model against the oracle
from correction_free import ALL_BF16  # noqa: E402


@pytest.mark.parametrize("seed", range(2))
def test_exact_form_is_the_oracles_quantizer(seed):
    """The model's exact form (IEEE quotients, x/s or x/d then u/s) gives the
    oracle's planes on every bf16 input, with and without a divisor, at steps
    and divisors that are not powers of two: the verdicts of the block test
    and of the plan are statements about the oracle's codes."""
    import oracle
    rng = np.random.default_rng(500 + seed)
    xb = np.ascontiguousarray(ALL_BF16.reshape(4096, 16))
    for _ in range(3):
        sp, sm = np.exp2(rng.uniform(-12, 4, 2)).astype(np.float32)
        s_act = np.array([[[sp, sm]]], np.float32)
        planes = oracle.quantize_act(xb, s_act)
        qp, qm = codes(xb.ravel(), sp, sm, False)
        assert np.array_equal(planes[0, 0].ravel(), qp), (float(sp), float(sm))
        assert np.array_equal(planes[0, 1].ravel(), qm), (float(sp), float(sm))
        dv = np.float32(np.exp2(rng.uniform(-4, 4)))
        planes = oracle.quantize_act(xb, s_act, d=np.full((1, 16), dv, np.float32))
        qp, qm = codes_d(xb.ravel(), dv, sp, sm, False)
        assert np.array_equal(planes[0, 0].ravel(), qp), (float(dv), float(sp), float(sm))
        assert np.array_equal(planes[0, 1].ravel(), qm), (float(dv), float(sp), float(sm))


def test_uncorrected_form_departs_from_the_oracle_where_the_plan_says():
    """At a divisor the plan rejects, the uncorrected codes differ from the
    oracle's for some bf16 input; at one it accepts, they agree everywhere."""
    import oracle
    s = np.float32(float.fromhex("0x1.0adc5p-7"))
    s_act = np.array([[[s, s]]], np.float32)
    xb = np.ascontiguousarray(ALL_BF16.reshape(4096, 16))
    bad = np.float32(divisors_where_forms_differ(1, s, seed=29)[0])
    good = np.float32(1.5)
    assert not channel_passes_test_d(bad, s, s) and channel_passes_test_d(good, s, s)
    for dv, agree in ((bad, False), (good, True)):
        planes = oracle.quantize_act(xb, s_act, d=np.full((1, 16), dv, np.float32))
        qp, qm = codes_d(xb.ravel(), dv, s, s, True)
        same = (np.array_equal(planes[0, 0].ravel(), qp)
                and np.array_equal(planes[0, 1].ravel(), qm))
        assert same == agree, float(dv)
