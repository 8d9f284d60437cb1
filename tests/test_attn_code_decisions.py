"""Host-only proof that the attention kernel's numerator codes are those of the exact
exponential.

The kernel never forms 2^(t - c): a key's scaled numerator is x = 2^m 2^g with
n = rint(t), g = t - n in [-1/2, 1/2] and m = n - c - e, and its E2M1 code only depends on
which rounding boundaries x passes.  Inside the octaves that carry codes, those boundaries
sit at four levels of 2^g -- 0.75, 0.875, 1 and 1.25 -- so the kernel evaluates a cubic
q(g) (FP32 Horner, the last step rounded toward +infinity) whose FP32 values cross the
levels exactly where 2^g does.  These tests check that property for every FP32 g (exhaustive
windows around each crossing, a monotonicity and error-bound argument outside them), the
kernel's integer rule for the block exponent against the oracle's MX rule, and the whole
decision chain against the oracle's encoder on sampled scores.  Every FP32 operation is
emulated exactly with rationals.

[MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for MXFP4
 Attention -- "Architecture" (exp, then PNQ before the row sum), "What it actually does"]
"""

import math
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
from mxfp4_block_scaled_mxq_b200 import build, mxq

getcontext().prec = 60


@pytest.fixture(scope="module")
def coeffs():
    build.build()
    c = mxq.mxq_attn_code_poly()
    assert c[0] == 1.0
    return [Fraction(x) for x in c]


# ---------------------------------------------------------------- exact FP32 arithmetic

def _round32(q: Fraction, up: bool = False) -> Fraction:
    """q rounded to FP32 (nearest-even, or toward +infinity), as an exact rational."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                      # subnormals share the 2^-149 step
    step = Fraction(2) ** (e - 23)
    k, rem = divmod(a, step)              # a = k step + rem, 0 <= rem < step
    k = int(k)
    if up:
        if rem and sign > 0:
            k += 1                        # toward +inf: magnitude up for positive values
    elif rem * 2 > step or (rem * 2 == step and k % 2 == 1):
        k += 1
    return sign * k * step


def _fma(a, b, c, up=False):
    return _round32(a * b + c, up)


def _q(cf, g: Fraction) -> Fraction:
    p = _fma(cf[3], g, cf[2])
    p = _fma(p, g, cf[1])
    return _fma(p, g, cf[0], up=True)


def _f32_neighbours(d: Decimal):
    """Largest FP32 below the irrational d and the next FP32 up."""
    lo = np.float32(float(d))
    while Fraction(float(lo)) > Fraction(str(d)):
        lo = np.nextafter(lo, np.float32(-np.inf))
    while Fraction(float(np.nextafter(lo, np.float32(np.inf)))) < Fraction(str(d)):
        lo = np.nextafter(lo, np.float32(np.inf))
    return lo, np.nextafter(lo, np.float32(np.inf))


def _log2(x: Decimal) -> Decimal:
    return x.ln() / Decimal(2).ln()


# (level, how the E2M1 conversion breaks a tie exactly at the level: True = up)
# 0.75 = 0.75 (m = 0: 0.5 | 1.0 -> even 1.0 is up); 0.875 = 1.75/2, 3.5/4 (1.5 | 2, 3 | 4: up);
# 1.25 = 1.25, 2.5/2, 5/4 (1 | 1.5, 2 | 3, 4 | 6: the even code is down).
LEVELS = [(Decimal(3) / 4, True), (Decimal(7) / 8, True), (Decimal(5) / 4, False)]
WINDOW = 2048  # FP32 values on each side of each crossing, checked one by one


def _reaches(q: Fraction, level: Decimal, tie_up: bool) -> bool:
    lv = Fraction(str(level))
    return q >= lv if tie_up else q > lv


@pytest.mark.parametrize("level,tie_up", LEVELS)
def test_cubic_crosses_each_level_where_the_exponential_does(coeffs, level, tie_up):
    """For the WINDOW FP32 values of g on either side of log2(level): the kernel's cubic
    reaches the level (under the conversion's tie rule) exactly when g > log2(level)."""
    below, above = _f32_neighbours(_log2(level))
    g = below
    for _ in range(WINDOW):
        assert not _reaches(_q(coeffs, Fraction(float(g))), level, tie_up), float(g)
        g = np.nextafter(g, np.float32(-np.inf))
    g = above
    for _ in range(WINDOW):
        assert _reaches(_q(coeffs, Fraction(float(g))), level, tie_up), float(g)
        g = np.nextafter(g, np.float32(np.inf))


def test_rounded_up_last_step_decides_level_one_exactly(coeffs):
    """q(g) > 1 exactly when g > 0 (the boundary 0.25 at m = -2, where a tie goes down to
    0): the inner Horner value is positive, so the rounded-up 1 + (inner) g is above 1 for
    every positive g, however small, and at most 1 otherwise."""
    tiny = [Fraction(2) ** -149, Fraction(2) ** -126, Fraction(2) ** -60, Fraction(2) ** -25, Fraction(2) ** -24,
            Fraction(2) ** -23, Fraction(3, 2 ** 24)]
    for t in tiny:
        assert _q(coeffs, t) > 1
        assert _q(coeffs, -t) <= 1
    assert _q(coeffs, Fraction(0)) == 1


def test_no_other_crossing_outside_the_windows(coeffs):
    """Outside the windows the decision cannot flip: the real cubic rises with slope >= 0.45
    on [-1/2, 1/2], so at a window's edge it is at least 0.45 * WINDOW * 2^-26 from the level
    (2^-26 is the smallest FP32 step of g near any crossing), far above the Horner rounding
    bound of the FP32 evaluation (three roundings of values below 1.5, plus the rounded-up
    step).  It also stays inside (0.625, 1.5), so no other boundary of an octave is met."""
    a = [float(x) for x in coeffs]
    g = np.linspace(-0.5, 0.5, 100001)
    slope = a[1] + 2 * a[2] * g + 3 * a[3] * g ** 2
    assert slope.min() >= 0.45
    horner_bound = 4 * 1.5 * 2.0 ** -23
    assert 0.45 * WINDOW * 2.0 ** -26 > 10 * horner_bound
    assert float(_q(coeffs, Fraction(-1, 2))) > 0.625 + 1e-6
    assert float(_q(coeffs, Fraction(1, 2))) < 1.5 - 1e-6
    # and the real cubic tracks 2^g closely everywhere (it interpolates it at the levels)
    real = a[0] + a[1] * g + a[2] * g ** 2 + a[3] * g ** 3
    assert np.abs(real / np.exp2(g) - 1).max() < 5e-4


# ---------------------------------------------------------------- the kernel's decision chain

UOS_FRAC = np.float32(float.fromhex("-0x1.22dadep-3"))  # log2(0.90625) rounded down to FP32


def test_uos_fraction_constant_is_log2_of_0_90625_rounded_down():
    lo, hi = _f32_neighbours(_log2(Decimal("0.90625")))
    assert lo == UOS_FRAC


def _kernel_block_exponent(tmax: np.float32, cp: int, uos: bool) -> int:
    """The kernel's integer rule: floor(tmax - cp) - 2 from n = rint(tmax), g = tmax - n, one
    more under UOS when g is in (log2(0.90625), 0), clamped to -127."""
    if not tmax >= np.float32(cp - 127):
        return -127
    n = np.rint(tmax)                       # ties to even, like the kernel's rintf
    g = np.float32(tmax - n)                # exact
    e = int(n) - cp - 2
    if g < 0 and not (uos and g > UOS_FRAC):
        e -= 1
    return max(e, -127)


def _sample_scores(rng, count):
    """FP32 scores spread over several octaves, plus values one and two FP32 steps around
    every crossing of a numerator with a boundary or a scale threshold."""
    t = (rng.standard_normal(count) * rng.choice([0.1, 2.0, 20.0], count)).astype(np.float32)
    near = []
    for lv in [Decimal(3) / 4, Decimal(7) / 8, Decimal(5) / 4, Decimal("0.90625")]:
        lo, hi = _f32_neighbours(_log2(lv))
        for k in range(-6, 7):
            for x in (lo, hi, np.nextafter(lo, np.float32(-1)), np.nextafter(hi, np.float32(1))):
                near.append(np.float32(x + np.float32(k)))
    near += [np.float32(k) for k in range(-8, 9)]
    near += [np.float32(k + 0.5) for k in range(-8, 9)]
    return np.concatenate([t, np.array(near, np.float32)])


@pytest.mark.parametrize("rule", [oracle.RULE_OCP, oracle.RULE_UOS])
def test_block_exponent_matches_the_mx_rule_on_the_exact_numerator(rule):
    rng = np.random.default_rng(7)
    for tmax in _sample_scores(rng, 3000):
        for cp in (int(np.ceil(tmax)), int(np.ceil(tmax)) + 3, int(np.ceil(tmax)) + 8):
            want = oracle.block_exponent(2.0 ** (float(tmax) - cp), rule)
            assert _kernel_block_exponent(tmax, cp, rule == oracle.RULE_UOS) == want, (float(tmax), cp)


@pytest.mark.parametrize("rule", [oracle.RULE_OCP, oracle.RULE_UOS])
def test_codes_match_the_exact_exponential(coeffs, rule):
    """Whole chain on sampled scores: block exponent from the block's largest score, code
    from q(g) 2^(n - c - e) rounded to E2M1 -- against the oracle's encoder applied to
    2^(t - c - e) in FP64 (the exact numerator in FP64 arithmetic)."""
    rng = np.random.default_rng(11 + rule)
    t = _sample_scores(rng, 1500)
    for i in range(0, t.size - 32, 7):
        blk = t[i:i + 32]
        tmax = blk.max()
        cp = int(np.ceil(tmax)) + int(rng.integers(0, 9))
        e = _kernel_block_exponent(tmax, cp, rule == oracle.RULE_UOS)
        assert e == oracle.block_exponent(2.0 ** (float(tmax) - cp), rule)
        for x in blk[:8]:
            n = np.rint(x)
            g = Fraction(float(np.float32(x - n)))
            if int(n) - cp < -126:               # flushed to 0 by the kernel: not compared
                continue
            m = int(n) - cp - e
            val = _q(coeffs, g) * Fraction(2) ** m
            got = oracle.e2m1_encode(float(val))   # val is an FP32 value: exact as a double
            want = oracle.e2m1_encode(2.0 ** (float(x) - cp - e))
            assert got == want, (float(x), cp, e)
