"""Pins of the oracle's precision selection: the SQNR against closed forms, and the
tiered decision at and around its thresholds.

[AMD Quark adds native W4A8 mixed-precision for Wan2.2 video generation on MI350 --
 "Block-level SQNR calibration": whole-block output SQNR against BF16 under plain MXFP4
 and under the rotation + SmoothQuant transform, then tiered thresholds choose plain
 W4A4, W4A8 promotion, transform-enabled W4A4 or BF16]
"""

import math

import numpy as np
import pytest

import oracle


@pytest.mark.parametrize("eps", [0.5, 0.1, 1e-3])
def test_sqnr_of_a_uniform_relative_error(eps):
    """y = ref (1 + eps) everywhere: SQNR = -20 log10(eps) for any ref."""
    ref = np.random.default_rng(1).normal(size=(37, 53))
    s, n = oracle.sqnr_sums(ref * (1 + eps), ref)
    assert s == pytest.approx(float((ref ** 2).sum()), rel=1e-13)
    assert oracle.sqnr_db(s, n) == pytest.approx(-20 * math.log10(eps), abs=1e-9)


def test_sqnr_sums_of_a_known_pair():
    ref = np.array([3.0, -4.0, 0.0, 1.0])
    y = np.array([3.0, -3.0, 2.0, 1.0])   # errors 0, 1, 2, 0
    assert oracle.sqnr_sums(y, ref) == (26.0, 5.0)
    assert oracle.sqnr_db(26.0, 5.0) == pytest.approx(10 * math.log10(26 / 5), abs=1e-12)


def test_sqnr_limits():
    assert oracle.sqnr_db(1.0, 0.0) == math.inf    # exact output
    assert oracle.sqnr_db(0.0, 1.0) == -math.inf   # silent reference, noisy output


@pytest.mark.parametrize("plain,transform,want", [
    (20.0, 5.0, oracle.PREC_W4A4),             # plain clears the high tier
    (15.0, 15.0, oracle.PREC_W4A4),            # ties pass (>=); plain wins over the transform
    (14.99, 15.0, oracle.PREC_W4A4_TRANSFORM), # only the transform clears it
    (14.0, 12.0, oracle.PREC_W4A8),            # the better one clears the low tier
    (9.0, 10.0, oracle.PREC_W4A8),
    (9.99, 9.0, oracle.PREC_BF16),             # neither tier
    (-math.inf, -math.inf, oracle.PREC_BF16),
])
def test_tiers(plain, transform, want):
    assert oracle.select_precision(plain, transform, 15.0, 10.0) == want
