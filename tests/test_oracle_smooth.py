"""Pins of the oracle's SmoothQuant step (per-channel multiplier after the fixed
rotation), its calibration statistic and its migration factors.

[AMD Quark adds native W4A8 mixed-precision for Wan2.2 video generation on MI350 --
 "Fixed rotation selector": fixed Hadamard rotations followed by SmoothQuant]
"""

import numpy as np
import pytest

import oracle
from mxfp4_block_scaled_mxq_b200 import inputs


@pytest.mark.parametrize("rule", [oracle.RULE_OCP, oracle.RULE_UOS])
@pytest.mark.parametrize("hadamard", [False, True])
def test_unit_multiplier_is_the_plain_quantiser(rule, hadamard):
    x = inputs.heavy_tailed_bf16(40, 256, seed=11)
    want = oracle.quantize_mxfp4(x, rule=rule, hadamard=hadamard)
    got = oracle.quantize_mxfp4_smooth(x, np.ones(256, np.float32), rule=rule, hadamard=hadamard)
    np.testing.assert_array_equal(got[0], want[0])
    np.testing.assert_array_equal(got[1], want[1])


@pytest.mark.parametrize("j", [-3, 5])
@pytest.mark.parametrize("hadamard", [False, True])
def test_power_of_two_multiplier_only_shifts_the_scale(j, hadamard):
    """Multiplying every channel by 2^j is exact: the codes are unchanged and every block
    exponent moves by j (no block near the clamp)."""
    x = inputs.normal_bf16(24, 384, 1.0, seed=12)
    codes0, sf0 = oracle.quantize_mxfp4(x, hadamard=hadamard)
    codes, sf = oracle.quantize_mxfp4_smooth(x, np.full(384, 2.0 ** j, np.float32), hadamard=hadamard)
    np.testing.assert_array_equal(codes, codes0)
    np.testing.assert_array_equal(sf.astype(int), sf0.astype(int) + j)


@pytest.mark.parametrize("rule", [oracle.RULE_OCP, oracle.RULE_UOS])
def test_rotation_comes_before_the_channel_multiplier(rule):
    """Worked example from the definitions: x = e_0 (one 128-chunk), multiplier 4 on
    channel 0.  Rotation first: y = 1/sqrt(128) everywhere, then y_0 = 4/sqrt(128) =
    0.354 -> block 0 exponent floor(log2 0.354) - 2 = -4 (byte 123), y_0 * 16 = 5.66 -> 6
    (code 0x7), the other elements 0.0884 * 16 = 1.41 -> 1.5 (code 0x3); blocks 1..3:
    amax 0.0884 -> exponent -6 (byte 121), 0.0884 * 64 = 5.66 -> 6 (code 0x7).
    (Multiplier first would give every block byte 123 and all codes 0x7.)  UOS: 5.66 <=
    7.25, no bump, so the same bytes."""
    bits = np.zeros((1, 128), np.uint16)
    bits[0, 0] = 0x3F80  # 1.0
    c = np.ones(128, np.float32)
    c[0] = 4.0
    codes, sf = oracle.quantize_mxfp4_smooth(bits, c, rule=rule, hadamard=True)
    np.testing.assert_array_equal(sf[0], [123, 121, 121, 121])
    nib = np.stack([codes[0] & 0xF, codes[0] >> 4], axis=1).reshape(-1)
    assert nib[0] == 0x7
    assert (nib[1:32] == 0x3).all()
    assert (nib[32:] == 0x7).all()


@pytest.mark.parametrize("hadamard", [False, True])
def test_channel_absmax_is_the_column_maximum(hadamard):
    x = inputs.outlier_channels_bf16(70, 256, 0.02, 25.0, seed=13)
    y = oracle.rotate_rows(x, hadamard=hadamard)
    np.testing.assert_array_equal(oracle.channel_absmax(x, hadamard=hadamard), np.abs(y).max(axis=0))


def test_smooth_factor_closed_forms():
    ax = np.array([4.0, 9.0, 3.0, 0.0, 5.0, 2.0], np.float32)
    aw = np.array([1.0, 4.0, 7.0, 2.0, 0.0, 8.0], np.float32)
    lam, inv = oracle.smooth_factors(ax, aw, alpha=0.5)
    # sqrt(4/1), sqrt(9/4), sqrt(3/7); ax = 0 clamps to 1e-5; aw = 0 -> 1e-5; sqrt(2/8)
    want = np.array([2.0, 1.5, np.sqrt(3 / 7), 1e-5, np.sqrt(5 / 1e-5), 0.5], np.float64)
    np.testing.assert_allclose(lam.astype(np.float64), want, rtol=1e-7)
    np.testing.assert_array_equal(inv, np.float32(1.0) / lam)
    lam1, _ = oracle.smooth_factors(ax[:3], aw[:3], alpha=1.0)     # all migrated: lambda = ax
    np.testing.assert_array_equal(lam1, ax[:3])
    lam0, _ = oracle.smooth_factors(ax[:3], aw[:3], alpha=0.0)     # none: lambda = 1 / aw
    np.testing.assert_allclose(lam0, 1.0 / aw[:3], rtol=1e-7)


def _layer_error(x, w, cx, cw, hadamard=False):
    """Relative Frobenius error of the W4A4 layer with multipliers cx (activations) and cw
    (weights) against the unquantised X W^T."""
    M, K = x.shape
    N = w.shape[0]
    a, asl = oracle.quantize_mxfp4_smooth(x, cx, hadamard=hadamard)
    b, bsl = oracle.quantize_mxfp4_smooth(w, cw, hadamard=hadamard)
    y = oracle.gemm(a, oracle.sf_swizzle(asl, M, K), b, oracle.sf_swizzle(bsl, N, K), M, N, K)
    ref = x.double().numpy() @ w.double().numpy().T
    return np.linalg.norm(y - ref) / np.linalg.norm(ref)


def test_multiplier_direction_on_outlier_channels():
    """With 2 % of the channels 30x larger, the SmoothQuant assignment (X / lambda,
    W * lambda) keeps the W4A4 error at or below the plain layer's, while the swapped
    assignment (X * lambda, W / lambda) piles the outliers up and at least 1.5x's it.
    (With 32-element block scales the gain itself is small: about 5 % here.)"""
    x = inputs.outlier_channels_bf16(96, 512, 0.02, 30.0, seed=14)
    w = inputs.normal_bf16(128, 512, 0.02, seed=15)
    lam, inv = oracle.smooth_factors(oracle.channel_absmax(x), oracle.channel_absmax(w), alpha=0.5)
    one = np.ones(512, np.float32)
    e_plain = _layer_error(x, w, one, one)
    e_smooth = _layer_error(x, w, inv, lam)
    e_swapped = _layer_error(x, w, lam, inv)
    assert e_smooth < e_plain, (e_smooth, e_plain)
    assert e_swapped > 1.5 * e_plain, (e_swapped, e_plain)


def test_unquantised_product_is_invariant():
    """X diag(1/lambda) (W diag(lambda))^T = X W^T, with and without the rotation
    (FP64, no quantisation)."""
    x = inputs.outlier_channels_bf16(16, 256, 0.02, 30.0, seed=16)
    w = inputs.normal_bf16(32, 256, 0.02, seed=17)
    for hadamard in (False, True):
        lam, inv = oracle.smooth_factors(oracle.channel_absmax(x, hadamard), oracle.channel_absmax(w, hadamard))
        xr = oracle.rotate_rows(x, hadamard=hadamard).astype(np.float64) / lam.astype(np.float64)
        wr = oracle.rotate_rows(w, hadamard=hadamard).astype(np.float64) * lam.astype(np.float64)
        ref = x.double().numpy() @ w.double().numpy().T
        np.testing.assert_allclose(xr @ wr.T, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())
