"""Host-only proof behind the rotated quantiser's folded scaling.

With the 128-point rotation the definition quantises y = fl32(t * c) (t a butterfly output,
c = fl32(1/sqrt(128))) with the block scale 2^e: code = E2M1(fl32(y * 2^-e)).  The quantiser
multiplies once, code = E2M1(fl32(t * fl32(c * 2^-e))), and takes the block exponent from
fl32(max |t| * c).  These checks cover every case in which the two could differ: rounding is
monotone (the block maximum), power-of-two scaling commutes with rounding in the normal
range, and where fl32(t * c) is subnormal t is a multiple of 2^-133 (the BF16 grid), which
the enumeration below covers completely.

[AMD Quark adds native W4A8 mixed-precision for Wan2.2 video generation on MI350 --
 "Fixed rotation selector": a fixed Hadamard rotation ahead of MXFP4 quantisation]
"""

import numpy as np
import pytest

import oracle

F32 = np.float32
C = F32(oracle.hadamard_scale())
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e2m1_index(v):
    """E2M1 magnitude index of FP32 values (nearest, ties to the even index, saturating)."""
    a = np.minimum(np.abs(v.astype(np.float64)), 6.0)
    d = np.abs(a[..., None] - GRID)
    tied = d == d.min(-1, keepdims=True)
    even = tied & (np.arange(8) % 2 == 0)
    return np.where(even.any(-1), np.argmax(even, -1), np.argmax(tied, -1)) | (np.signbit(v) << 3)


def _two(t, e):
    return ((t * C).astype(F32) * F32(2.0 ** -e)).astype(F32)


def _folded(t, e):
    return (t * (C * F32(2.0 ** -e)).astype(F32)).astype(F32)


def test_encoder_matches_the_oracle():
    v = np.float32(np.linspace(-7, 7, 4001))
    want = np.array([oracle.e2m1_encode(float(x)) for x in v])
    np.testing.assert_array_equal(_e2m1_index(v), want)


def test_c_is_the_oracle_rotation_scale():
    assert C == F32(1.0 / np.sqrt(128.0))


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_every_small_bf16_grid_value_every_exponent(sign):
    """All t = k 2^-133 with |t| < 2^-117 (every value for which fl32(t * c) can be
    subnormal, with room to spare), against every block exponent from -127 to 122."""
    k = np.arange(0, 1 << 16, dtype=np.float64)
    t = (sign * k * 2.0 ** -133).astype(F32)
    assert np.all(np.abs(t.astype(np.float64)) == k * 2.0 ** -133)
    for e in range(-127, 123):
        np.testing.assert_array_equal(_e2m1_index(_two(t, e)), _e2m1_index(_folded(t, e)), err_msg=f"e={e}")


def test_normal_range_agrees_for_random_values():
    """Random FP32 t over the whole normal range of t c, every block exponent for which the
    scaled values reach the codes."""
    rng = np.random.default_rng(3)
    mant = rng.integers(1 << 23, 1 << 24, 200000)
    for e in range(-127, 123, 7):
        ex = rng.integers(-2, 5, mant.size) + e + 3     # |t c 2^-e| around [2^-5, 2^8)
        t = (mant * np.exp2(ex - 23.0) * rng.choice([-1.0, 1.0], mant.size)).astype(F32)
        ok = np.isfinite(t) & (np.abs(t * np.float64(C)) >= 2.0 ** -126)
        np.testing.assert_array_equal(_e2m1_index(_two(t[ok], e)), _e2m1_index(_folded(t[ok], e)), err_msg=f"e={e}")


def test_block_maximum_commutes_with_the_rounding():
    rng = np.random.default_rng(4)
    t = (rng.standard_normal((20000, 32)) * np.exp2(rng.integers(-140, 120, (20000, 1)))).astype(F32)
    np.testing.assert_array_equal(np.abs((t * C).astype(F32)).max(1), (np.abs(t).max(1) * C).astype(F32))


def test_infinite_block_maximum():
    """A butterfly overflow gives amax = inf and e = 127: infinite elements saturate to 6
    and finite ones (below 2^128) give 0 in both forms."""
    t = np.array([np.inf, -np.inf, 3.4e38, -1e30, 1.0, 0.0], F32)
    with np.errstate(over="ignore"):
        np.testing.assert_array_equal(_e2m1_index(_two(t, 127)), _e2m1_index(_folded(t, 127)))
    assert list(_e2m1_index(_folded(t, 127))[:3]) == [7, 15, 0]
