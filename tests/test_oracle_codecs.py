"""Pins for the oracle's element codecs and block-scale rules.

Each check compares the oracle with something other than itself: the OCP element
tables, a first-principles round-half-even in exact rationals (a different
formulation from the oracle's nearest-candidate search), closed forms of the
exponent rules, and the constant Qmax = 7.25 printed by the MXAttention page.
"""

import math
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import golden


def bf16_to_float(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0]


def f32_bits(v: float) -> int:
    return struct.unpack("<I", struct.pack("<f", v))[0]


ALL_BF16_FINITE = [b for b in range(1 << 16) if ((b >> 7) & 0xFF) != 0xFF]


# ----------------------------------------------------------------- E2M1 decode
def test_e2m1_decode_matches_ocp_table():
    for code_s, val_s in golden("e2m1_values.txt"):
        code, val = int(code_s, 16), float(val_s)
        got = oracle.e2m1_decode(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def _e2m1_from_fields(code: int) -> float:
    """E2M1 value from its bit fields (bias 1, exponent field 0 subnormal)."""
    s, e, m = code >> 3, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_decode_matches_bit_fields():
    for c in range(16):
        assert oracle.e2m1_decode(c) == _e2m1_from_fields(c)


# ----------------------------------------------------------------- E2M1 encode
def _rne_e2m1_magnitude(a: Fraction) -> Fraction:
    """Round-half-even of a >= 0 onto the E2M1 grid, saturating at 6, by binade ulp."""
    if a >= 6:
        return Fraction(6)
    if a < 2:
        ulp = Fraction(1, 2)          # subnormal [0,1) and [1,2) share ulp 0.5
    elif a < 4:
        ulp = Fraction(1)
    else:
        ulp = Fraction(2)
    q = round(a / ulp) * ulp          # Python rounds Fraction halves to even
    return min(q, Fraction(6))


def _check_e2m1(v: float):
    code = oracle.e2m1_encode(v)
    assert (code >> 3) == (1 if math.copysign(1.0, v) < 0 else 0), (v, code)
    want = _rne_e2m1_magnitude(abs(Fraction(v)))
    assert Fraction(abs(oracle.e2m1_decode(code))) == want, (v, code, want)


def test_e2m1_encode_all_bf16_values():
    for b in ALL_BF16_FINITE:
        _check_e2m1(bf16_to_float(b))


def test_e2m1_encode_dense_grid_and_ties():
    grid = [i / 64 for i in range(-64 * 9, 64 * 9 + 1)]
    for v in grid:
        _check_e2m1(v)
    # Tie table: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4.
    for v, mag in [(0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),
                   (5.0000001, 6.0), (6.5, 6.0), (7.9, 6.0), (1e30, 6.0)]:
        assert abs(oracle.e2m1_decode(oracle.e2m1_encode(v))) == mag
        assert oracle.e2m1_decode(oracle.e2m1_encode(-v)) == -mag


def test_e2m1_signed_zero():
    assert oracle.e2m1_encode(0.0) == 0x0
    assert oracle.e2m1_encode(-0.0) == 0x8
    assert oracle.e2m1_encode(-0.1) == 0x8
    assert oracle.e2m1_encode(-1e-30) == 0x8


# ----------------------------------------------------------------- block exponent
def _ocp_closed_form(amax: float) -> int:
    if amax == 0:
        return -127
    _, E = math.frexp(amax)           # amax = m * 2^E, m in [0.5, 1): floor(log2) = E - 1
    return max(-127, min(127, (E - 1) - 2))


def _uos_bit_rule(amax: float) -> int:
    """Bump the OCP exponent iff the FP32 significand exceeds 1.8125 = 7.25/4
    (biased exponent >= 2, so the OCP exponent is not clamped)."""
    e = _ocp_closed_form(amax)
    bits = f32_bits(amax)
    biased = (bits >> 23) & 0xFF
    if biased >= 2 and (bits & 0x7FFFFF) > 0x680000:
        e += 1
    return min(e, 127)


def test_ocp_exponent_all_bf16():
    for b in ALL_BF16_FINITE:
        a = abs(bf16_to_float(b))
        assert oracle.block_exponent(a, oracle.RULE_OCP) == _ocp_closed_form(a), a


def test_uos_exponent_all_bf16():
    for b in ALL_BF16_FINITE:
        a = abs(bf16_to_float(b))
        e_ocp = oracle.block_exponent(a, oracle.RULE_OCP)
        e_uos = oracle.block_exponent(a, oracle.RULE_UOS)
        assert e_uos == _uos_bit_rule(a), a
        assert e_uos in (e_ocp, e_ocp + 1)


def test_uos_boundary_from_page_constant():
    rows = dict((r[0], r[1]) for r in golden("uos_qmax.txt"))
    qmax = float(rows["qmax"])
    assert qmax == 7.25 and int(rows["block"]) == 32
    for e in range(-120, 121, 7):
        at = math.ldexp(qmax, e)
        above = float(np.nextafter(np.float32(at), np.float32(np.inf)))
        below = float(np.nextafter(np.float32(at), np.float32(0)))
        assert oracle.block_exponent(at, oracle.RULE_UOS) == e          # tie: no bump (<= Qmax)
        assert oracle.block_exponent(above, oracle.RULE_UOS) == e + 1
        assert oracle.block_exponent(below, oracle.RULE_UOS) == e
        # OCP keeps e for every amax in [4, 8) * 2^e.
        assert oracle.block_exponent(at, oracle.RULE_OCP) == e
        assert oracle.block_exponent(math.ldexp(4.0, e), oracle.RULE_OCP) == e
        assert oracle.block_exponent(math.ldexp(8.0, e), oracle.RULE_OCP) == e + 1


def test_exponent_special_cases():
    for rule in (oracle.RULE_OCP, oracle.RULE_UOS):
        assert oracle.block_exponent(0.0, rule) == -127
        assert oracle.block_exponent(1e-45, rule) == -127       # FP32 subnormal
        assert oracle.block_exponent(2.0 ** -126, rule) == -127
    assert oracle.block_exponent(3.3895313892515355e38, oracle.RULE_OCP) == 125   # BF16 max
    assert oracle.block_exponent(3.3895313892515355e38, oracle.RULE_UOS) == 126


# ----------------------------------------------------------------- E4M3
def _e4m3_from_fields(code: int) -> float:
    s, e, m = code >> 7, (code >> 3) & 0xF, code & 7
    if e == 0xF and m == 7:
        return float("nan")
    mag = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -mag if s else mag


def test_e4m3_decode_closed_forms():
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x38) == 1.0
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))
    assert math.copysign(1, oracle.e4m3_decode(0x80)) < 0
    vals = [oracle.e4m3_decode(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    for c in range(256):
        a, b = oracle.e4m3_decode(c), _e4m3_from_fields(c)
        assert (math.isnan(a) and math.isnan(b)) or a == b


def _rne_e4m3_magnitude(a: Fraction) -> Fraction:
    if a >= 448:
        return Fraction(448)
    if a < Fraction(1, 64):
        ulp = Fraction(1, 512)
    else:
        E = math.floor(math.log2(a))
        while Fraction(2) ** E > a:
            E -= 1
        while Fraction(2) ** (E + 1) <= a:
            E += 1
        ulp = Fraction(2) ** (E - 3)
    return min(round(a / ulp) * ulp, Fraction(448))


def test_e4m3_encode_first_principles():
    rng = np.random.default_rng(7)
    samples = [bf16_to_float(b) for b in ALL_BF16_FINITE[::3]]
    samples += list((2.0 ** rng.uniform(-14, 10, 20000)).astype(np.float32).astype(float))
    samples += [i / 1024 for i in range(0, 64)] + [448.0, 464.0, 465.0, 1e9, 2.0 ** -10, 3 * 2.0 ** -11]
    for v in samples:
        for s in (v, -v):
            code = oracle.e4m3_encode(s)
            assert (code >> 7) == (1 if math.copysign(1.0, s) < 0 else 0)
            assert Fraction(abs(oracle.e4m3_decode(code))) == _rne_e4m3_magnitude(abs(Fraction(s))), s


def test_e4m3_round_trip_all_finite_codes():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c
