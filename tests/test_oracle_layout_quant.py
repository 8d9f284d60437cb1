"""Pins for the oracle's scale-factor layout, block quantisers and rotation.

The bulk quantisers are checked against a recomposition from independently
written scalar rules (closed-form exponent, round-half-even in exact rationals),
so that a wrong block index, nibble order or row stride fails; the rotation is
checked against scipy's Sylvester Hadamard matrix and its orthogonality.
"""

import math
import struct
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import inputs


# ----------------------------------------------------------------- SF layout
def test_sf_offsets_atom_structure():
    K = 512  # 16 scale columns -> C = 16
    assert oracle.sf_offset(0, 0, K) == 0
    assert oracle.sf_offset(1, 0, K) == 16
    assert oracle.sf_offset(31, 0, K) == 31 * 16
    assert oracle.sf_offset(32, 0, K) == 4
    assert oracle.sf_offset(127, 3, K) == 31 * 16 + 3 * 4 + 3 == 511
    assert oracle.sf_offset(0, 4, K) == 512
    assert oracle.sf_offset(128, 0, K) == (16 // 4) * 512
    # sizes: rows padded to 128, columns to 4
    assert oracle.sf_bytes(1, 32) == 128 * 4
    assert oracle.sf_bytes(129, 160) == 256 * 8
    assert oracle.sf_bytes(32760, 5120) == 32768 * 160


@pytest.mark.parametrize("rows,K", [(1, 32), (130, 96), (257, 512), (128, 128)])
def test_sf_swizzle_is_a_padded_bijection(rows, K):
    rng = np.random.default_rng(rows + K)
    logical = rng.integers(1, 256, size=(rows, K // 32), dtype=np.uint8)
    phys = oracle.sf_swizzle(logical, rows, K)
    assert phys.size == oracle.sf_bytes(rows, K)
    np.testing.assert_array_equal(oracle.sf_unswizzle(phys, rows, K), logical)
    # every logical entry lands on a distinct byte; everything else is zero padding
    offs = {oracle.sf_offset(r, c, K) for r in range(rows) for c in range(K // 32)}
    assert len(offs) == rows * (K // 32)
    pad = np.ones(phys.size, bool)
    pad[list(offs)] = False
    assert not phys[pad].any()
    # each 512-byte atom holds one 128-row x 4-column block
    for r in range(0, rows, 37):
        for c in range(K // 32):
            o = oracle.sf_offset(r, c, K)
            assert o // 512 == (r // 128) * ((K // 32 + 3) // 4) + c // 4


# ----------------------------------------------------------------- scalar rules written independently here
def _f32(v):
    return struct.unpack("<f", struct.pack("<f", v))[0]


def _exp_ocp(amax: float) -> int:
    if amax == 0:
        return -127
    return max(-127, min(127, math.frexp(amax)[1] - 3))


def _exp_uos(amax: float) -> int:
    if amax == 0:
        return -127
    e = max(-127, math.ceil(math.log2(amax / 7.25)) - 2)   # start below, walk up exactly
    while Fraction(amax) > Fraction(29, 4) * Fraction(2) ** e:
        e += 1
    while e > -127 and Fraction(amax) <= Fraction(29, 4) * Fraction(2) ** (e - 1):
        e -= 1
    return min(e, 127)


def _rne_e2m1(v: float) -> int:
    a = abs(Fraction(v))
    if a >= 6:
        idx = 7
    else:
        ulp = Fraction(1, 2) if a < 2 else (Fraction(1) if a < 4 else Fraction(2))
        q = min(round(a / ulp) * ulp, Fraction(6))
        idx = [0, Fraction(1, 2), 1, Fraction(3, 2), 2, 3, 4, 6].index(q)
    return (8 if math.copysign(1.0, v) < 0 else 0) | idx


def _recompose(y: np.ndarray, rule: int):
    rows, K = y.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    sf = np.zeros((rows, K // 32), np.uint8)
    for r in range(rows):
        for b in range(K // 32):
            blk = y[r, 32 * b:32 * b + 32].astype(np.float64)
            amax = float(np.max(np.abs(blk)))
            e = _exp_ocp(amax) if rule == oracle.RULE_OCP else _exp_uos(amax)
            sf[r, b] = e + 127
            for i, v in enumerate(blk):
                k = 32 * b + i
                q = _rne_e2m1(math.ldexp(float(v), -e))
                codes[r, k // 2] |= q << (4 * (k % 2))
    return codes, sf


def _edge_case_rows(K: int) -> torch.Tensor:
    """All-zero block, BF16 subnormals, -0, a 7.25 tie, 6.0 boundary, BF16 max, 5.0 tie."""
    x = torch.zeros(8, K, dtype=torch.float32)
    x[1, :32] = torch.tensor(struct.unpack("<f", struct.pack("<I", 0x00010000))[0])  # bf16 subnormal
    x[1, 32:64] = -0.0
    x[2, :32] = 1.0
    x[2, 5] = 7.25
    x[3, :32] = 0.3
    x[3, 0] = 6.0
    x[4, :32] = -8.0
    x[5, 0] = 3.3895313892515355e38
    x[5, 1] = -3.3895313892515355e38
    x[6, :32] = 5.0
    x[6, 0] = 7.5
    x[7] = torch.linspace(-9, 9, K)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rule", [oracle.RULE_OCP, oracle.RULE_UOS])
def test_quantize_mxfp4_matches_recomposition(rule):
    x, _ = inputs.tiny(seed=0)
    x = torch.cat([x[:6], _edge_case_rows(512)])
    codes, sf = oracle.quantize_mxfp4(x, rule=rule, hadamard=False)
    want_codes, want_sf = _recompose(x.float().numpy(), rule)
    np.testing.assert_array_equal(sf, want_sf)
    np.testing.assert_array_equal(codes, want_codes)


def test_quantize_worked_examples():
    K = 32
    def q(vals, rule):
        x = torch.tensor([vals], dtype=torch.float32).to(torch.bfloat16)
        c, s = oracle.quantize_mxfp4(x, rule=rule)
        return int(s[0, 0]), int(c[0, 0] & 0xF), c
    ones = [1.0] * K
    assert q(ones, oracle.RULE_OCP)[:2] == (125, 0x6)
    assert q(ones, oracle.RULE_UOS)[:2] == (125, 0x6)
    m75 = [7.5] + [0.0] * 31
    assert q(m75, oracle.RULE_OCP)[:2] == (127, 0x7)
    assert q(m75, oracle.RULE_UOS)[:2] == (128, 0x6)
    m725 = [7.25] + [0.0] * 31
    assert q(m725, oracle.RULE_OCP)[:2] == (127, 0x7)
    assert q(m725, oracle.RULE_UOS)[:2] == (127, 0x7)
    m8 = [-8.0] + [0.0] * 31
    assert q(m8, oracle.RULE_OCP)[:2] == (128, 0xE)
    assert q(m8, oracle.RULE_UOS)[:2] == (128, 0xE)
    assert q([0.0] * K, oracle.RULE_OCP)[:2] == (0, 0x0)
    five = [5.0, 7.0] + [0.0] * 30            # e = 0, 5.0 -> 4 (tie to even)
    assert q(five, oracle.RULE_OCP)[:2] == (127, 0x6)
    neg = [-0.1, 7.0] + [0.0] * 30
    assert q(neg, oracle.RULE_OCP)[:2] == (127, 0x8)
    # nibble order: element 0 in the low nibble, element 1 in the high nibble
    c = q([0.5, 1.0, 6.0] + [0.0] * 29, oracle.RULE_OCP)[2]   # e = 0
    assert c[0, 0] == (0x2 << 4) | 0x1 and c[0, 1] == 0x7


def test_quantize_handles_row_stride_and_ragged_rows():
    x = inputs.normal_bf16(37, 96, 1.0, seed=11)
    codes, sf = oracle.quantize_mxfp4(x)
    for r in (0, 17, 36):
        c1, s1 = oracle.quantize_mxfp4(x[r:r + 1].clone())
        np.testing.assert_array_equal(codes[r:r + 1], c1)
        np.testing.assert_array_equal(sf[r:r + 1], s1)


def test_dequant_error_bound():
    """|x - deq(q(x))| <= half an E2M1 step at the block scale, or the clip to 6 * 2^e."""
    x, _ = inputs.tiny(seed=0)
    codes, sf = oracle.quantize_mxfp4(x)
    deq = oracle.dequant_mxfp4(codes, oracle.sf_swizzle(sf, 128, 512), 128, 512)
    xf = x.double().numpy()
    for b in range(512 // 32):
        e = sf[:, b].astype(np.float64) - 127
        blk = xf[:, 32 * b:32 * b + 32]
        err = np.abs(blk - deq[:, 32 * b:32 * b + 32])
        step = np.where(np.abs(blk) < 2 * 2.0 ** e[:, None], 0.25, np.where(np.abs(blk) < 4 * 2.0 ** e[:, None], 0.5, 1.0))
        bound = np.maximum(step * 2.0 ** e[:, None], np.abs(blk) - 6 * 2.0 ** e[:, None])
        assert np.all(err <= bound + 1e-300)


# ----------------------------------------------------------------- rotation
def test_hadamard_scale_constant():
    assert struct.unpack("<I", struct.pack("<f", oracle.hadamard_scale()))[0] == 0x3DB504F3
    assert oracle.hadamard_scale() == _f32(2.0 ** -3.5)


def test_fwht_is_sylvester_hadamard():
    H = scipy.linalg.hadamard(128)
    c = np.float32(oracle.hadamard_scale())
    for j in range(128):
        e = np.zeros(128, np.float32)
        e[j] = 1.0
        np.testing.assert_array_equal(oracle.fwht128(e), (H[:, j] * c).astype(np.float32))
    assert np.array_equal(H @ H.T, 128 * np.eye(128, dtype=H.dtype))


def test_fwht_matches_dense_product_and_is_orthonormal():
    rng = np.random.default_rng(3)
    R = scipy.linalg.hadamard(128) / math.sqrt(128.0)
    for _ in range(20):
        x = rng.standard_normal(128).astype(np.float32)
        y = oracle.fwht128(x).astype(np.float64)
        ref = R @ x.astype(np.float64)
        assert np.max(np.abs(y - ref)) <= 1e-6 * np.max(np.abs(ref))
    # (X R)(W R)^T == X W^T in FP64 for the rotated rows the quantiser sees
    x = inputs.normal_bf16(4, 256, 1.0, seed=5)
    w = inputs.normal_bf16(3, 256, 0.02, seed=6)
    xr = oracle.rotate_rows(x).astype(np.float64)
    wr = oracle.rotate_rows(w).astype(np.float64)
    lhs = xr @ wr.T
    rhs = x.double().numpy() @ w.double().numpy().T
    assert np.max(np.abs(lhs - rhs)) <= 1e-5 * np.max(np.abs(rhs))
    np.testing.assert_allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x.double().numpy(), axis=1), rtol=1e-6)


def test_quantize_with_hadamard_is_quantize_of_rotated_rows():
    x = inputs.heavy_tailed_bf16(6, 256, seed=9, token_fraction=0.2, token_factor=50.0)
    y = oracle.rotate_rows(x)
    for rule in (oracle.RULE_OCP, oracle.RULE_UOS):
        codes, sf = oracle.quantize_mxfp4(x, rule=rule, hadamard=True)
        want_codes, want_sf = _recompose(y, rule)
        np.testing.assert_array_equal(sf, want_sf)
        np.testing.assert_array_equal(codes, want_codes)


# ----------------------------------------------------------------- FP8 activations
def test_quantize_fp8_matches_elementwise_rule():
    x, _, x_cal = inputs.flux_w4a8(seed=3000, M=64)
    s = inputs.static_fp8_scale(x_cal)
    inv = np.float32(1.0) / np.float32(s)
    q = oracle.quantize_fp8(x, s)
    xv = x.float().numpy()
    prods = (xv * inv).astype(np.float32)
    for (r, k) in [(0, 0), (3, 17), (63, 3071)] + [(int(a), int(b)) for a, b in zip(*np.nonzero(np.abs(xv) > 10))][:50]:
        assert q[r, k] == oracle.e4m3_encode(float(prods[r, k]))
    # every value within calibration range decodes within half an E4M3 ulp
    deq = np.vectorize(oracle.e4m3_decode)(q[:8]).astype(np.float64)
    rel = np.abs(deq - prods[:8]) / np.maximum(np.abs(prods[:8]), 2.0 ** -6)
    assert np.all(rel <= 2.0 ** -4 + 1e-12)
