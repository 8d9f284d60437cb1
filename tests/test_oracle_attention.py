"""Pins of the oracle's MXFP4 attention (UOS + PNQ): its exponential, closed-form
outputs, and the properties the MXAttention page states.

[MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for MXFP4
 Attention -- TL;DR, "What it actually does"]
"""

import math

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import inputs


def _f32(x):
    return float(np.float32(x))


def test_pnq_exp2_accuracy():
    """Relative error against 2^(t - c) over the range softmax numerators use: below the
    degree-3 Taylor remainder of 2^g on |g| <= 1/2, (ln 2 / 2)^4 / 4! * 2^(1/2) = 8.50e-4,
    and above (ln 2 / 2)^4 / 4! = 6.01e-4, which it reaches near g = 1/2 (so a polynomial
    of another degree fails one side)."""
    ts = np.float32(np.linspace(-40.0, 8.0, 20011))
    worst = 0.0
    for t in ts:
        want = 2.0 ** (float(t) - 3)
        worst = max(worst, abs(oracle.pnq_exp2(float(t), 3) - want) / want)
    assert 5.5e-4 < worst < 8.6e-4, worst


@pytest.mark.parametrize("t", [-17.37, -0.001, 0.0, 2.5, 7.99])
def test_pnq_exp2_offset_is_an_exact_power_of_two(t):
    """Changing the integer offset scales the numerator by exactly a power of two (the
    property that makes the MXFP4 codes independent of the offset)."""
    t = _f32(t)
    a, b = oracle.pnq_exp2(t, 0), oracle.pnq_exp2(t, 5)
    assert a == b * 32.0


def test_pnq_exp2_flushes_below_2_to_minus_126():
    """Zero once the rounded integer part is below -126 (rint(-126.5) = -126: ties to even)."""
    assert oracle.pnq_exp2(-127.0, 0) == 0.0
    assert oracle.pnq_exp2(-126.6, 0) == 0.0
    assert oracle.pnq_exp2(-126.5, 0) > 0.0
    assert oracle.pnq_exp2(-126.0, 0) > 0.0


def test_pnq_exp2_is_exact_at_integers():
    """g = 0 at integer t, and p(0) = a_0 = 1: an exact power of two."""
    for t in (-100.0, -3.0, 0.0, 5.0):
        assert oracle.pnq_exp2(t, 2) == 2.0 ** (t - 2)


def test_equal_scores_average_the_values():
    """Identical keys: every score is equal, every numerator is equal, so O is the
    plain mean of the dequantised values over the keys (PNQ's l cancels exactly)."""
    H, d, S = 1, 64, 96
    q = inputs.normal_bf16(4, H * d, 1.0, seed=1)
    k = inputs.normal_bf16(1, H * d, 1.0, seed=2).repeat(S, 1)
    v = inputs.normal_bf16(S, H * d, 1.0, seed=3)
    out, ws = oracle.attention_mxfp4(q, k, v, H, d)
    codes, sl = oracle.quantize_mxfp4(v.t().contiguous(), rule=oracle.RULE_UOS)   # V^T, blocks along keys
    deq_vt = oracle.dequant_mxfp4(codes, oracle.sf_swizzle(sl, H * d, S), H * d, S)
    want = deq_vt.mean(axis=1)
    np.testing.assert_allclose(out[:, 0, :], np.broadcast_to(want, (4, d)), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(ws, 1.0, rtol=1e-14)


def test_one_dominant_key_returns_its_value():
    """One key's score exceeds the others' by more than 126 in base 2: every other
    numerator flushes to 0, so O is exactly that key's dequantised value row."""
    H, d, S = 1, 32, 64
    q = torch.zeros(1, d, dtype=torch.bfloat16)
    q[0, 0] = 24.0
    k = torch.zeros(S, d, dtype=torch.bfloat16)
    k[17, 0] = 24.0            # S = 576, t = 576 * log2(e) / sqrt(32) = 147 vs 0
    v = inputs.normal_bf16(S, d, 1.0, seed=4)
    out, _ = oracle.attention_mxfp4(q, k, v, H, d)
    codes, sl = oracle.quantize_mxfp4(v.t().contiguous(), rule=oracle.RULE_UOS)
    deq_vt = oracle.dequant_mxfp4(codes, oracle.sf_swizzle(sl, d, S), d, S)
    np.testing.assert_array_equal(out[0, 0], deq_vt[:, 17])


def _three_modes(scale, rule=oracle.RULE_UOS):
    H, d, S = 2, 128, 300
    q = inputs.normal_bf16(S, H * d, scale, seed=1)
    k = inputs.normal_bf16(S, H * d, scale, seed=2)
    v = inputs.normal_bf16(S, H * d, 1.0, seed=3)
    rows = np.arange(0, S, 7)
    return [oracle.attention_mxfp4(q, k, v, H, d, rows, rule=rule, mode=m) for m in (0, 1, 2)]


def test_pnq_preserves_normalisation_and_the_conventional_order_does_not():
    """PNQ: the implied attention weights of every row sum to 1 (by construction).
    Quantising after the row normalisation leaves rows whose weights do not."""
    (o0, w0), (o1, w1), _ = _three_modes(1.0)
    assert np.abs(w0 - 1.0).max() < 1e-12
    assert np.abs(w1 - 1.0).max() > 1e-3


def test_pnq_beats_the_conventional_order_on_peaked_attention():
    """Peaked score distributions (Q, K ~ N(0, 4)): PNQ's output is closer to the
    unquantised-P attention than quantise-after-normalise's (0.067 vs 0.101 here)."""
    (o0, _), (o1, _), (o2, _) = _three_modes(2.0)
    err = lambda o: np.linalg.norm(o - o2) / np.linalg.norm(o2)
    assert err(o0) < 0.8 * err(o1), (err(o0), err(o1))


@pytest.mark.parametrize("scale", [2.0, 3.0])
def test_uos_beats_ocp(scale):
    """UOS (Qmax = 7.25) against the stock OCP rule, both with PNQ, on peaked scores:
    the quantised P moves the output less from the unquantised-P attention (each rule
    against its own unquantised-P output, so only the numerators' quantisation differs;
    0.067 vs 0.081 and 0.040 vs 0.047 here -- on diffuse scores the two are within 2 %)."""
    (u, _), _, (u_ref, _) = _three_modes(scale, oracle.RULE_UOS)
    (o, _), _, (o_ref, _) = _three_modes(scale, oracle.RULE_OCP)
    err = lambda a, r: np.linalg.norm(a - r) / np.linalg.norm(r)
    assert err(u, u_ref) < err(o, o_ref), (err(u, u_ref), err(o, o_ref))


def _deq(x, rule):
    """MXFP4 round trip of the rows of x (blocks along the rows), FP64."""
    codes, sl = oracle.quantize_mxfp4(x.contiguous(), rule=rule)
    rows, K = x.shape
    return oracle.dequant_mxfp4(codes, oracle.sf_swizzle(sl, rows, K), rows, K)


@pytest.mark.parametrize("rule", [oracle.RULE_UOS, oracle.RULE_OCP])
def test_unquantised_mode_is_the_textbook_softmax_of_the_quantised_operands(rule):
    """With P left unquantised, the oracle is softmax(Q K^T / sqrt(d)) V over the
    dequantised MXFP4 Q and K (blocks along the head dimension) and V (blocks along the
    keys), head by head -- written here independently in FP64 NumPy.  The oracle takes
    the exponent in base 2 from FP32 scores, so the two agree to FP32 rounding; a wrong
    scale, a transposed product or a head mix-up would not."""
    H, d, Sq, Skv = 2, 64, 5, 70
    q = inputs.normal_bf16(Sq, H * d, 1.5, seed=41)
    k = inputs.normal_bf16(Skv, H * d, 1.5, seed=42)
    v = inputs.heavy_tailed_bf16(Skv, H * d, seed=43)
    got, ws = oracle.attention_mxfp4(q, k, v, H, d, rule=rule, mode=oracle.ATTN_UNQUANTISED_P)
    Q, K = _deq(q, rule), _deq(k, rule)
    Skv_pad = (Skv + 31) // 32 * 32
    vt = torch.zeros(H * d, Skv_pad, dtype=torch.bfloat16)
    vt[:, :Skv] = v.t()
    V = _deq(vt, rule)[:, :Skv].T  # [Skv][H*d]
    for h in range(H):
        cols = slice(h * d, (h + 1) * d)
        s = Q[:, cols] @ K[:, cols].T / math.sqrt(d)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        want = (p / p.sum(axis=1, keepdims=True)) @ V[:, cols]
        np.testing.assert_allclose(got[:, h, :], want, rtol=2e-5, atol=2e-5 * np.abs(want).max())
    np.testing.assert_allclose(ws, 1.0, rtol=1e-12)
