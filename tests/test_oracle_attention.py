"""Pins of the oracle's MXFP4 attention (UOS + PNQ): an independent FP64 NumPy
restatement of both quantisation orders, closed-form outputs, and the properties the
MXAttention page states.

[MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for MXFP4
 Attention -- TL;DR, "What it actually does"]
"""

import math

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import inputs


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
    numerator is below 2^-126, under a quarter of the smallest E8M0 step (2^-127 x 0.5
    is the least non-zero E2M1 value), so it quantises to 0 and O is exactly that key's
    dequantised value row."""
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


def _mx_round_rows(p, rule):
    """MXFP4 round trip of FP64 values in 32-element blocks along the last axis, written
    from the MX definition alone: the block scale is the smallest power of two 2^e with
    amax / 2^e < 8 (OCP) or <= 7.25 (UOS), e >= -127; each value goes to the nearest
    E2M1 magnitude (ties to the even code index), saturating at 6."""
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    blocks = p.reshape(p.shape[:-1] + (-1, 32))
    amax = np.abs(blocks).max(axis=-1, keepdims=True)
    mant, ex = np.frexp(amax)                          # amax = mant 2^ex, mant in [0.5, 1)
    e = np.where(amax > 0, ex - 1 - 2, -127)           # floor(log2 amax) - 2
    if rule == oracle.RULE_UOS:
        e = np.where(amax > np.ldexp(7.25, e), e + 1, e)
    e = np.maximum(e, -127)
    a = np.minimum(np.abs(blocks) / np.ldexp(1.0, e), 6.0)
    dist = np.abs(a[..., None] - grid)
    best = dist.min(axis=-1, keepdims=True)
    tied = dist == best
    # lowest index among the minima, unless a tie offers an even index
    idx = np.where(tied[..., ::2].any(axis=-1), np.argmax(tied * (np.arange(8) % 2 == 0), axis=-1),
                   np.argmax(tied, axis=-1))
    return (np.sign(blocks) * grid[idx] * np.ldexp(1.0, e)).reshape(p.shape)


@pytest.mark.parametrize("mode", [oracle.ATTN_PNQ, oracle.ATTN_NORMALISE_THEN_QUANTISE])
@pytest.mark.parametrize("rule,scale", [(oracle.RULE_UOS, 1.0), (oracle.RULE_UOS, 2.5), (oracle.RULE_OCP, 2.0)])
def test_quantised_p_matches_an_independent_fp64_restatement(mode, rule, scale):
    """PNQ (quantise the unnormalised exponentials, then sum the quantised values and
    divide) and the conventional order (normalise, then quantise) restated in FP64 NumPy:
    scores t = fl32(fl32(S) fl32(log2 e / sqrt d)), numerators 2^(t - ceil(max t)) by
    NumPy's exp2, MX blocks of 32 keys with the scale from the block maximum.  A wrong
    block maximum, offset, rounding rule or quantisation point moves whole codes, so
    agreement to 1e-12 leaves no room for any of them."""
    H, d, Sq, Skv = 2, 64, 6, 150        # 150 keys: a ragged last block, zero-padded
    q = inputs.normal_bf16(Sq, H * d, scale, seed=61)
    k = inputs.normal_bf16(Skv, H * d, scale, seed=62)
    v = inputs.heavy_tailed_bf16(Skv, H * d, seed=63)
    got, ws = oracle.attention_mxfp4(q, k, v, H, d, rule=rule, mode=mode)
    Q, K = _deq(q, rule), _deq(k, rule)
    Skv_pad = (Skv + 31) // 32 * 32
    vt = torch.zeros(H * d, Skv_pad, dtype=torch.bfloat16)
    vt[:, :Skv] = v.t()
    V = _deq(vt, rule).T                 # [Skv_pad][H*d], zero rows past Skv
    c32 = np.float32(1.4426950408889634 / math.sqrt(d))
    for h in range(H):
        cols = slice(h * d, (h + 1) * d)
        t = (Q[:, cols] @ K[:, cols].T).astype(np.float32) * c32          # FP32 product
        c = np.ceil(t.max(axis=1, keepdims=True).astype(np.float64))
        p = np.zeros((Sq, Skv_pad))
        p[:, :Skv] = np.exp2(t.astype(np.float64) - c)
        if mode == oracle.ATTN_PNQ:
            pq = _mx_round_rows(p, rule)
            w = pq / pq.sum(axis=1, keepdims=True)
        else:
            w = _mx_round_rows(p / p.sum(axis=1, keepdims=True), rule)
        want = w @ V[:, cols]
        np.testing.assert_allclose(got[:, h, :], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
        np.testing.assert_allclose(ws[:, h], w.sum(axis=1), rtol=1e-12)
    if mode == oracle.ATTN_PNQ:
        np.testing.assert_allclose(ws, 1.0, rtol=1e-12)


def test_the_restatement_sees_a_wrong_quantisation_point():
    """The restatement above tells the two orders apart on this input (so a swapped mode
    in the oracle would fail it)."""
    H, d, Sq, Skv = 1, 64, 6, 150
    q = inputs.normal_bf16(Sq, H * d, 2.5, seed=61)
    k = inputs.normal_bf16(Skv, H * d, 2.5, seed=62)
    v = inputs.heavy_tailed_bf16(Skv, H * d, seed=63)
    a, _ = oracle.attention_mxfp4(q, k, v, H, d, mode=oracle.ATTN_PNQ)
    b, _ = oracle.attention_mxfp4(q, k, v, H, d, mode=oracle.ATTN_NORMALISE_THEN_QUANTISE)
    assert np.abs(a - b).max() > 1e-3 * np.abs(a).max()
