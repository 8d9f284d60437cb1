"""GPU parity of MXFP4 attention with UOS + PNQ: the V^T quantiser bit for bit,
and the attention output against the oracle's FP64 attention (exact exponentials, MX block
maxima) on the same quantised operands: max|O - O_ref| / max|O_ref| <= 5e-3 (BF16 output
rounding, at most 2^-8 of a value, and FP32 accumulation; the kernel's numerator codes are
those of the exact exponential, which tests/test_attn_code_decisions.py proves on the
host).

[MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for MXFP4
 Attention -- TL;DR, "What it actually does"]
"""

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import build, inputs, mxq
from parity import assert_status_clean, sample_rows

pytestmark = pytest.mark.gpu

ATTN_TOL = 5e-3
D = 128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    mxq.lib()
    yield
    assert_status_clean()


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_UOS, mxq.MXQ_SCALE_OCP])
@pytest.mark.parametrize("S,HD", [(1, 128), (300, 256), (512, 128)])
def test_quantize_vt_bit_exact(rule, S, HD):
    v = inputs.heavy_tailed_bf16(S, HD, seed=S + HD)
    codes, sf = mxq.quantize_vt(v.cuda(), rule)
    torch.cuda.synchronize()
    Sp = mxq.mxq_attn_padded_keys(S)
    vt = torch.zeros(HD, Sp, dtype=torch.bfloat16)
    vt[:, :S] = v.t()
    want_c, want_sl = oracle.quantize_mxfp4(vt, rule=rule)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(sf.cpu().numpy(), oracle.sf_swizzle(want_sl, HD, Sp))


def _check(q, k, v, H, rule=mxq.MXQ_SCALE_UOS, rows=None):
    o = mxq.attention_mxfp4(q.cuda(), k.cuda(), v.cuda(), H, rule)
    torch.cuda.synchronize()
    Sq = q.shape[0]
    rows = np.arange(Sq) if rows is None else rows
    want, ws = oracle.attention_mxfp4(q, k, v, H, D, rows, rule=rule)
    got = o.float().cpu().numpy()[rows].reshape(len(rows), H, D)
    err = np.abs(got - want).max() / np.abs(want).max()
    assert err <= ATTN_TOL, err
    np.testing.assert_allclose(ws, 1.0, rtol=1e-12)
    return err


@pytest.mark.parametrize("Sq,Skv,H", [(1, 1, 1), (200, 300, 2), (128, 40, 1), (130, 512, 1), (257, 700, 2)])
def test_attention_shapes(Sq, Skv, H):
    """Ragged query tiles, a single partial key tile, exact and ragged key tiles."""
    q = inputs.normal_bf16(Sq, H * D, 1.0, seed=Sq)
    k = inputs.normal_bf16(Skv, H * D, 1.0, seed=Skv + 1)
    v = inputs.normal_bf16(Skv, H * D, 1.0, seed=Skv + 2)
    _check(q, k, v, H)


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_UOS, mxq.MXQ_SCALE_OCP])
@pytest.mark.parametrize("scale", [0.25, 2.0])
def test_attention_diffuse_and_peaked(rule, scale):
    """Diffuse (small scores) and peaked (Q, K ~ N(0, 4)) attention, both rules."""
    q = inputs.normal_bf16(160, 2 * D, scale, seed=11)
    k = inputs.normal_bf16(600, 2 * D, scale, seed=12)
    v = inputs.heavy_tailed_bf16(600, 2 * D, seed=13)
    _check(q, k, v, 2, rule)


def test_attention_rescales_when_the_maximum_jumps():
    """Keys after the first tile score ~8x higher: the running offset moves by far more
    than 8 in base 2, so O and l are rescaled in TMEM by exact powers of two."""
    q = inputs.normal_bf16(128, D, 1.0, seed=21)
    k = inputs.normal_bf16(768, D, 1.0, seed=22)
    k[256:] = (k[256:].float() * 8.0).to(torch.bfloat16)
    v = inputs.normal_bf16(768, D, 1.0, seed=23)
    _check(q, k, v, 1)


@pytest.mark.slow
def test_full_size_wan_self_attention_sampled():
    """Wan2.2-shaped self-attention (32760 tokens, 40 heads of 128): all heads on the
    GPU; two heads' sampled query rows against the oracle."""
    S, H = 32760, 40
    q = inputs.normal_bf16(S, H * D, 1.0, seed=31, device="cuda")
    k = inputs.normal_bf16(S, H * D, 1.0, seed=32, device="cuda")
    v = inputs.heavy_tailed_bf16(S, H * D, seed=33, device="cuda")
    o = mxq.attention_mxfp4(q, k, v, H)
    torch.cuda.synchronize()
    rows = sample_rows(S, 24)
    for h in (0, 39):
        cols = slice(h * D, (h + 1) * D)
        want, _ = oracle.attention_mxfp4(q[:, cols].cpu().contiguous(), k[:, cols].cpu().contiguous(),
                                         v[:, cols].cpu().contiguous(), 1, D, rows)
        got = o[:, cols].float().cpu().numpy()[rows]
        err = np.abs(got - want[:, 0, :]).max() / np.abs(want).max()
        assert err <= ATTN_TOL, (h, err)


def test_attention_writes_stay_inside_o():
    """O with a padded row stride (ldo = H*d + 64) inside a larger buffer filled with a
    sentinel: the padding columns and the rows past Sq keep it; O itself matches."""
    Sq, Skv, H = 130, 300, 2
    q = inputs.normal_bf16(Sq, H * D, 1.0, seed=51)
    k = inputs.normal_bf16(Skv, H * D, 1.0, seed=52)
    v = inputs.normal_bf16(Skv, H * D, 1.0, seed=53)
    sentinel = -12288.0  # exact in BF16
    buf = torch.full((Sq + 3, H * D + 64), sentinel, dtype=torch.bfloat16, device="cuda")
    mxq.attention_mxfp4(q.cuda(), k.cuda(), v.cuda(), H, out=buf[:Sq, :H * D])
    torch.cuda.synchronize()
    host = buf.float().cpu()
    assert (host[:Sq, H * D:] == sentinel).all()
    assert (host[Sq:, :] == sentinel).all()
    rows = np.arange(Sq)
    want, _ = oracle.attention_mxfp4(q, k, v, H, D, rows)
    got = host[:Sq, :H * D].numpy().reshape(Sq, H, D)
    assert np.abs(got - want).max() / np.abs(want).max() <= ATTN_TOL


def test_quantize_vt_sixteen_byte_aligned_rows():
    """V as a column slice 8 elements (16 bytes) into a wider buffer with ldv % 16 == 8:
    rows alternate between 32- and 16-byte alignment; V^T codes and scales bit for bit."""
    S, HD = 300, 256
    v = inputs.heavy_tailed_bf16(S, HD, seed=77)
    base = torch.zeros(S, HD + 8, dtype=torch.bfloat16, device="cuda")
    base[:, 8:] = v.cuda()
    view = base[:, 8:]
    assert view.data_ptr() % 32 == 16
    codes, sf = mxq.quantize_vt(view, mxq.MXQ_SCALE_UOS)
    torch.cuda.synchronize()
    Sp = mxq.mxq_attn_padded_keys(S)
    vt = torch.zeros(HD, Sp, dtype=torch.bfloat16)
    vt[:, :S] = v.t()
    want_c, want_sl = oracle.quantize_mxfp4(vt, rule=oracle.RULE_UOS)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(sf.cpu().numpy(), oracle.sf_swizzle(want_sl, HD, Sp))


def test_attention_blocks_spanning_the_e8m0_range():
    """Scores about 400 apart (base 2, +-204) inside one 32-key block: such blocks take the
    kernel's general path (the numerators scaled by explicit powers of two, keys far below
    the row maximum flushed), and rows whose strong keys sit in several blocks keep the
    usual path elsewhere.  The flushed numerators are below 2^-126 of the row's largest, so
    the exact-exponential oracle agrees within the tolerance."""
    Sq, Skv, d = 96, 320, D
    g = torch.Generator().manual_seed(91)
    q = (torch.randn(Sq, d, generator=g) * 0.5)
    q[:, 0] = 40.0
    k = (torch.randn(Skv, d, generator=g) * 0.5)
    k[:, 0] = torch.where(torch.rand(Skv, generator=g) < 0.5, torch.tensor(40.0), torch.tensor(-40.0))
    v = inputs.normal_bf16(Skv, d, 1.0, seed=92)
    err = _check(q.to(torch.bfloat16), k.to(torch.bfloat16), v, 1)
    assert err <= ATTN_TOL
