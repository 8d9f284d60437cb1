"""GPU parity of the SmoothQuant pieces: channel maxima (bit-exact), migration factors
(FP32 powf against the FP64 definition, a few ulps), the quantiser with the per-channel
multiplier after the rotation (codes and scales bit-exact), and the smoothed W4A4 layer
end to end (GEMM tolerance).

[AMD Quark adds native W4A8 mixed-precision for Wan2.2 video generation on MI350 --
 "Fixed rotation selector": fixed Hadamard rotations followed by SmoothQuant]
"""

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import build, inputs, mxq
from parity import GEMM_TOL, assert_status_clean, gemm_rel_err, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    mxq.lib()
    yield
    assert_status_clean()


@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("rows,K", [(1, 128), (130, 384), (300, 1024)])
def test_channel_absmax(hadamard, rows, K):
    x = inputs.outlier_channels_bf16(rows, K, 0.02, 30.0, seed=rows + K)
    got = mxq.channel_absmax(x.cuda(), hadamard128=hadamard)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got.cpu().numpy(), oracle.channel_absmax(x, hadamard=hadamard))


def test_channel_absmax_ragged_k_stride_and_accumulate():
    """K % 128 == 32 (partial column tile), ldx > K, and two batches folded together."""
    full = inputs.heavy_tailed_bf16(200, 256, seed=21)
    a, b = full[:120, :160], full[120:, :160]
    out = mxq.channel_absmax(full.cuda()[:120, :160])
    mxq.channel_absmax(full.cuda()[120:, :160], out=out, accumulate=True)
    torch.cuda.synchronize()
    want = np.maximum(oracle.channel_absmax(a.contiguous()), oracle.channel_absmax(b.contiguous()))
    np.testing.assert_array_equal(out.cpu().numpy(), want)


@pytest.mark.parametrize("alpha", [0.0, 0.5, 0.85, 1.0])
def test_smooth_factors(alpha):
    rng = np.random.default_rng(22)
    ax = rng.lognormal(0.0, 2.0, 4099).astype(np.float32)
    aw = rng.lognormal(-4.0, 1.0, 4099).astype(np.float32)
    ax[:3] = [0.0, 1e-7, 3e4]
    aw[3:6] = [0.0, 1e-7, 2.0]
    lam, inv = mxq.smooth_factors(torch.from_numpy(ax).cuda(), torch.from_numpy(aw).cuda(), alpha)
    torch.cuda.synchronize()
    want_lam, _ = oracle.smooth_factors(ax, aw, alpha)
    np.testing.assert_allclose(lam.cpu().numpy(), want_lam, rtol=5e-7)
    np.testing.assert_array_equal(inv.cpu().numpy(), np.float32(1.0) / lam.cpu().numpy())


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS])
@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("rows,K", [(1, 128), (131, 384), (257, 1024)])
def test_quantize_smooth_bit_exact(rule, hadamard, rows, K):
    x = inputs.outlier_channels_bf16(rows, K, 0.02, 30.0, seed=3 * rows + K)
    rng = np.random.default_rng(rows + 7 * K)
    chan = rng.lognormal(0.0, 1.5, K).astype(np.float32)  # arbitrary positive factors
    q, sf = mxq.quantize_smooth(x.cuda(), torch.from_numpy(chan).cuda(), rule, hadamard)
    torch.cuda.synchronize()
    want_q, want_sl = oracle.quantize_mxfp4_smooth(x, chan, rule=rule, hadamard=hadamard)
    np.testing.assert_array_equal(q.cpu().numpy(), want_q)
    np.testing.assert_array_equal(sf.cpu().numpy(), oracle.sf_swizzle(want_sl, rows, K))


def test_quantize_smooth_ragged_k_and_stride():
    full = inputs.heavy_tailed_bf16(77, 256, seed=23)
    chan = np.random.default_rng(24).lognormal(0.0, 1.0, 160).astype(np.float32)
    q, sf = mxq.quantize_smooth(full.cuda()[:, :160], torch.from_numpy(chan).cuda())
    torch.cuda.synchronize()
    want_q, want_sl = oracle.quantize_mxfp4_smooth(full[:, :160].contiguous(), chan)
    np.testing.assert_array_equal(q.cpu().numpy(), want_q)
    np.testing.assert_array_equal(sf.cpu().numpy(), oracle.sf_swizzle(want_sl, 77, 160))


@pytest.mark.parametrize("hadamard", [False, True])
def test_smoothed_layer_end_to_end(hadamard):
    """Calibrate on the activations, migrate, quantise both sides, W4A4 GEMM -- each
    side computing its own factors -- then compare D with the oracle's layer."""
    M, K, N = 300, 512, 392
    x = inputs.outlier_channels_bf16(M, K, 0.02, 30.0, seed=25)
    w = inputs.normal_bf16(N, K, 0.02, seed=26)
    xd, wd = x.cuda(), w.cuda()
    lam, inv = mxq.smooth_factors(mxq.channel_absmax(xd, hadamard), mxq.channel_absmax(wd, hadamard), 0.5)
    wc, wsf = mxq.quantize_smooth(wd, lam, hadamard128=hadamard)
    q, sf = mxq.quantize_smooth(xd, inv, hadamard128=hadamard)
    d = mxq.gemm_w4a4(q, sf, wc, wsf, M, N, K)
    torch.cuda.synchronize()
    o_lam, o_inv = oracle.smooth_factors(oracle.channel_absmax(x, hadamard), oracle.channel_absmax(w, hadamard), 0.5)
    a, asl = oracle.quantize_mxfp4_smooth(x, o_inv, hadamard=hadamard)
    b, bsl = oracle.quantize_mxfp4_smooth(w, o_lam, hadamard=hadamard)
    y = oracle.gemm(a, oracle.sf_swizzle(asl, M, K), b, oracle.sf_swizzle(bsl, N, K), M, N, K)
    assert gemm_rel_err(d, np.arange(M), y) <= GEMM_TOL


@pytest.mark.slow
def test_full_size_smoothed_hadamard_activations():
    """The Wan attention-projection activations (32760 x 5120, rotated), row sample."""
    x, _ = inputs.wan_attn(device="cuda")
    chan_np = np.random.default_rng(27).lognormal(0.0, 1.0, x.shape[1]).astype(np.float32)
    q, sf = mxq.quantize_smooth(x, torch.from_numpy(chan_np).cuda(), mxq.MXQ_SCALE_UOS, True)
    torch.cuda.synchronize()
    M, K = x.shape
    rows = sample_rows(M, 64)
    idx = torch.as_tensor(rows, device="cuda")
    want_q, want_sl = oracle.quantize_mxfp4_smooth(x[idx].cpu(), chan_np, rule=oracle.RULE_UOS, hadamard=True)
    np.testing.assert_array_equal(q[idx].cpu().numpy(), want_q)
    np.testing.assert_array_equal(oracle.sf_unswizzle(sf.cpu().numpy(), M, K)[rows], want_sl)
