"""The seeded input recipes (CPU): determinism per seed, the shapes of the named workloads,
and the value distributions they promise — N(0, std^2); outlier channels and tokens of the
stated count and factor; Student-t(3) values times a per-channel lognormal(0, 0.5) scale;
the FP8 calibration scale amax / 448.  Statistical checks use sample sizes whose
tolerances sit many standard errors wide."""

import math

import numpy as np
import torch

from mxfp4_block_scaled_mxq_b200 import inputs


def _f(t: torch.Tensor) -> np.ndarray:
    return t.float().numpy().astype(np.float64)


def test_same_seed_same_tensor_other_seed_other_tensor():
    a = inputs.heavy_tailed_bf16(64, 256, seed=5)
    b = inputs.heavy_tailed_bf16(64, 256, seed=5)
    c = inputs.heavy_tailed_bf16(64, 256, seed=6)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))
    assert a.dtype == torch.bfloat16 and a.shape == (64, 256)


def test_normal_draw_has_the_stated_spread():
    w = _f(inputs.normal_bf16(512, 512, 0.02, seed=7))
    assert abs(w.mean()) < 0.02 * 0.01
    assert abs(w.std() / 0.02 - 1.0) < 0.01  # 262144 draws: standard error ~0.14 %


def test_outlier_channels_count_and_factor():
    rows, cols, frac, factor = 2000, 1000, 0.02, 30.0
    x = _f(inputs.outlier_channels_bf16(rows, cols, frac, factor, seed=8))
    sd = x.std(axis=0)
    big = sd > math.sqrt(factor)  # between the two populations (1 and 30) on a log scale
    assert big.sum() == round(frac * cols)
    assert np.all(np.abs(sd[big] / factor - 1.0) < 0.1)
    assert np.all(np.abs(sd[~big] - 1.0) < 0.1)


def test_heavy_tailed_values_and_channel_scales():
    """Per channel, median |x| / 0.7649 estimates the lognormal factor (0.7649 is the
    median of |t| for Student-t with 3 degrees of freedom); log of those factors has
    standard deviation 0.5; normalised values exceed 3.182 (the t(3) 97.5 % quantile) in
    magnitude 5 % of the time."""
    rows, cols = 4000, 2048
    x = _f(inputs.heavy_tailed_bf16(rows, cols, seed=9))
    scale = np.median(np.abs(x), axis=0) / 0.7649
    assert abs(np.log(scale).std() - 0.5) < 0.03
    assert abs(np.log(scale).mean()) < 0.03
    tail = np.mean(np.abs(x / scale) > 3.182)
    assert abs(tail - 0.05) < 0.003
    # heavier than normal: a standard normal exceeds 3.182 only 0.15 % of the time
    assert tail > 10 * 0.0015


def test_token_outliers_scale_whole_rows():
    rows, cols = 2000, 512
    base = _f(inputs.heavy_tailed_bf16(rows, cols, seed=10))
    x = _f(inputs.heavy_tailed_bf16(rows, cols, seed=10, token_fraction=0.001, token_factor=50.0))
    ratio = np.abs(x).sum(axis=1) / np.abs(base).sum(axis=1)
    hot = ratio > 10
    assert hot.sum() == round(0.001 * rows)
    assert np.all(np.abs(ratio[hot] / 50.0 - 1.0) < 0.01)
    assert np.all(np.abs(ratio[~hot] - 1.0) < 1e-6)


def test_named_workload_shapes():
    x, w = inputs.tiny()
    assert tuple(x.shape) == (128, 512) and tuple(w.shape) == (512, 512)
    x, w = inputs.wan_ffn(which="up", M=8)
    assert tuple(x.shape) == (8, 5120) and tuple(w.shape) == (13824, 5120)
    x, w = inputs.wan_ffn(which="down", M=8)
    assert tuple(x.shape) == (8, 13824) and tuple(w.shape) == (5120, 13824)
    x, w, x_cal = inputs.flux_w4a8(which="mlp", M=8)
    assert tuple(x.shape) == (8, 3072) and tuple(w.shape) == (12288, 3072) and x_cal.shape == x.shape
    x, ws = inputs.wan_attn(M=8)
    assert tuple(x.shape) == (8, 5120) and len(ws) == 4 and all(tuple(t.shape) == (5120, 5120) for t in ws)
    x, w = inputs.m_sweep(16)
    assert tuple(x.shape) == (16, 5120) and tuple(w.shape) == (13824, 5120)


def test_flux_calibration_shares_the_outlier_channels_and_sets_the_scale():
    x, _, x_cal = inputs.flux_w4a8(M=2000)
    hot_x = _f(x).std(axis=0) > math.sqrt(30.0)
    hot_c = _f(x_cal).std(axis=0) > math.sqrt(30.0)
    assert hot_x.sum() == round(0.005 * 3072) and np.array_equal(hot_x, hot_c)
    s = inputs.static_fp8_scale(x_cal)
    amax = np.float32(np.abs(_f(x_cal)).max())
    assert s == float(np.float32(amax) / np.float32(448.0))
