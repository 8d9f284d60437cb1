"""GPU parity of the one-call quantized linear layer (mxq_linear_w4a4): D against the
oracle's layer (GEMM tolerance), and the quantised activations the call leaves in its
workspace against the oracle's quantiser, bit for bit."""

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import build, inputs, mxq
from parity import GEMM_TOL, assert_status_clean, gemm_rel_err, oracle_w4a4, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    mxq.lib()
    yield
    assert_status_clean()


def _run(x, w, rule=mxq.MXQ_SCALE_OCP, alpha=1.0, bias=None, workspace=None):
    xd, wd = x.cuda(), w.cuda()
    wc, wsf = mxq.pack_weight(wd)
    M, K = x.shape
    ws = mxq.linear_workspace(M, K, "cuda") if workspace is None else workspace
    d = mxq.linear_w4a4_ws(xd, wc, wsf, w.shape[0], rule, alpha, None if bias is None else bias.cuda(), ws)
    torch.cuda.synchronize()
    return d, ws


def _check_workspace(x, ws, rule):
    M, K = x.shape
    want_c, want_sl = oracle.quantize_mxfp4(x, rule=rule)
    raw = ws.cpu().numpy()
    sf_off = (M * K // 2 + 1023) // 1024 * 1024
    np.testing.assert_array_equal(raw[: M * K // 2].reshape(M, K // 2), want_c)
    np.testing.assert_array_equal(raw[sf_off: sf_off + mxq.mxq_sf_bytes(M, K)], oracle.sf_swizzle(want_sl, M, K))


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS])
@pytest.mark.parametrize("M,N,K", [(129, 256, 256), (300, 520, 1280), (1000, 264, 384), (257, 136, 640),
                                   (64, 392, 512)])
def test_linear_layer(rule, M, N, K):
    x = inputs.heavy_tailed_bf16(M, K, seed=M + K)
    w = inputs.normal_bf16(N, K, 0.02, seed=N)
    d, ws = _run(x, w, rule)
    rows = np.arange(M)
    assert gemm_rel_err(d, rows, oracle_w4a4(x, w, rows, rule_a=rule)) <= GEMM_TOL
    _check_workspace(x, ws, rule)


def test_linear_layer_bias_alpha_and_workspace_reuse():
    """Two calls in a row on one workspace."""
    x1 = inputs.outlier_channels_bf16(700, 512, 0.02, 30.0, seed=41)
    x2 = inputs.heavy_tailed_bf16(700, 512, seed=42)
    w = inputs.normal_bf16(300, 512, 0.02, seed=43)
    bias = (torch.randn(300, generator=torch.Generator().manual_seed(44)) * 0.5).to(torch.bfloat16)
    ws = mxq.linear_workspace(700, 512, "cuda")
    rows = np.arange(700)
    for x in (x1, x2):
        d, _ = _run(x, w, alpha=0.37, bias=bias, workspace=ws)
        assert gemm_rel_err(d, rows, oracle_w4a4(x, w, rows, alpha=0.37, bias=bias)) <= GEMM_TOL
        _check_workspace(x, ws, mxq.MXQ_SCALE_OCP)


@pytest.mark.slow
@pytest.mark.parametrize("which", ["up", "down"])
def test_full_size_linear_wan_ffn(which):
    x, w = inputs.wan_ffn(which=which, device="cuda")
    wc, wsf = mxq.pack_weight(w)
    d = mxq.linear_w4a4_ws(x, wc, wsf, w.shape[0])
    torch.cuda.synchronize()
    rows = sample_rows(x.shape[0], 96)
    assert gemm_rel_err(d, rows, oracle_w4a4(x, w, rows)) <= GEMM_TOL
