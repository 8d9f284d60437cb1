"""GPU parity of the precision-selection measurement: the FP64 SQNR sums (against the
oracle's, to FP64 rounding), and the SQNR of plain and transform-enabled W4A4 layers
(against the oracle's FP64 layers, within 0.05 dB: the device reference is the BF16
cuBLAS layer and the device outputs are BF16, both ~2^-9 relative) with the decisions
they lead to.

[AMD Quark adds native W4A8 mixed-precision for Wan2.2 video generation on MI350 --
 "Block-level SQNR calibration"]
"""

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import build, inputs, mxq, policy
from parity import assert_status_clean

pytestmark = pytest.mark.gpu

DB_TOL = 0.05


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    mxq.lib()
    yield
    assert_status_clean()


@pytest.mark.parametrize("M,N,ld", [(1, 8, 8), (37, 53, 64), (300, 1000, 1000)])
def test_sqnr_sums(M, N, ld):
    g = torch.Generator().manual_seed(M + N)
    ref = torch.randn(M, ld, generator=g).to(torch.bfloat16)
    y = (ref.float() + 0.1 * torch.randn(M, ld, generator=g)).to(torch.bfloat16)
    acc = torch.zeros(2, dtype=torch.float64, device="cuda")
    yd, rd = y.cuda(), ref.cuda()
    mxq.mxq_sqnr_accumulate(yd.data_ptr(), ld, rd.data_ptr(), ld, M, N, False, acc)
    mxq.mxq_sqnr_accumulate(yd.data_ptr(), ld, rd.data_ptr(), ld, M, N, True, acc)  # accumulates: twice
    torch.cuda.synchronize()
    s, n = oracle.sqnr_sums(y[:, :N].double().numpy(), ref[:, :N].double().numpy())
    got = acc.cpu().numpy()
    np.testing.assert_allclose(got, [2 * s, 2 * n], rtol=1e-12)


def _oracle_layer_sums(x, w, transform):
    M, K = x.shape
    N = w.shape[0]
    ref = x.double().numpy() @ w.double().numpy().T
    if transform:
        lam, inv = oracle.smooth_factors(oracle.channel_absmax(x, True), oracle.channel_absmax(w, True), 0.5)
        a, asl = oracle.quantize_mxfp4_smooth(x, inv, hadamard=True)
        b, bsl = oracle.quantize_mxfp4_smooth(w, lam, hadamard=True)
    else:
        a, asl = oracle.quantize_mxfp4(x)
        b, bsl = oracle.quantize_mxfp4(w)
    y = oracle.gemm(a, oracle.sf_swizzle(asl, M, K), b, oracle.sf_swizzle(bsl, N, K), M, N, K)
    return np.array(oracle.sqnr_sums(y, ref))


LAYERS = {  # synthetic calibration layers (x, w) with different activation statistics
    "normal": lambda: (inputs.normal_bf16(128, 512, 1.0, seed=2), inputs.normal_bf16(264, 512, 0.02, seed=1)),
    "outlier_channels": lambda: (inputs.outlier_channels_bf16(128, 512, 0.02, 30.0, seed=3),
                                 inputs.normal_bf16(264, 512, 0.02, seed=1)),
    "heavy_tailed": lambda: (inputs.heavy_tailed_bf16(96, 384, seed=4), inputs.normal_bf16(200, 384, 0.02, seed=7)),
}
HIGH, LOW = 15.5, 14.0


@pytest.mark.parametrize("name", list(LAYERS))
def test_layer_sqnr_and_decision(name):
    x, w = LAYERS[name]()
    got = policy.select_block_precision([(x.cuda(), w.cuda())], HIGH, LOW)
    sp = oracle.sqnr_db(*_oracle_layer_sums(x, w, False))
    st = oracle.sqnr_db(*_oracle_layer_sums(x, w, True))
    assert abs(got.sqnr_plain_db - sp) <= DB_TOL, (got, sp)
    assert abs(got.sqnr_transform_db - st) <= DB_TOL, (got, st)
    # the decision is compared where no SQNR sits within the tolerance of a threshold
    if min(abs(v - t) for v in (sp, st) for t in (HIGH, LOW)) > DB_TOL:
        assert got.precision == oracle.select_precision(sp, st, HIGH, LOW)


def test_block_sums_over_layers():
    """A block's SQNR is taken over all its layers' outputs together."""
    pairs = [LAYERS[n]() for n in LAYERS]
    got = policy.select_block_precision([(x.cuda(), w.cuda()) for x, w in pairs], HIGH, LOW)
    plain = sum(_oracle_layer_sums(x, w, False) for x, w in pairs)
    tr = sum(_oracle_layer_sums(x, w, True) for x, w in pairs)
    assert abs(got.sqnr_plain_db - oracle.sqnr_db(*plain)) <= DB_TOL
    assert abs(got.sqnr_transform_db - oracle.sqnr_db(*tr)) <= DB_TOL


def test_outlier_channels_select_the_transform():
    """2 % of the channels 30x larger: plain W4A4 falls below 15.5 dB (14.2 in the oracle),
    the rotation + SmoothQuant lifts it above (16.0): transform-enabled W4A4."""
    x, w = LAYERS["outlier_channels"]()
    got = policy.select_block_precision([(x.cuda(), w.cuda())], HIGH, LOW)
    assert got.precision == mxq.MXQ_PREC_W4A4_TRANSFORM, got
