"""GPU parity of the MXFP4 -> BF16 expansion and of the quantise-dequantise (fake
quantisation) pass: BF16 bit patterns equal to the oracle's, element by element."""

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import build, inputs, mxq
from parity import assert_status_clean, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    mxq.lib()
    yield
    assert_status_clean()


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _all_finite_bf16(perm_seed=None) -> torch.Tensor:
    bits = np.arange(1 << 16, dtype=np.uint32)
    finite = bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    if perm_seed is not None:
        finite = np.random.default_rng(perm_seed).permutation(finite)
    n = finite.size // 128 * 128
    return torch.from_numpy(finite[:n].astype(np.int16)).view(torch.bfloat16).reshape(-1, 128)


@pytest.mark.parametrize("rows,K", [(1, 32), (37, 96), (128, 512), (300, 1280)])
def test_dequant_random_codes_and_scales(rows, K):
    """Every code nibble, scale bytes over the whole finite E8M0 range (0 .. 254),
    including products that are FP32 subnormals or overflow to Inf."""
    rng = np.random.default_rng(rows * 7 + K)
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    sl = rng.integers(0, 255, (rows, K // 32), dtype=np.uint8)
    sl.flat[: min(sl.size, 4)] = [0, 1, 253, 254][: min(sl.size, 4)]
    sf = oracle.sf_swizzle(sl, rows, K)
    out = mxq.dequant_mxfp4(torch.from_numpy(codes).cuda(), torch.from_numpy(sf).cuda(), K)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(out), oracle.dequant_mxfp4_bf16(codes, sf, rows, K))


def test_dequant_of_packed_weights_with_row_stride():
    w = inputs.normal_bf16(200, 640, 0.02, seed=11)
    codes, sf = mxq.pack_weight(w.cuda())
    out = torch.full((200, 704), float("nan"), dtype=torch.bfloat16, device="cuda")
    mxq.dequant_mxfp4(codes, sf, 640, out=out[:, :640])
    torch.cuda.synchronize()
    want = oracle.dequant_mxfp4_bf16(codes.cpu().numpy(), sf.cpu().numpy(), 200, 640)
    np.testing.assert_array_equal(_bits(out[:, :640]), want)
    assert torch.isnan(out[:, 640:].float()).all()  # the row padding is not written


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS])
def test_qdq_every_bf16_value(rule):
    for x in (_all_finite_bf16(), _all_finite_bf16(perm_seed=2)):
        got = mxq.qdq_act(x.cuda(), rule=rule)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_bits(got), oracle.qdq_mxfp4(x, rule=rule))


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS])
@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (130, 384), (257, 1024)])
def test_qdq_matches_oracle(rule, hadamard, M, K):
    x = inputs.heavy_tailed_bf16(M, K, seed=M + K)
    got = mxq.qdq_act(x.cuda(), rule=rule, hadamard128=hadamard)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(got), oracle.qdq_mxfp4(x, rule=rule, hadamard=hadamard))


def test_qdq_ragged_k_and_strides():
    """K % 128 == 32 (a partial column tile), padded input and output rows."""
    x_full = inputs.outlier_channels_bf16(77, 256, 0.02, 20.0, seed=5)
    x = x_full[:, :160]
    out = torch.zeros(77, 176, dtype=torch.bfloat16, device="cuda")
    mxq.qdq_act(x_full.cuda()[:, :160], out=out[:, :160])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(out[:, :160]), oracle.qdq_mxfp4(x.contiguous()))
    assert (out[:, 160:].float() == 0).all()


def test_qdq_equals_dequant_of_quantiser_output():
    """The fused pass and quantise -> expand give the same BF16 values."""
    x = inputs.heavy_tailed_bf16(200, 512, seed=3)
    xd = x.cuda()
    q, sf = mxq.quantize_act(xd, mxq.MXQ_SCALE_UOS, True)
    a = mxq.dequant_mxfp4(q, sf, 512)
    b = mxq.qdq_act(xd, rule=mxq.MXQ_SCALE_UOS, hadamard128=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(a), _bits(b))


@pytest.mark.parametrize("M,K", [(1, 64), (300, 3072)])
def test_qdq_fp8(M, K):
    x, _, x_cal = inputs.flux_w4a8(M=M)
    x = x[:, :K].contiguous()
    s = inputs.static_fp8_scale(x_cal)
    got = mxq.qdq_act(x.cuda(), fmt=mxq.MXQ_ACT_FP8_E4M3, act_scale=s)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(got), oracle.qdq_fp8(x, s))


def test_qdq_fp8_every_bf16_value():
    x = _all_finite_bf16()
    for s in (1.0, 0.0123, 3.5e-3):
        got = mxq.qdq_act(x.cuda(), fmt=mxq.MXQ_ACT_FP8_E4M3, act_scale=s)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_bits(got), oracle.qdq_fp8(x, s))


@pytest.mark.slow
def test_full_size_qdq_wan_ffn_activations():
    x, _ = inputs.wan_ffn(which="up", device="cuda")
    got = mxq.qdq_act(x)
    torch.cuda.synchronize()
    rows = sample_rows(x.shape[0], 96)
    idx = torch.as_tensor(rows, device="cuda")
    np.testing.assert_array_equal(_bits(got[idx]), oracle.qdq_mxfp4(x[idx].cpu()))


@pytest.mark.parametrize("fmt,hadamard", [(mxq.MXQ_ACT_MXFP4, False), (mxq.MXQ_ACT_MXFP4, True),
                                          (mxq.MXQ_ACT_FP8_E4M3, False)])
def test_outputs_stay_inside_their_rows(fmt, hadamard):
    """QDQ (and, for plain MXFP4, the expansion) into buffers with a padded row stride
    (+64 columns) and 3 rows more than written, filled with a sentinel: only the
    [rows][K] block changes, and it equals the oracle's bits (ragged rows: 130)."""
    rows, K, s = 130, 384, 0.05
    x = inputs.heavy_tailed_bf16(rows, K, seed=61)
    sentinel = -12288.0  # exact in BF16

    def padded():
        return torch.full((rows + 3, K + 64), sentinel, dtype=torch.bfloat16, device="cuda")

    def check(buf, want_bits):
        host = buf.float().cpu()
        assert (host[:rows, K:] == sentinel).all() and (host[rows:, :] == sentinel).all()
        np.testing.assert_array_equal(_bits(buf[:rows, :K]), want_bits)

    buf = padded()
    mxq.qdq_act(x.cuda(), fmt, mxq.MXQ_SCALE_OCP, hadamard, act_scale=s, out=buf[:rows, :K])
    torch.cuda.synchronize()
    if fmt == mxq.MXQ_ACT_FP8_E4M3:
        check(buf, oracle.qdq_fp8(x, s))
        return
    check(buf, oracle.qdq_mxfp4(x, hadamard=hadamard))
    if not hadamard:
        codes, sl = oracle.quantize_mxfp4(x)
        sf = oracle.sf_swizzle(sl, rows, K)
        buf2 = padded()
        mxq.dequant_mxfp4(torch.from_numpy(codes).cuda(), torch.from_numpy(sf).cuda(), K, out=buf2[:rows, :K])
        torch.cuda.synchronize()
        check(buf2, oracle.dequant_mxfp4_bf16(codes, sf, rows, K))
