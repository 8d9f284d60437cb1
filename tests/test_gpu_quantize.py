"""GPU parity of the quantisers: codes and E8M0 scales must equal the oracle's bit
for bit, over the whole physical scale buffer (padding included)."""

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import build, inputs, mxq
from parity import assert_status_clean

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    mxq.lib()
    yield
    assert_status_clean()


def _check_mxfp4(x: torch.Tensor, rule=mxq.MXQ_SCALE_OCP, hadamard=False, weight=False, rows=None):
    xd = x.cuda()
    if weight:
        q, sf = mxq.pack_weight(xd, rule, hadamard)
    else:
        q, sf = mxq.quantize_act(xd, rule, hadamard)
    torch.cuda.synchronize()
    M, K = x.shape
    q = q.cpu().numpy()
    sf = sf.cpu().numpy()
    if rows is None:
        want_q, want_sl = oracle.quantize_mxfp4(x.cpu(), rule=rule, hadamard=hadamard)
        np.testing.assert_array_equal(q, want_q)
        np.testing.assert_array_equal(sf, oracle.sf_swizzle(want_sl, M, K))
    else:
        want_q, want_sl = oracle.quantize_mxfp4(x.cpu()[torch.as_tensor(rows)], rule=rule, hadamard=hadamard)
        np.testing.assert_array_equal(q[rows], want_q)
        got_sl = oracle.sf_unswizzle(sf, M, K)
        np.testing.assert_array_equal(got_sl[rows], want_sl)


def _all_finite_bf16(perm_seed=None, max_biased_exp=254) -> torch.Tensor:
    bits = np.arange(1 << 16, dtype=np.uint32)
    finite = bits[((bits >> 7) & 0xFF) <= max_biased_exp].astype(np.uint16)
    if perm_seed is not None:
        finite = np.random.default_rng(perm_seed).permutation(finite)
    n = finite.size // 128 * 128
    t = torch.from_numpy(finite[:n].astype(np.int16)).view(torch.bfloat16)
    return t.reshape(-1, 128)


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS])
def test_every_bf16_value(rule):
    _check_mxfp4(_all_finite_bf16(), rule)           # blocks of neighbouring bit patterns
    _check_mxfp4(_all_finite_bf16(perm_seed=1), rule)  # the same values under other block scales


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS])
def test_every_bf16_value_rotated(rule):
    """Every BF16 value below 2^119 through the 128-point rotation (rows of neighbouring bit
    patterns and a shuffled order), so that no butterfly sum overflows FP32 (a row mixing
    +Inf and -Inf would give Inf - Inf, outside the contract; single overflows to Inf are
    covered by test_edge_blocks); tiny rows give FP32-subnormal rotated values.  Codes and
    scales bit for bit."""
    _check_mxfp4(_all_finite_bf16(max_biased_exp=245), rule, hadamard=True)
    _check_mxfp4(_all_finite_bf16(perm_seed=2, max_biased_exp=245), rule, hadamard=True)


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS])
def test_rotated_blocks_near_the_bottom_of_the_fp32_range(rule):
    """Heavy-tailed rows scaled so that block maxima sit between 2^-130 and 2^-110: the
    rotated values of such blocks are partly FP32-subnormal and their block scales reach the
    bottom of the E8M0 range, where the quantiser multiplies by 1/sqrt(128) and by 2^-e
    separately."""
    g = torch.Generator().manual_seed(5)
    base = inputs.heavy_tailed_bf16(96, 1024, seed=9).float()
    scale = torch.pow(2.0, -torch.randint(108, 132, (96, 1), generator=g).float())
    x = (base * scale).to(torch.bfloat16)
    _check_mxfp4(x, rule, hadamard=True)


def test_tiny_config_ocp():
    x, w = inputs.tiny(seed=0)
    _check_mxfp4(x)
    _check_mxfp4(w, weight=True)


def test_edge_blocks():
    K = 256
    x = torch.zeros(9, K)
    x[1, :32] = -0.0
    x[2, :32] = torch.tensor(np.float32(1e-40))            # FP32/BF16 subnormal block
    x[3, :32] = 1.0
    x[3, 7] = 7.25                                          # UOS tie
    x[4, :32] = -8.0
    x[5, 0] = 3.3895313892515355e38                         # BF16 max
    x[5, 32] = -3.3895313892515355e38
    x[6, :32] = 5.0
    x[6, 0] = 7.0
    x[7, :] = torch.linspace(-7.5, 7.5, K)
    x[8, 64:96] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4)
    xb = x.to(torch.bfloat16)
    for rule in (mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS):
        for had in (False, True):
            _check_mxfp4(xb, rule, had)


@pytest.mark.parametrize("M,K", [(1, 32), (7, 96), (130, 160), (129, 384), (300, 4064)])
def test_ragged_shapes(M, K):
    x = inputs.heavy_tailed_bf16(M, K, seed=M + K)
    _check_mxfp4(x, mxq.MXQ_SCALE_OCP)
    _check_mxfp4(x, mxq.MXQ_SCALE_UOS, weight=True)


def test_leading_dimension():
    full = inputs.normal_bf16(70, 320, 1.0, seed=3).cuda()
    view = full[:, 64:320]        # ldx = 320, K = 256
    q, sf = torch.empty(70, 128, dtype=torch.uint8, device="cuda"), torch.empty(mxq.mxq_sf_bytes(70, 256), dtype=torch.uint8, device="cuda")
    mxq.mxq_quantize_act(view.data_ptr(), 70, 256, 320, mxq.MXQ_ACT_MXFP4, mxq.MXQ_SCALE_OCP, 0, 1.0, q, sf)
    want_q, want_sl = oracle.quantize_mxfp4(full.cpu()[:, 64:].contiguous())
    np.testing.assert_array_equal(q.cpu().numpy(), want_q)
    np.testing.assert_array_equal(sf.cpu().numpy(), oracle.sf_swizzle(want_sl, 70, 256))


@pytest.mark.parametrize("rule", [mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS])
def test_hadamard_attention_activations(rule):
    x, ws = inputs.wan_attn(M=1000)
    _check_mxfp4(x, rule, hadamard=True)
    _check_mxfp4(ws[0][:300], mxq.MXQ_SCALE_OCP, hadamard=True, weight=True)


def test_fp8_static_activations():
    x, _, x_cal = inputs.flux_w4a8(M=512)
    s = inputs.static_fp8_scale(x_cal)
    q = mxq.quantize_act_fp8(x.cuda(), s)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(q.cpu().numpy(), oracle.quantize_fp8(x, s))
    # out-of-calibration values saturate, signs and zeros are kept
    y = torch.tensor([[0.0, -0.0, 1e-30, -1e-30, 1e6, -1e6, 448.0, 3.0] * 4], dtype=torch.bfloat16)
    q = mxq.quantize_act_fp8(y.cuda(), 1.0)
    np.testing.assert_array_equal(q.cpu().numpy(), oracle.quantize_fp8(y, 1.0))


@pytest.mark.parametrize("M,K,pad", [(17, 96, 0), (130, 1056, 8), (1, 32, 8), (1048600, 32, 0)])
def test_fp8_ragged_shapes(M, K, pad):
    """Row counts that are not multiples of a CTA's 16 rows, chunk columns that do not fill
    a CTA's 64 (K = 96, 1056), 16-byte aligned row slices, and more row groups than one
    grid dimension holds (1048600 rows: the kernel strides over the rest)."""
    base = inputs.normal_bf16(M, K + pad, 3.0, seed=M + K)
    xd = base.cuda()[:, pad:]  # row stride K + pad on the device
    assert xd.stride(0) == K + pad
    s = 0.01
    q = mxq.quantize_act_fp8(xd, s)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(q.cpu().numpy(), oracle.quantize_fp8(base[:, pad:].contiguous(), s))


@pytest.mark.slow
def test_full_size_wan_ffn_up_activations():
    x, _ = inputs.wan_ffn(which="up", device="cuda")
    _check_mxfp4(x.cpu(), mxq.MXQ_SCALE_OCP)


@pytest.mark.slow
def test_full_size_wan_ffn_down_sampled_rows():
    x, _ = inputs.wan_ffn(which="down", device="cuda")
    from parity import sample_rows
    _check_mxfp4(x.cpu(), mxq.MXQ_SCALE_OCP, rows=sample_rows(x.shape[0], 512))


@pytest.mark.parametrize("pad", [8, 16])
@pytest.mark.parametrize("hadamard", [False, True])
def test_sixteen_byte_aligned_rows(pad, hadamard):
    """X as a column slice starting 8 elements (16 bytes) into a wider buffer: the rows are
    16-byte aligned only (pad 16: every row; pad 8: ldx % 16 == 8, so rows alternate between
    32- and 16-byte alignment).  Codes and scales bit for bit, for the activation quantiser
    (both rules), the weight packer, the FP8 quantiser and the quantise-dequantise kernel."""
    M, K = 130, 512
    x = inputs.heavy_tailed_bf16(M, K, seed=pad + 2 * hadamard)
    base = torch.zeros(M, K + pad, dtype=torch.bfloat16, device="cuda")
    base[:, 8:8 + K] = x.cuda()
    view = base[:, 8:8 + K]
    assert view.data_ptr() % 32 == 16 and view.stride(0) == K + pad
    for rule in (mxq.MXQ_SCALE_OCP, mxq.MXQ_SCALE_UOS):
        q, sf = mxq.quantize_act(view, rule, hadamard)
        w, wsf = mxq.pack_weight(view, rule, hadamard)
        qd = mxq.qdq_act(view, rule=rule, hadamard128=hadamard)
        torch.cuda.synchronize()
        want_q, want_sl = oracle.quantize_mxfp4(x, rule=rule, hadamard=hadamard)
        np.testing.assert_array_equal(q.cpu().numpy(), want_q)
        np.testing.assert_array_equal(sf.cpu().numpy(), oracle.sf_swizzle(want_sl, M, K))
        np.testing.assert_array_equal(w.cpu().numpy(), want_q)
        np.testing.assert_array_equal(wsf.cpu().numpy(), oracle.sf_swizzle(want_sl, M, K))
        bits = qd.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(bits, oracle.qdq_mxfp4(x, rule=rule, hadamard=hadamard))
    if not hadamard:
        s = 0.05
        q8 = mxq.quantize_act_fp8(view, s)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(q8.cpu().numpy(), oracle.quantize_fp8(x, s))
