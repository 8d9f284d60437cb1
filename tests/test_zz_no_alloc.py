"""mxq_linear_w4a4_static: the quantized linear layer with the library's fixed scratch
buffer instead of a caller workspace.  Same kernels as mxq_linear_w4a4, so the outputs
match it bit for bit; checked on two calls in a row with different inputs (no state
carried between calls) and against the oracle.  Collected last on purpose: it must pass
after everything else has used the device, as well as alone."""

import numpy as np
import pytest
import torch

from mxfp4_block_scaled_mxq_b200 import build, inputs, mxq
from parity import GEMM_TOL, assert_status_clean, gemm_rel_err, oracle_w4a4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    mxq.lib()
    yield
    assert_status_clean()


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy()


@pytest.mark.parametrize("M,N,K,rule", [(700, 520, 1280, mxq.MXQ_SCALE_OCP), (64, 392, 512, mxq.MXQ_SCALE_UOS)])
def test_static_scratch_matches_the_workspace_call_twice_in_a_row(M, N, K, rule):
    w = inputs.normal_bf16(N, K, 0.02, seed=N).cuda()
    wc, wsf = mxq.pack_weight(w)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(M)) * 0.3).to(torch.bfloat16).cuda()
    for seed in (M, M + 1):
        x = inputs.heavy_tailed_bf16(M, K, seed=seed)
        xd = x.cuda()
        a = mxq.linear_w4a4_ws(xd, wc, wsf, N, rule, 0.5, bias)
        b = mxq.linear_w4a4_static(xd, wc, wsf, N, rule, 0.5, bias)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_bits(b), _bits(a))
        rows = np.arange(M)
        assert gemm_rel_err(b, rows, oracle_w4a4(x, w.cpu(), rows, rule_a=rule, alpha=0.5, bias=bias.cpu())) <= GEMM_TOL


def test_static_scratch_rejects_oversize():
    M, K, N = 8192, 5120, 256  # 22 MB of quantised activations > 16 MiB
    assert mxq.mxq_linear_workspace_bytes(M, K) > 16 << 20
    x = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    wc = torch.zeros(N, K // 2, dtype=torch.uint8, device="cuda")
    wsf = torch.zeros(mxq.mxq_sf_bytes(N, K), dtype=torch.uint8, device="cuda")
    with pytest.raises(mxq.MxqError) as e:
        mxq.linear_w4a4_static(x, wc, wsf, N)
    assert e.value.status == 2  # MXQ_ERR_SHAPE
