"""The bounded-wait failure path on the GPU, exercised without a fault: a kernel whose
wait nothing completes gives up after about a second, records MXQ_ERR_TIMEOUT in the
library's status word and returns; the host reads (and clears) it with
mxq_debug_poll, and the device keeps working."""

import time

import numpy as np
import pytest
import torch

from mxfp4_block_scaled_mxq_b200 import build, inputs, mxq
from parity import GEMM_TOL, gemm_rel_err, oracle_w4a4

pytestmark = pytest.mark.gpu

MXQ_ERR_TIMEOUT = 6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    mxq.lib()


def test_a_wait_nothing_completes_gives_up_reports_and_leaves_the_device_usable():
    assert mxq.mxq_debug_poll() == 0
    t0 = time.perf_counter()
    mxq.mxq_selftest_wait_timeout()
    status = mxq.mxq_debug_poll()  # synchronises the device
    elapsed = time.perf_counter() - t0
    assert status == MXQ_ERR_TIMEOUT
    assert 0.1 < elapsed < 30.0, elapsed  # the wait's limit is about a second of SM clocks
    assert mxq.mxq_debug_poll() == 0  # read once, then cleared

    # afterwards the library's kernels run and agree with the oracle as before
    x, w = inputs.tiny(seed=0)
    M, K = x.shape
    N = w.shape[0]
    wc, wsf = mxq.pack_weight(w.cuda())
    q, sf = mxq.quantize_act(x.cuda())
    d = mxq.gemm_w4a4(q, sf, wc, wsf, M, N, K)
    torch.cuda.synchronize()
    rows = np.arange(M)
    assert gemm_rel_err(d, rows, oracle_w4a4(x, w, rows)) <= GEMM_TOL
    assert mxq.mxq_debug_poll() == 0
