"""The library on the caller's streams: every call is asynchronous on the stream it is
given, so results must not depend on which stream runs them, on work running beside them
on another stream, or on being captured into a CUDA graph and replayed.  The kernels are
deterministic (fixed accumulation order), so each result is compared bit for bit with the
same call on the default stream, and that one with the oracle's layer (GEMM tolerance)."""

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


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy()


def _layer(M, N, K, seed):
    x = inputs.heavy_tailed_bf16(M, K, seed=seed)
    w = inputs.normal_bf16(N, K, 0.02, seed=seed + 1)
    wc, wsf = mxq.pack_weight(w.cuda())
    return x, w, wc, wsf


def test_side_stream_with_pinned_host_copies():
    """Copy-in from pinned host memory, quantise + GEMM and copy-out, all on a side stream
    ordered only by the stream itself: the host copy of D equals the default-stream D."""
    M, N, K = 300, 520, 1280
    x, w, wc, wsf = _layer(M, N, K, 71)
    want = mxq.linear_w4a4(x.cuda(), wc, wsf, N)
    torch.cuda.synchronize()
    rows = np.arange(M)
    assert gemm_rel_err(want, rows, oracle_w4a4(x, w, rows)) <= GEMM_TOL

    s = torch.cuda.Stream()
    x_host = x.pin_memory()
    d_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    with torch.cuda.stream(s):
        xd = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
        xd.copy_(x_host, non_blocking=True)
        d = mxq.linear_w4a4(xd, wc, wsf, N, stream=s)
        d_host.copy_(d, non_blocking=True)
    s.synchronize()
    np.testing.assert_array_equal(_bits(d_host), _bits(want))


def test_two_streams_at_once():
    """Two layers of different shapes issued alternately on two streams (each a quantiser
    followed by a dependent GEMM launch), so that their kernels can overlap: each result
    equals its default-stream result."""
    shapes = [(257, 392, 640), (1000, 264, 384)]
    layers = [_layer(M, N, K, 80 + i) for i, (M, N, K) in enumerate(shapes)]
    wants = []
    for (x, _, wc, wsf), (M, N, K) in zip(layers, shapes):
        wants.append(mxq.linear_w4a4(x.cuda(), wc, wsf, N))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    xs = [x.cuda() for x, *_ in layers]
    torch.cuda.synchronize()
    outs = [[], []]
    for _ in range(3):
        for i, ((_, _, wc, wsf), (M, N, K)) in enumerate(zip(layers, shapes)):
            with torch.cuda.stream(streams[i]):
                outs[i].append(mxq.linear_w4a4(xs[i], wc, wsf, N, stream=streams[i]))
    torch.cuda.synchronize()
    for i in range(2):
        for d in outs[i]:
            np.testing.assert_array_equal(_bits(d), _bits(wants[i]))


@pytest.mark.parametrize("M", [48, 300])  # the few-token kernel and the CTA-pair kernel
def test_cuda_graph_replay_matches_eager(M):
    """Quantiser + GEMM captured once into a CUDA graph (the library's host work -- checks,
    tensor maps -- runs at capture), replayed on fresh input data copied into the captured
    input buffer: every replay equals the eager call on the same data."""
    N, K = 520, 1280
    _, _, wc, wsf = _layer(M, N, K, 90)
    xs = [inputs.heavy_tailed_bf16(M, K, seed=91 + i).cuda() for i in range(3)]
    wants = [mxq.linear_w4a4(x, wc, wsf, N) for x in xs]
    torch.cuda.synchronize()

    x_in = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(mxq.mxq_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
    d = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    x_in.copy_(xs[0])
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        mxq.quantize_act(x_in, out=(q, sf))
        mxq.gemm_w4a4(q, sf, wc, wsf, M, N, K, out=d)
    for x, want in zip(xs, wants):
        x_in.copy_(x)
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_bits(d), _bits(want))
    del g


@pytest.mark.parametrize("as_handle", [False, True])
def test_helpers_given_a_stream_from_another_stream(as_handle):
    """The allocating helpers called with `stream=` while torch's current stream is the
    default one (a torch stream or a raw cudaStream_t handle): their temporaries (the
    quantised activations) are allocated on that stream, and D equals the default-stream D."""
    M, N, K = 300, 520, 1280
    x, _, wc, wsf = _layer(M, N, K, 95)
    xd = x.cuda()
    want = mxq.linear_w4a4(xd, wc, wsf, N)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    outs = [mxq.linear_w4a4(xd, wc, wsf, N, stream=s.cuda_stream if as_handle else s) for _ in range(4)]
    s.synchronize()
    for d in outs:
        np.testing.assert_array_equal(_bits(d), _bits(want))
