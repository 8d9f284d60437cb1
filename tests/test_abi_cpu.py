"""Host-only checks of the C ABI: the library loads, exports exactly the entry points
include/mxq.h declares, and rejects bad arguments before touching any device.
No kernel is launched here."""

import ctypes
import os
import re

import pytest

import oracle
from mxfp4_block_scaled_mxq_b200 import build, mxq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return mxq.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mxq.h")).read()
    return sorted(set(re.findall(r"MXQ_API\s+[\w\s\*]+?\b(mxq_\w+)\s*\(", src)))


def test_header_declares_the_bound_entry_points():
    assert declared_functions() == sorted(mxq.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert isinstance(getattr(L, name), ctypes._CFuncPtr)


def test_status_strings(L):
    for code, name in mxq.STATUS_NAMES.items():
        assert mxq.mxq_status_string(code) == name
    assert mxq.mxq_status_string(99) == "MXQ_ERR_UNKNOWN"


@pytest.mark.parametrize("rows,K", [(1, 32), (128, 512), (130, 96), (32760, 5120), (32760, 13824), (3, 4064)])
def test_sf_bytes_matches_oracle_layout(L, rows, K):
    assert mxq.mxq_sf_bytes(rows, K) == oracle.sf_bytes(rows, K)


def test_sf_bytes_rejects_bad_sizes(L):
    assert mxq.mxq_sf_bytes(0, 32) == -1
    assert mxq.mxq_sf_bytes(4, 33) == -1
    assert mxq.mxq_sf_bytes(4, 0) == -1


def _status(fn, *args):
    return getattr(mxq.lib(), fn)(*args)


FAKE = 1 << 20  # a 16-byte-aligned non-null value; never dereferenced (validation fails first)


def test_quantize_validation_happens_before_any_launch(L):
    INV, SHAPE, ALIGN = 1, 2, 3
    q = lambda *a: L.mxq_quantize_act(*a)
    assert q(None, 4, 32, 32, 0, 0, 0, 1.0, FAKE, FAKE, None) == INV          # null x
    assert q(FAKE, 4, 32, 32, 0, 0, 0, 1.0, FAKE, None, None) == INV          # null sf for MXFP4
    assert q(FAKE, 4, 32, 32, 0, 7, 0, 1.0, FAKE, FAKE, None) == INV          # bad rule
    assert q(FAKE, 4, 32, 32, 9, 0, 0, 1.0, FAKE, FAKE, None) == INV          # bad format
    assert q(FAKE, 0, 32, 32, 0, 0, 0, 1.0, FAKE, FAKE, None) == SHAPE        # M = 0
    assert q(FAKE, 4, 48, 48, 0, 0, 0, 1.0, FAKE, FAKE, None) == SHAPE        # K % 32
    assert q(FAKE, 4, 96, 96, 0, 0, 1, 1.0, FAKE, FAKE, None) == SHAPE        # hadamard needs K % 128
    assert q(FAKE, 4, 64, 60, 0, 0, 0, 1.0, FAKE, FAKE, None) == ALIGN        # ldx < K
    assert q(FAKE + 2, 4, 64, 64, 0, 0, 0, 1.0, FAKE, FAKE, None) == ALIGN    # misaligned x
    assert q(FAKE + 8, 4, 64, 64, 0, 0, 0, 1.0, FAKE, FAKE, None) == ALIGN    # x needs 16 bytes
    assert q(FAKE, 4, 64, 68, 0, 0, 0, 1.0, FAKE, FAKE, None) == ALIGN        # ldx % 8
    # a 16-byte-aligned x with ldx % 16 == 8 passes validation (no device here: then fails)
    assert q(FAKE + 16, 4, 64, 72, 0, 0, 0, 1.0, FAKE, FAKE, None) not in (INV, SHAPE, ALIGN)
    assert q(FAKE, 4, 64, 64, 1, 0, 0, 1.0, FAKE, FAKE, None) == INV          # FP8 must not get sf
    assert q(FAKE, 4, 64, 64, 1, 0, 0, 0.0, FAKE, None, None) == INV          # FP8 scale <= 0
    assert q(FAKE, 4, 64, 64, 1, 0, 0, float("nan"), FAKE, None, None) == INV
    assert q(FAKE, 4, 64, 64, 1, 1, 0, 1.0, FAKE, None, None) == INV          # FP8 with UOS rule
    assert q(FAKE, 4, 64, 64, 1, 0, 1, 1.0, FAKE, None, None) == INV          # FP8 with hadamard


def test_gemm_validation_happens_before_any_launch(L):
    INV, SHAPE, ALIGN = 1, 2, 3
    g4 = lambda *a: L.mxq_gemm_w4a4(*a)
    ok = (FAKE, FAKE, FAKE, FAKE, 128, 256, 256, 1.0, None, FAKE, 256, None)
    args = list(ok)
    args[0] = None
    assert g4(*args) == INV
    args = list(ok); args[1] = None
    assert g4(*args) == INV
    args = list(ok); args[6] = 192
    assert g4(*args) == SHAPE                                                # K % 128
    args = list(ok); args[4] = 0
    assert g4(*args) == SHAPE
    args = list(ok); args[10] = 250
    assert g4(*args) == ALIGN                                                # ldd < N
    args = list(ok); args[9] = FAKE + 8
    assert g4(*args) == ALIGN
    args = list(ok); args[7] = float("inf")
    assert g4(*args) == INV
    g8 = lambda *a: L.mxq_gemm_w4a8(*a)
    assert g8(FAKE, 0.0, FAKE, FAKE, 128, 256, 256, None, FAKE, 256, None) == INV
    assert g8(FAKE, 1.0, FAKE + 16, FAKE, 128, 256, 256, None, FAKE, 256, None) == ALIGN  # B needs 32 B


def test_dequant_and_qdq_validation_happens_before_any_launch(L):
    INV, SHAPE, ALIGN = 1, 2, 3
    dq = lambda *a: L.mxq_dequant_mxfp4(*a)
    assert dq(None, FAKE, 4, 64, FAKE, 64, None) == INV
    assert dq(FAKE, None, 4, 64, FAKE, 64, None) == INV
    assert dq(FAKE, FAKE, 0, 64, FAKE, 64, None) == SHAPE
    assert dq(FAKE, FAKE, 4, 48, FAKE, 48, None) == SHAPE                    # K % 32
    assert dq(FAKE, FAKE, 4, 64, FAKE, 60, None) == ALIGN                    # ldo < K
    assert dq(FAKE, FAKE, 4, 64, FAKE, 68, None) == ALIGN                    # ldo % 8
    assert dq(FAKE + 8, FAKE, 4, 64, FAKE, 64, None) == ALIGN                # codes 16-byte aligned
    assert dq(FAKE, FAKE, 4, 64, FAKE + 8, 64, None) == ALIGN
    qq = lambda *a: L.mxq_qdq_act(*a)
    assert qq(None, 4, 64, 64, 0, 0, 0, 1.0, FAKE, 64, None) == INV
    assert qq(FAKE, 4, 64, 64, 0, 0, 0, 1.0, None, 64, None) == INV
    assert qq(FAKE, 4, 64, 64, 5, 0, 0, 1.0, FAKE, 64, None) == INV          # bad format
    assert qq(FAKE, 4, 64, 64, 0, 3, 0, 1.0, FAKE, 64, None) == INV          # bad rule
    assert qq(FAKE, 4, 64, 64, 1, 0, 0, -1.0, FAKE, 64, None) == INV         # FP8 scale <= 0
    assert qq(FAKE, 4, 64, 64, 1, 1, 0, 1.0, FAKE, 64, None) == INV          # FP8 with UOS
    assert qq(FAKE, 4, 64, 64, 1, 0, 1, 1.0, FAKE, 64, None) == INV          # FP8 with hadamard
    assert qq(FAKE, 4, 96, 96, 0, 0, 1, 1.0, FAKE, 96, None) == SHAPE        # hadamard needs K % 128
    assert qq(FAKE, 0, 64, 64, 0, 0, 0, 1.0, FAKE, 64, None) == SHAPE
    assert qq(FAKE + 8, 4, 64, 64, 0, 0, 0, 1.0, FAKE, 64, None) == ALIGN    # x needs 16 bytes
    assert qq(FAKE, 4, 64, 68, 0, 0, 0, 1.0, FAKE, 64, None) == ALIGN        # ldx % 8
    assert qq(FAKE, 4, 64, 64, 0, 0, 0, 1.0, FAKE + 8, 64, None) == ALIGN    # out needs 16 bytes
    assert qq(FAKE, 4, 64, 64, 0, 0, 0, 1.0, FAKE, 68, None) == ALIGN        # ldo % 8


def test_smoothing_validation_happens_before_any_launch(L):
    INV, SHAPE, ALIGN = 1, 2, 3
    ca = lambda *a: L.mxq_channel_absmax(*a)
    assert ca(FAKE, 4, 64, 64, 0, 0, None, None) == INV                      # null output
    assert ca(None, 4, 64, 64, 0, 0, FAKE, None) == INV
    assert ca(FAKE, 4, 96, 96, 1, 0, FAKE, None) == SHAPE                    # hadamard needs K % 128
    assert ca(FAKE, 4, 64, 64, 0, 0, FAKE + 4, None) == ALIGN
    sf = lambda *a: L.mxq_smooth_factors(*a)
    assert sf(FAKE, FAKE, 64, 1.5, FAKE, FAKE, None) == INV                  # alpha outside [0, 1]
    assert sf(FAKE, FAKE, 64, float("nan"), FAKE, FAKE, None) == INV
    assert sf(FAKE, None, 64, 0.5, FAKE, FAKE, None) == INV
    assert sf(FAKE, FAKE, 0, 0.5, FAKE, FAKE, None) == SHAPE
    qs = lambda *a: L.mxq_quantize_smooth(*a)
    assert qs(FAKE, 4, 64, 64, 0, 0, None, FAKE, FAKE, None) == INV          # null factors
    assert qs(FAKE, 4, 64, 64, 0, 0, FAKE + 8, FAKE, FAKE, None) == ALIGN    # factors 16-byte aligned
    assert qs(FAKE, 4, 64, 64, 2, 0, FAKE, FAKE, FAKE, None) == INV          # bad rule
    assert qs(FAKE, 4, 48, 48, 0, 0, FAKE, FAKE, FAKE, None) == SHAPE


def test_host_side_precision_selection_matches_the_oracle(L):
    """The tier decision and the dB conversion are host-only C functions: compared with
    the oracle's on a grid around both thresholds and on random values."""
    import math
    import random
    vals = [-math.inf, 0.0, 9.99, 10.0, 10.01, 14.99, 15.0, 15.01, 30.0, math.inf]
    rng = random.Random(3)
    pairs = [(a, b) for a in vals for b in vals] + [(rng.uniform(0, 30), rng.uniform(0, 30)) for _ in range(200)]
    for a, b in pairs:
        assert mxq.mxq_select_precision(a, b, 15.0, 10.0) == oracle.select_precision(a, b, 15.0, 10.0), (a, b)
    for s, n in [(26.0, 5.0), (1.0, 0.0), (0.0, 1.0), (3.5e7, 2.25e-3)]:
        assert mxq.mxq_sqnr_db(s, n) == oracle.sqnr_db(s, n)


def test_sqnr_validation_happens_before_any_launch(L):
    INV, SHAPE, ALIGN = 1, 2, 3
    sq = lambda *a: L.mxq_sqnr_accumulate(*a)
    assert sq(None, 8, FAKE, 8, 4, 8, 0, FAKE, None) == INV
    assert sq(FAKE, 8, FAKE, 8, 4, 8, 0, None, None) == INV
    assert sq(FAKE, 8, FAKE, 8, 0, 8, 0, FAKE, None) == SHAPE
    assert sq(FAKE, 4, FAKE, 8, 4, 8, 0, FAKE, None) == ALIGN                # ldy < N
    assert sq(FAKE, 12, FAKE, 16, 4, 8, 0, FAKE, None) == ALIGN              # ldy % 8
    assert sq(FAKE + 8, 8, FAKE, 8, 4, 8, 0, FAKE, None) == ALIGN


def test_attention_validation_happens_before_any_launch(L):
    INV, SHAPE, ALIGN, UNSUP = 1, 2, 3, 4
    assert L.mxq_attn_padded_keys(1) == 256 and L.mxq_attn_padded_keys(512) == 512
    assert L.mxq_attn_padded_keys(0) == -1
    vt = lambda *a: L.mxq_quantize_vt(*a)
    assert vt(None, 10, 128, 128, 1, FAKE, FAKE, None) == INV
    assert vt(FAKE, 10, 128, 128, 5, FAKE, FAKE, None) == INV
    assert vt(FAKE, 0, 128, 128, 1, FAKE, FAKE, None) == SHAPE
    assert vt(FAKE, 10, 96, 96, 1, FAKE, FAKE, None) == SHAPE                # HD % 128
    assert vt(FAKE, 10, 128, 120, 1, FAKE, FAKE, None) == ALIGN              # ldv < HD
    assert vt(FAKE + 8, 10, 128, 128, 1, FAKE, FAKE, None) == ALIGN          # v 16-byte aligned
    assert vt(FAKE, 10, 128, 132, 1, FAKE, FAKE, None) == ALIGN              # ldv % 8
    at = lambda *a: L.mxq_attention_mxfp4(*a)
    ok = [FAKE] * 6 + [100, 100, 2, 128, 1, FAKE, 256, None]
    a = list(ok); a[0] = None
    assert at(*a) == INV
    a = list(ok); a[9] = 64
    assert at(*a) == UNSUP                                                  # d != 128
    a = list(ok); a[6] = 0
    assert at(*a) == SHAPE
    a = list(ok); a[12] = 200
    assert at(*a) == ALIGN                                                  # ldo < H d
    a = list(ok); a[11] = FAKE + 8
    assert at(*a) == ALIGN


def test_static_scratch_rejects_oversize_before_any_launch(L):
    SHAPE = 2
    assert L.mxq_linear_w4a4_static(FAKE, 8192, 5120, 5120, 0, FAKE, FAKE, 256, 1.0, None, FAKE, 256, None) == SHAPE
    assert L.mxq_linear_w4a4_static(FAKE, 10, 100, 128, 0, FAKE, FAKE, 256, 1.0, None, FAKE, 256, None) == SHAPE


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        mxq.quantize_act(torch.zeros(4, 32, dtype=torch.bfloat16))


def test_selftest_without_a_b200_launches_nothing(L):
    """Off a B200 (here: no GPU at all) the diagnostic launches nothing and reports why."""
    UNSUPPORTED, CUDA = 4, 5
    assert L.mxq_selftest_wait_timeout(None) in (UNSUPPORTED, CUDA)


class _FakeCudaTensor:
    """Just enough of a tensor for the binding's argument checks (no device needed)."""
    dtype = None
    is_cuda = True

    def __init__(self, index):
        import torch
        self.dtype = torch.bfloat16
        self.device = torch.device("cuda", index)

    def dim(self):
        return 2

    def stride(self, i):
        return 1 if i == 1 else 64


def test_binding_refuses_a_tensor_on_another_device(monkeypatch):
    """The helpers launch on the current device: an input on another device is an error,
    not a silent read through the wrong context."""
    import torch
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    mxq._bf16_2d(_FakeCudaTensor(0), "x")
    with pytest.raises(ValueError, match="current CUDA device"):
        mxq._bf16_2d(_FakeCudaTensor(1), "x")
