"""CPU oracle for the MXFP4 quantized linear layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; the product package never imports it.

A thin ctypes + numpy wrapper around ``mxq_oracle.cpp`` (plain C++17, FP64 where
the definitions leave the precision open).  Every function here only marshals
arguments; the arithmetic, with its citations, lives in the C++ file.

Parity status per function (what pins each one is in ``tests/test_oracle_*.py``):
  e2m1_encode / e2m1_decode   pinned: OCP E2M1 value set, brute force, tie table
  block_exponent (OCP / UOS)  pinned: exact-rational brute force, Qmax = 7.25
  fwht128                     pinned: Sylvester matrix (scipy), H H^T = 128 I,
                              orthogonality; bit-level FP32 order is pinned only
                              by its own definition ("parity unpinned" at the
                              bit level with respect to the pages)
  e4m3_encode / e4m3_decode   pinned: brute force, OCP FP8 closed forms
  sf_swizzle                  pinned: round trip, atom-structure properties
  quantize_mxfp4 / _fp8       pinned: element-wise recomposition from the pinned codecs
  gemm                        pinned: exact-rational brute force on tiny shapes,
                              identities, error-quadrature property
  bf16_rne / qdq_* /          pinned: torch's FP32->BF16 conversion, tie cases,
  dequant_mxfp4_bf16          recomposition from the pinned codecs
  quantize_mxfp4_smooth       pinned: unit multiplier = plain quantiser, powers of two
                              shift only the scale, a worked rotation-then-multiplier case
  channel_absmax /            pinned: column maxima of the (rotated) rows; closed forms of
  smooth_factors              the migration factors at alpha = 0.5, 1 and 0
  sqnr_sums / sqnr_db         pinned: closed forms (uniform relative error, known pairs,
                              limits)
  select_precision            parity unpinned (tier order is a reading): the page names
                              the four tiers but not the order they are tried in; tested
                              at every threshold boundary
  attention_mxfp4             pinned: the textbook FP64 softmax of the dequantised
                              operands (P unquantised); PNQ and the conventional order
                              against an independent FP64 NumPy restatement (exact
                              exponentials, MX block maxima); equal-score and
                              dominant-key closed forms, PNQ weights summing to one
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxq_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libmxq_oracle.so")

RULE_OCP = 0
RULE_UOS = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (IEEE-exact flags: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-pthread", "-o", _LIB_PATH + ".tmp", _SRC]
        subprocess.run(cmd, check=True)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.oracle_e2m1_encode.argtypes = [ctypes.c_double]
    lib.oracle_e2m1_encode.restype = ctypes.c_uint8
    lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_block_exponent.argtypes = [ctypes.c_double, ctypes.c_int]
    lib.oracle_block_exponent.restype = ctypes.c_int
    lib.oracle_fwht128.argtypes = [P, P]
    lib.oracle_fwht128.restype = None
    lib.oracle_hadamard_scale.argtypes = []
    lib.oracle_hadamard_scale.restype = ctypes.c_float
    for name in ("oracle_sf_padded_rows", "oracle_sf_padded_cols"):
        getattr(lib, name).argtypes = [I64]
        getattr(lib, name).restype = I64
    lib.oracle_sf_bytes.argtypes = [I64, I64]
    lib.oracle_sf_bytes.restype = I64
    lib.oracle_sf_offset.argtypes = [I64, I64, I64]
    lib.oracle_sf_offset.restype = I64
    lib.oracle_sf_swizzle.argtypes = [P, I64, I64, P]
    lib.oracle_sf_swizzle.restype = None
    lib.oracle_sf_unswizzle.argtypes = [P, I64, I64, P]
    lib.oracle_sf_unswizzle.restype = None
    lib.oracle_quantize_mxfp4.argtypes = [P, I64, I64, I64, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int]
    lib.oracle_quantize_mxfp4.restype = None
    lib.oracle_rotate_rows.argtypes = [P, I64, I64, I64, ctypes.c_int, P]
    lib.oracle_rotate_rows.restype = None
    lib.oracle_quantize_fp8.argtypes = [P, I64, I64, I64, ctypes.c_float, P, ctypes.c_int]
    lib.oracle_quantize_fp8.restype = None
    lib.oracle_dequant_mxfp4.argtypes = [P, P, I64, I64, P]
    lib.oracle_dequant_mxfp4.restype = None
    lib.oracle_bf16_rne.argtypes = [ctypes.c_float]
    lib.oracle_bf16_rne.restype = ctypes.c_uint16
    lib.oracle_dequant_mxfp4_bf16.argtypes = [P, P, I64, I64, P]
    lib.oracle_dequant_mxfp4_bf16.restype = None
    lib.oracle_qdq_mxfp4.argtypes = [P, I64, I64, I64, ctypes.c_int, ctypes.c_int, P, ctypes.c_int]
    lib.oracle_qdq_mxfp4.restype = None
    lib.oracle_qdq_fp8.argtypes = [P, I64, I64, I64, ctypes.c_float, ctypes.c_float, P, ctypes.c_int]
    lib.oracle_qdq_fp8.restype = None
    lib.oracle_quantize_mxfp4_smooth.argtypes = [P, I64, I64, I64, ctypes.c_int, ctypes.c_int, P, P, P,
                                                 ctypes.c_int]
    lib.oracle_quantize_mxfp4_smooth.restype = None
    lib.oracle_channel_absmax.argtypes = [P, I64, I64, I64, ctypes.c_int, P]
    lib.oracle_channel_absmax.restype = None
    lib.oracle_smooth_factors.argtypes = [P, P, I64, ctypes.c_double, P, P]
    lib.oracle_smooth_factors.restype = None
    lib.oracle_sqnr_sums.argtypes = [P, P, I64, P]
    lib.oracle_sqnr_sums.restype = None
    lib.oracle_sqnr_db.argtypes = [ctypes.c_double, ctypes.c_double]
    lib.oracle_sqnr_db.restype = ctypes.c_double
    lib.oracle_select_precision.argtypes = [ctypes.c_double] * 4
    lib.oracle_select_precision.restype = ctypes.c_int
    lib.oracle_attention_mxfp4.argtypes = [P, P, P, I64, I64, I64, I64, I64, ctypes.c_int, ctypes.c_int, P, I64,
                                           P, P, ctypes.c_int]
    lib.oracle_attention_mxfp4.restype = None
    lib.oracle_gemm.argtypes = [ctypes.c_int, P, P, I64, P, P, I64, I64, ctypes.c_double, P, P, I64,
                                P, ctypes.c_int]
    lib.oracle_gemm.restype = None
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _threads(nthreads: int | None) -> int:
    return int(nthreads) if nthreads else (os.cpu_count() or 1)


def _bf16_bits(x) -> np.ndarray:
    """Accepts a uint16 array of BF16 bit patterns, or a torch bfloat16 CPU tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # only for the tensor -> bits view

    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


# ---------------------------------------------------------------- scalar codecs
def e2m1_encode(v: float) -> int:
    return int(_load().oracle_e2m1_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return float(_load().oracle_e2m1_decode(int(code)))


def e4m3_encode(v: float) -> int:
    return int(_load().oracle_e4m3_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return float(_load().oracle_e4m3_decode(int(code)))


def block_exponent(amax: float, rule: int) -> int:
    return int(_load().oracle_block_exponent(float(amax), int(rule)))


def hadamard_scale() -> float:
    return float(_load().oracle_hadamard_scale())


def fwht128(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.shape == (128,)
    y = np.empty(128, np.float32)
    _load().oracle_fwht128(_ptr(x), _ptr(y))
    return y


# ---------------------------------------------------------------- layouts
def sf_bytes(rows: int, K: int) -> int:
    return int(_load().oracle_sf_bytes(rows, K))


def sf_offset(r: int, c: int, K: int) -> int:
    return int(_load().oracle_sf_offset(r, c, K))


def sf_swizzle(logical: np.ndarray, rows: int, K: int) -> np.ndarray:
    logical = np.ascontiguousarray(logical, dtype=np.uint8)
    assert logical.size == rows * (K // 32)
    out = np.empty(sf_bytes(rows, K), np.uint8)
    _load().oracle_sf_swizzle(_ptr(logical), rows, K, _ptr(out))
    return out


def sf_unswizzle(physical: np.ndarray, rows: int, K: int) -> np.ndarray:
    physical = np.ascontiguousarray(physical, dtype=np.uint8)
    out = np.empty((rows, K // 32), np.uint8)
    _load().oracle_sf_unswizzle(_ptr(physical), rows, K, _ptr(out))
    return out


# ---------------------------------------------------------------- quantisers
def quantize_mxfp4(x, rule: int = RULE_OCP, hadamard: bool = False, nthreads: int | None = None):
    """x: [rows, K] BF16 (bits or tensor).  Returns (codes [rows, K/2] u8, sf_logical [rows, K/32] u8)."""
    xb = _bf16_bits(x)
    rows, K = xb.shape
    assert K % 32 == 0 and (not hadamard or K % 128 == 0)
    codes = np.zeros((rows, K // 2), np.uint8)
    sf = np.zeros((rows, K // 32), np.uint8)
    _load().oracle_quantize_mxfp4(_ptr(xb), rows, K, K, int(rule), int(bool(hadamard)), _ptr(codes),
                                  _ptr(sf), _threads(nthreads))
    return codes, sf


def rotate_rows(x, hadamard: bool = True) -> np.ndarray:
    xb = _bf16_bits(x)
    rows, K = xb.shape
    y = np.empty((rows, K), np.float32)
    _load().oracle_rotate_rows(_ptr(xb), rows, K, K, int(bool(hadamard)), _ptr(y))
    return y


def fp8_inv_scale(act_scale: float) -> float:
    """The reciprocal the FP8 quantiser multiplies by: fl32(1 / s)."""
    return float(np.float32(1.0) / np.float32(act_scale))


def quantize_fp8(x, act_scale: float, nthreads: int | None = None) -> np.ndarray:
    xb = _bf16_bits(x)
    rows, K = xb.shape
    q = np.empty((rows, K), np.uint8)
    _load().oracle_quantize_fp8(_ptr(xb), rows, K, K, ctypes.c_float(fp8_inv_scale(act_scale)), _ptr(q),
                                _threads(nthreads))
    return q


def dequant_mxfp4(codes: np.ndarray, sf_physical: np.ndarray, rows: int, K: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf_physical = np.ascontiguousarray(sf_physical, dtype=np.uint8)
    out = np.empty((rows, K), np.float64)
    _load().oracle_dequant_mxfp4(_ptr(codes), _ptr(sf_physical), rows, K, _ptr(out))
    return out


def gemm(a_codes: np.ndarray, a_sf: np.ndarray | None, b_codes: np.ndarray, b_sf: np.ndarray,
         M: int, N: int, K: int, alpha: float = 1.0, bias_bits: np.ndarray | None = None,
         rows: np.ndarray | None = None, a_fp8: bool = False, nthreads: int | None = None) -> np.ndarray:
    """FP64 y = alpha * deq(A) deq(B)^T + bias for the requested rows of A (all rows by default).

    a_codes: MXFP4 codes [M, K/2] with swizzled a_sf, or E4M3 codes [M, K] when a_fp8.
    b_codes/b_sf: MXFP4 weights [N, K/2] + swizzled scales.  bias_bits: N BF16 bit patterns.
    """
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((rows.size, N), np.float64)
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    b_codes = np.ascontiguousarray(b_codes, dtype=np.uint8)
    b_sf = np.ascontiguousarray(b_sf, dtype=np.uint8)
    a_sf = None if a_fp8 else np.ascontiguousarray(a_sf, dtype=np.uint8)
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
    _load().oracle_gemm(1 if a_fp8 else 0, _ptr(a_codes), _ptr(a_sf), M, _ptr(b_codes), _ptr(b_sf), N, K,
                        float(alpha), _ptr(bias_bits), _ptr(rows), rows.size, _ptr(y), _threads(nthreads))
    return y


# ---------------------------------------------------------------- QDQ emulation / dequantisation
def bf16_rne(v: float) -> int:
    return int(_load().oracle_bf16_rne(ctypes.c_float(v)))


def dequant_mxfp4_bf16(codes: np.ndarray, sf_physical: np.ndarray, rows: int, K: int) -> np.ndarray:
    """BF16 bit patterns [rows, K] of the dequantised MXFP4 values."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf_physical = np.ascontiguousarray(sf_physical, dtype=np.uint8)
    out = np.empty((rows, K), np.uint16)
    _load().oracle_dequant_mxfp4_bf16(_ptr(codes), _ptr(sf_physical), rows, K, _ptr(out))
    return out


def qdq_mxfp4(x, rule: int = RULE_OCP, hadamard: bool = False, nthreads: int | None = None) -> np.ndarray:
    xb = _bf16_bits(x)
    rows, K = xb.shape
    out = np.empty((rows, K), np.uint16)
    _load().oracle_qdq_mxfp4(_ptr(xb), rows, K, K, int(rule), int(bool(hadamard)), _ptr(out), _threads(nthreads))
    return out


def qdq_fp8(x, act_scale: float, nthreads: int | None = None) -> np.ndarray:
    xb = _bf16_bits(x)
    rows, K = xb.shape
    out = np.empty((rows, K), np.uint16)
    _load().oracle_qdq_fp8(_ptr(xb), rows, K, K, ctypes.c_float(fp8_inv_scale(act_scale)),
                           ctypes.c_float(np.float32(act_scale)), _ptr(out), _threads(nthreads))
    return out


# ---------------------------------------------------------------- SmoothQuant after the rotation
def quantize_mxfp4_smooth(x, chan_scale: np.ndarray, rule: int = RULE_OCP, hadamard: bool = False,
                          nthreads: int | None = None):
    """MXFP4 quantisation of (x R) * chan_scale (per channel, FP32).  Returns (codes, sf_logical)."""
    xb = _bf16_bits(x)
    rows, K = xb.shape
    c = np.ascontiguousarray(chan_scale, dtype=np.float32)
    assert c.shape == (K,) and K % 32 == 0 and (not hadamard or K % 128 == 0)
    codes = np.zeros((rows, K // 2), np.uint8)
    sf = np.zeros((rows, K // 32), np.uint8)
    _load().oracle_quantize_mxfp4_smooth(_ptr(xb), rows, K, K, int(rule), int(bool(hadamard)), _ptr(c),
                                         _ptr(codes), _ptr(sf), _threads(nthreads))
    return codes, sf


def channel_absmax(x, hadamard: bool = False) -> np.ndarray:
    """max over rows of |(x R)[r][k]| per channel k (FP32)."""
    xb = _bf16_bits(x)
    rows, K = xb.shape
    out = np.empty(K, np.float32)
    _load().oracle_channel_absmax(_ptr(xb), rows, K, K, int(bool(hadamard)), _ptr(out))
    return out


def smooth_factors(ax: np.ndarray, aw: np.ndarray, alpha: float = 0.5):
    """SmoothQuant migration factors (lambda, fl32(1/lambda)) from the channel maxima."""
    ax = np.ascontiguousarray(ax, dtype=np.float32)
    aw = np.ascontiguousarray(aw, dtype=np.float32)
    K = ax.size
    lam = np.empty(K, np.float32)
    inv = np.empty(K, np.float32)
    _load().oracle_smooth_factors(_ptr(ax), _ptr(aw), K, float(alpha), _ptr(lam), _ptr(inv))
    return lam, inv


# ---------------------------------------------------------------- precision selection
PREC_W4A4, PREC_W4A4_TRANSFORM, PREC_W4A8, PREC_BF16 = 0, 1, 2, 3


def sqnr_sums(y: np.ndarray, ref: np.ndarray):
    """(sum ref^2, sum (y - ref)^2) in FP64."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    ref = np.ascontiguousarray(ref, dtype=np.float64)
    assert y.shape == ref.shape
    out = np.empty(2, np.float64)
    _load().oracle_sqnr_sums(_ptr(y), _ptr(ref), y.size, _ptr(out))
    return float(out[0]), float(out[1])


def sqnr_db(signal: float, noise: float) -> float:
    return float(_load().oracle_sqnr_db(float(signal), float(noise)))


def select_precision(sqnr_plain_db: float, sqnr_transform_db: float, high_db: float, low_db: float) -> int:
    return int(_load().oracle_select_precision(float(sqnr_plain_db), float(sqnr_transform_db), float(high_db),
                                               float(low_db)))


# ---------------------------------------------------------------- MXFP4 attention (UOS + PNQ)
ATTN_PNQ, ATTN_NORMALISE_THEN_QUANTISE, ATTN_UNQUANTISED_P = 0, 1, 2


def attention_mxfp4(q, k, v, H: int, d: int, rows=None, rule: int = RULE_UOS, mode: int = ATTN_PNQ,
                    nthreads: int | None = None):
    """MXFP4 attention of query rows `rows` (default all) for every head.
    q [Sq][H*d], k, v [Skv][H*d] BF16.  Returns (out [len(rows)][H][d] FP64,
    weight sums [len(rows)][H])."""
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    Sq, Skv = qb.shape[0], kb.shape[0]
    assert qb.shape[1] == kb.shape[1] == vb.shape[1] == H * d and d % 32 == 0
    rows = np.arange(Sq, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, H, d), np.float64)
    ws = np.empty((rows.size, H), np.float64)
    _load().oracle_attention_mxfp4(_ptr(qb), _ptr(kb), _ptr(vb), Sq, Skv, H, d, H * d, int(rule), int(mode),
                                   _ptr(rows), rows.size, _ptr(out), _ptr(ws), _threads(nthreads))
    return out, ws
