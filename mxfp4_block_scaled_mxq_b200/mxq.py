"""Thin Python binding of libmxq (the C ABI in include/mxq.h).

Argument marshalling only: every step of the quantized linear layer runs in the
library's sm_100a kernels.  Functions named ``mxq_*`` mirror the C entry points one
for one (device buffers may be given as torch CUDA tensors or raw integer device
pointers); the lower-case helpers below them allocate the output tensors and call
the ``mxq_*`` functions.  There is no fallback: if the shared library is missing or
the device is not an sm_100 GPU, calls raise.
"""

from __future__ import annotations

import ctypes
import functools
import inspect
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmxq.so")

MXQ_OK = 0
STATUS_NAMES = {0: "MXQ_OK", 1: "MXQ_ERR_INVALID_ARG", 2: "MXQ_ERR_SHAPE", 3: "MXQ_ERR_ALIGN",
                4: "MXQ_ERR_UNSUPPORTED", 5: "MXQ_ERR_CUDA", 6: "MXQ_ERR_TIMEOUT"}
MXQ_SCALE_OCP, MXQ_SCALE_UOS = 0, 1
MXQ_ACT_MXFP4, MXQ_ACT_FP8_E4M3 = 0, 1
MXQ_PREC_W4A4, MXQ_PREC_W4A4_TRANSFORM, MXQ_PREC_W4A8, MXQ_PREC_BF16 = 0, 1, 2, 3

EXPORTED = ("mxq_status_string", "mxq_sf_bytes", "mxq_quantize_act", "mxq_pack_weight", "mxq_gemm_w4a4",
            "mxq_gemm_w4a8", "mxq_dequant_mxfp4", "mxq_qdq_act", "mxq_channel_absmax", "mxq_smooth_factors",
            "mxq_quantize_smooth", "mxq_sqnr_accumulate", "mxq_sqnr_db", "mxq_select_precision", "mxq_attn_padded_keys",
            "mxq_attn_code_poly", "mxq_quantize_vt",
            "mxq_attention_mxfp4", "mxq_linear_workspace_bytes", "mxq_linear_w4a4", "mxq_linear_w4a4_static",
            "mxq_debug_poll", "mxq_selftest_wait_timeout")


class MxqError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libmxq.so from the package directory (built by ``build.py``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libmxq.so not built ({_LIB_PATH}); run `python -m mxfp4_block_scaled_mxq_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    P, I64, I32, F32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    L.mxq_status_string.argtypes = [I32]
    L.mxq_status_string.restype = ctypes.c_char_p
    L.mxq_sf_bytes.argtypes = [I64, I64]
    L.mxq_sf_bytes.restype = I64
    L.mxq_quantize_act.argtypes = [P, I64, I64, I64, I32, I32, I32, F32, P, P, P]
    L.mxq_quantize_act.restype = I32
    L.mxq_pack_weight.argtypes = [P, I64, I64, I64, I32, I32, P, P, P]
    L.mxq_pack_weight.restype = I32
    L.mxq_gemm_w4a4.argtypes = [P, P, P, P, I64, I64, I64, F32, P, P, I64, P]
    L.mxq_gemm_w4a4.restype = I32
    L.mxq_gemm_w4a8.argtypes = [P, F32, P, P, I64, I64, I64, P, P, I64, P]
    L.mxq_gemm_w4a8.restype = I32
    L.mxq_dequant_mxfp4.argtypes = [P, P, I64, I64, P, I64, P]
    L.mxq_dequant_mxfp4.restype = I32
    L.mxq_qdq_act.argtypes = [P, I64, I64, I64, I32, I32, I32, F32, P, I64, P]
    L.mxq_qdq_act.restype = I32
    L.mxq_channel_absmax.argtypes = [P, I64, I64, I64, I32, I32, P, P]
    L.mxq_channel_absmax.restype = I32
    L.mxq_smooth_factors.argtypes = [P, P, I64, F32, P, P, P]
    L.mxq_smooth_factors.restype = I32
    L.mxq_quantize_smooth.argtypes = [P, I64, I64, I64, I32, I32, P, P, P, P]
    L.mxq_quantize_smooth.restype = I32
    L.mxq_sqnr_accumulate.argtypes = [P, I64, P, I64, I64, I64, I32, P, P]
    L.mxq_sqnr_accumulate.restype = I32
    L.mxq_sqnr_db.argtypes = [ctypes.c_double, ctypes.c_double]
    L.mxq_sqnr_db.restype = ctypes.c_double
    L.mxq_select_precision.argtypes = [ctypes.c_double] * 4
    L.mxq_select_precision.restype = I32
    L.mxq_attn_padded_keys.argtypes = [I64]
    L.mxq_attn_padded_keys.restype = I64
    L.mxq_quantize_vt.argtypes = [P, I64, I64, I64, I32, P, P, P]
    L.mxq_quantize_vt.restype = I32
    L.mxq_attn_code_poly.argtypes = [P]
    L.mxq_attn_code_poly.restype = None
    L.mxq_attention_mxfp4.argtypes = [P, P, P, P, P, P, I64, I64, I64, I64, I32, P, I64, P]
    L.mxq_attention_mxfp4.restype = I32
    L.mxq_linear_workspace_bytes.argtypes = [I64, I64]
    L.mxq_linear_workspace_bytes.restype = I64
    L.mxq_linear_w4a4.argtypes = [P, I64, I64, I64, I32, P, P, I64, F32, P, P, I64, P, I64, P]
    L.mxq_linear_w4a4.restype = I32
    L.mxq_linear_w4a4_static.argtypes = [P, I64, I64, I64, I32, P, P, I64, F32, P, P, I64, P]
    L.mxq_linear_w4a4_static.restype = I32
    L.mxq_debug_poll.argtypes = []
    L.mxq_debug_poll.restype = I32
    L.mxq_selftest_wait_timeout.argtypes = [P]
    L.mxq_selftest_wait_timeout.restype = I32
    _lib = L
    return L


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libmxq takes device buffers: got a CPU tensor")
    if not t.is_contiguous():
        raise ValueError("libmxq buffers must be contiguous (use the leading-dimension argument for strides)")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != MXQ_OK:
        raise MxqError(status, where)


# ------------------------------------------------------------------ C entry points
def mxq_status_string(status: int) -> str:
    return lib().mxq_status_string(int(status)).decode()


def mxq_sf_bytes(rows: int, K: int) -> int:
    return int(lib().mxq_sf_bytes(int(rows), int(K)))


def mxq_quantize_act(x, M, K, ldx, fmt, rule, hadamard128, act_scale, q_out, sf_out, stream=None) -> None:
    _check(lib().mxq_quantize_act(_ptr(x), int(M), int(K), int(ldx), int(fmt), int(rule), int(bool(hadamard128)),
                                  float(act_scale), _ptr(q_out), _ptr(sf_out), _stream(stream)), "mxq_quantize_act")


def mxq_pack_weight(w, N, K, ldw, rule, hadamard128, codes_out, sf_out, stream=None) -> None:
    _check(lib().mxq_pack_weight(_ptr(w), int(N), int(K), int(ldw), int(rule), int(bool(hadamard128)),
                                 _ptr(codes_out), _ptr(sf_out), _stream(stream)), "mxq_pack_weight")


def mxq_gemm_w4a4(a_codes, a_sf, b_codes, b_sf, M, N, K, alpha, bias, d, ldd, stream=None) -> None:
    _check(lib().mxq_gemm_w4a4(_ptr(a_codes), _ptr(a_sf), _ptr(b_codes), _ptr(b_sf), int(M), int(N), int(K),
                               float(alpha), _ptr(bias), _ptr(d), int(ldd), _stream(stream)), "mxq_gemm_w4a4")


def mxq_gemm_w4a8(a_e4m3, act_scale, b_codes, b_sf, M, N, K, bias, d, ldd, stream=None) -> None:
    _check(lib().mxq_gemm_w4a8(_ptr(a_e4m3), float(act_scale), _ptr(b_codes), _ptr(b_sf), int(M), int(N), int(K),
                               _ptr(bias), _ptr(d), int(ldd), _stream(stream)), "mxq_gemm_w4a8")


def mxq_dequant_mxfp4(codes, sf, rows, K, out, ldo, stream=None) -> None:
    _check(lib().mxq_dequant_mxfp4(_ptr(codes), _ptr(sf), int(rows), int(K), _ptr(out), int(ldo), _stream(stream)),
           "mxq_dequant_mxfp4")


def mxq_qdq_act(x, M, K, ldx, fmt, rule, hadamard128, act_scale, out, ldo, stream=None) -> None:
    _check(lib().mxq_qdq_act(_ptr(x), int(M), int(K), int(ldx), int(fmt), int(rule), int(bool(hadamard128)),
                             float(act_scale), _ptr(out), int(ldo), _stream(stream)), "mxq_qdq_act")


def mxq_channel_absmax(x, rows, K, ldx, hadamard128, accumulate, amax_out, stream=None) -> None:
    _check(lib().mxq_channel_absmax(_ptr(x), int(rows), int(K), int(ldx), int(bool(hadamard128)),
                                    int(bool(accumulate)), _ptr(amax_out), _stream(stream)), "mxq_channel_absmax")


def mxq_smooth_factors(amax_x, amax_w, K, alpha, lambda_out, inv_lambda_out, stream=None) -> None:
    _check(lib().mxq_smooth_factors(_ptr(amax_x), _ptr(amax_w), int(K), float(alpha), _ptr(lambda_out),
                                    _ptr(inv_lambda_out), _stream(stream)), "mxq_smooth_factors")


def mxq_quantize_smooth(x, rows, K, ldx, rule, hadamard128, chan_scale, codes_out, sf_out, stream=None) -> None:
    _check(lib().mxq_quantize_smooth(_ptr(x), int(rows), int(K), int(ldx), int(rule), int(bool(hadamard128)),
                                     _ptr(chan_scale), _ptr(codes_out), _ptr(sf_out), _stream(stream)),
           "mxq_quantize_smooth")


def mxq_sqnr_accumulate(y, ldy, ref, ldr, M, N, accumulate, acc, stream=None) -> None:
    _check(lib().mxq_sqnr_accumulate(_ptr(y), int(ldy), _ptr(ref), int(ldr), int(M), int(N), int(bool(accumulate)),
                                     _ptr(acc), _stream(stream)), "mxq_sqnr_accumulate")


def mxq_sqnr_db(signal: float, noise: float) -> float:
    return float(lib().mxq_sqnr_db(float(signal), float(noise)))


def mxq_select_precision(sqnr_plain_db: float, sqnr_transform_db: float, high_db: float, low_db: float) -> int:
    return int(lib().mxq_select_precision(float(sqnr_plain_db), float(sqnr_transform_db), float(high_db),
                                          float(low_db)))


def mxq_attn_padded_keys(S_kv: int) -> int:
    return int(lib().mxq_attn_padded_keys(int(S_kv)))


def mxq_attn_code_poly() -> list[float]:
    """{1, a1, a2, a3}: the FP32 cubic the attention kernel decides the numerators' codes with."""
    c = (ctypes.c_float * 4)()
    lib().mxq_attn_code_poly(c)
    return [float(x) for x in c]


def mxq_quantize_vt(v, S, HD, ldv, rule, codes_out, sf_out, stream=None) -> None:
    _check(lib().mxq_quantize_vt(_ptr(v), int(S), int(HD), int(ldv), int(rule), _ptr(codes_out), _ptr(sf_out),
                                 _stream(stream)), "mxq_quantize_vt")


def mxq_attention_mxfp4(q_codes, q_sf, k_codes, k_sf, vt_codes, vt_sf, S_q, S_kv, H, d, rule, out, ldo,
                        stream=None) -> None:
    _check(lib().mxq_attention_mxfp4(_ptr(q_codes), _ptr(q_sf), _ptr(k_codes), _ptr(k_sf), _ptr(vt_codes),
                                     _ptr(vt_sf), int(S_q), int(S_kv), int(H), int(d), int(rule), _ptr(out),
                                     int(ldo), _stream(stream)), "mxq_attention_mxfp4")


def mxq_linear_workspace_bytes(M: int, K: int) -> int:
    return int(lib().mxq_linear_workspace_bytes(int(M), int(K)))


def mxq_linear_w4a4(x, M, K, ldx, rule, w_codes, w_sf, N, alpha, bias, workspace, workspace_bytes, d, ldd,
                    stream=None) -> None:
    _check(lib().mxq_linear_w4a4(_ptr(x), int(M), int(K), int(ldx), int(rule), _ptr(w_codes), _ptr(w_sf), int(N),
                                 float(alpha), _ptr(bias), _ptr(workspace), int(workspace_bytes), _ptr(d), int(ldd),
                                 _stream(stream)), "mxq_linear_w4a4")


def mxq_linear_w4a4_static(x, M, K, ldx, rule, w_codes, w_sf, N, alpha, bias, d, ldd, stream=None) -> None:
    _check(lib().mxq_linear_w4a4_static(_ptr(x), int(M), int(K), int(ldx), int(rule), _ptr(w_codes), _ptr(w_sf),
                                        int(N), float(alpha), _ptr(bias), _ptr(d), int(ldd), _stream(stream)),
           "mxq_linear_w4a4_static")


def mxq_debug_poll() -> int:
    return int(lib().mxq_debug_poll())


def mxq_selftest_wait_timeout(stream=None) -> None:
    _check(lib().mxq_selftest_wait_timeout(_stream(stream)), "mxq_selftest_wait_timeout")


# ------------------------------------------------------------------ allocating helpers
def _on_stream(fn):
    """Runs an allocating helper with its `stream` argument as torch's current stream.

    The caching allocator hands a freed block out again only after the work queued on the
    stream that allocated it, so tensors the helper allocates (outputs and temporaries such
    as the quantised activations of linear_w4a4) then stay valid for as long as the kernels
    the helper queued on `stream` read or write them, whatever stream the caller is on."""
    sig = inspect.signature(fn)

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        stream = kwargs["stream"] if "stream" in kwargs else sig.bind(*args, **kwargs).arguments.get("stream")
        if stream is None:
            return fn(*args, **kwargs)
        s = torch.cuda.ExternalStream(stream) if isinstance(stream, int) else stream
        with torch.cuda.stream(s):
            return fn(*args, **kwargs)

    return wrapper


def _bf16_2d(x: torch.Tensor, name: str) -> torch.Tensor:
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError(f"{name}: expected a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError(f"{name}: rows must be contiguous")
    _on_current_device(x, name)
    return x


def _on_current_device(x: torch.Tensor, name: str) -> None:
    """The library launches on the current CUDA device; a tensor on another device would
    be read through the wrong context, so it is refused here."""
    cur = torch.cuda.current_device()
    if x.device.index is not None and x.device.index != cur:
        raise ValueError(f"{name}: tensor on {x.device} but the current CUDA device is cuda:{cur} "
                         f"(run the call under torch.cuda.device({x.device.index}))")


@_on_stream
def quantize_act(x: torch.Tensor, rule: int = MXQ_SCALE_OCP, hadamard128: bool = False, out=None, stream=None):
    """Dynamic MXFP4 quantisation of X[M][K] -> (codes [M][K/2] uint8, sf uint8[mxq_sf_bytes(M, K)])."""
    x = _bf16_2d(x, "x")
    M, K = x.shape
    if out is None:
        out = (torch.empty(M, K // 2, dtype=torch.uint8, device=x.device),
               torch.empty(mxq_sf_bytes(M, K), dtype=torch.uint8, device=x.device))
    q, sf = out
    mxq_quantize_act(x.data_ptr(), M, K, x.stride(0), MXQ_ACT_MXFP4, rule, hadamard128, 1.0, q, sf, stream)
    return q, sf


@_on_stream
def quantize_act_fp8(x: torch.Tensor, act_scale: float, out=None, stream=None) -> torch.Tensor:
    """Static FP8 E4M3 quantisation of X[M][K] with per-tensor scale s -> uint8 [M][K]."""
    x = _bf16_2d(x, "x")
    M, K = x.shape
    q = torch.empty(M, K, dtype=torch.uint8, device=x.device) if out is None else out
    mxq_quantize_act(x.data_ptr(), M, K, x.stride(0), MXQ_ACT_FP8_E4M3, MXQ_SCALE_OCP, False, act_scale, q, None,
                     stream)
    return q


@_on_stream
def pack_weight(w: torch.Tensor, rule: int = MXQ_SCALE_OCP, hadamard128: bool = False, stream=None):
    """Offline MXFP4 packing of W[N][K] -> (codes [N][K/2] uint8, sf uint8[mxq_sf_bytes(N, K)])."""
    w = _bf16_2d(w, "w")
    N, K = w.shape
    codes = torch.empty(N, K // 2, dtype=torch.uint8, device=w.device)
    sf = torch.empty(mxq_sf_bytes(N, K), dtype=torch.uint8, device=w.device)
    mxq_pack_weight(w.data_ptr(), N, K, w.stride(0), rule, hadamard128, codes, sf, stream)
    return codes, sf


def _out_bf16(M: int, N: int, device) -> torch.Tensor:
    """[M][N] BF16 view of a buffer whose rows are padded to a multiple of 8 elements
    (the output's row stride must be a multiple of 16 bytes)."""
    ldd = (N + 7) // 8 * 8
    return torch.empty(M, ldd, dtype=torch.bfloat16, device=device)[:, :N]


@_on_stream
def gemm_w4a4(a_codes, a_sf, b_codes, b_sf, M, N, K, alpha=1.0, bias=None, out=None, stream=None) -> torch.Tensor:
    """D[M][N] (BF16) = alpha * deq(A) deq(B)^T + bias, on the tensor cores."""
    d = _out_bf16(M, N, a_codes.device) if out is None else out
    mxq_gemm_w4a4(a_codes, a_sf, b_codes, b_sf, M, N, K, alpha, bias, d.data_ptr(), d.stride(0), stream)
    return d


@_on_stream
def gemm_w4a8(a_e4m3, act_scale, b_codes, b_sf, M, N, K, bias=None, out=None, stream=None) -> torch.Tensor:
    """D[M][N] (BF16) = act_scale * e4m3(A) deq(B)^T + bias, on the tensor cores."""
    d = _out_bf16(M, N, a_e4m3.device) if out is None else out
    mxq_gemm_w4a8(a_e4m3, act_scale, b_codes, b_sf, M, N, K, bias, d.data_ptr(), d.stride(0), stream)
    return d


@_on_stream
def dequant_mxfp4(codes: torch.Tensor, sf: torch.Tensor, K: int, out=None, stream=None) -> torch.Tensor:
    """MXFP4 codes [rows][K/2] + swizzled scales -> BF16 [rows][K] (exact values)."""
    rows = codes.shape[0]
    o = _out_bf16(rows, K, codes.device) if out is None else out
    mxq_dequant_mxfp4(codes, sf, rows, K, o.data_ptr(), o.stride(0), stream)
    return o


@_on_stream
def qdq_act(x: torch.Tensor, fmt: int = MXQ_ACT_MXFP4, rule: int = MXQ_SCALE_OCP, hadamard128: bool = False,
            act_scale: float = 1.0, out=None, stream=None) -> torch.Tensor:
    """BF16 dequant(quant(X)) with the activation quantiser's arithmetic (fake quantisation)."""
    x = _bf16_2d(x, "x")
    M, K = x.shape
    o = _out_bf16(M, K, x.device) if out is None else out
    mxq_qdq_act(x.data_ptr(), M, K, x.stride(0), fmt, rule, hadamard128, act_scale, o.data_ptr(), o.stride(0),
                stream)
    return o


@_on_stream
def channel_absmax(x: torch.Tensor, hadamard128: bool = False, out=None, accumulate: bool = False,
                   stream=None) -> torch.Tensor:
    """Per-channel max |x R| over the rows (FP32 [K]); accumulate merges into `out`."""
    x = _bf16_2d(x, "x")
    rows, K = x.shape
    o = torch.empty(K, dtype=torch.float32, device=x.device) if out is None else out
    mxq_channel_absmax(x.data_ptr(), rows, K, x.stride(0), hadamard128, accumulate, o, stream)
    return o


@_on_stream
def smooth_factors(amax_x: torch.Tensor, amax_w: torch.Tensor, alpha: float = 0.5, stream=None):
    """SmoothQuant (lambda, 1/lambda) from the channel maxima of activations and weights."""
    K = amax_x.numel()
    lam = torch.empty(K, dtype=torch.float32, device=amax_x.device)
    inv = torch.empty_like(lam)
    mxq_smooth_factors(amax_x, amax_w, K, alpha, lam, inv, stream)
    return lam, inv


@_on_stream
def quantize_smooth(x: torch.Tensor, chan_scale: torch.Tensor, rule: int = MXQ_SCALE_OCP,
                    hadamard128: bool = False, out=None, stream=None):
    """MXFP4 codes + scales of (x R) * chan_scale (per channel): 1/lambda for activations,
    lambda for weights."""
    x = _bf16_2d(x, "x")
    rows, K = x.shape
    if out is None:
        out = (torch.empty(rows, K // 2, dtype=torch.uint8, device=x.device),
               torch.empty(mxq_sf_bytes(rows, K), dtype=torch.uint8, device=x.device))
    q, sf = out
    mxq_quantize_smooth(x.data_ptr(), rows, K, x.stride(0), rule, hadamard128, chan_scale, q, sf, stream)
    return q, sf


@_on_stream
def quantize_vt(v: torch.Tensor, rule: int = MXQ_SCALE_UOS, out=None, stream=None):
    """V [S][H*d] -> V^T MXFP4 (codes [H*d][Sp/2], scales) with 32-key blocks."""
    v = _bf16_2d(v, "v")
    S, HD = v.shape
    Sp = mxq_attn_padded_keys(S)
    if out is None:
        out = (torch.empty(HD, Sp // 2, dtype=torch.uint8, device=v.device),
               torch.empty(mxq_sf_bytes(HD, Sp), dtype=torch.uint8, device=v.device))
    mxq_quantize_vt(v.data_ptr(), S, HD, v.stride(0), rule, out[0], out[1], stream)
    return out


@_on_stream
def attention_mxfp4(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, H: int, rule: int = MXQ_SCALE_UOS,
                    out=None, stream=None) -> torch.Tensor:
    """MXFP4 attention with UOS / PNQ: q [Sq][H*d], k, v [Skv][H*d] BF16 -> O [Sq][H*d] BF16.
    Quantises Q, K (blocks along d) and V (blocks along the keys), then one attention launch."""
    Sq, HD = q.shape
    Skv = k.shape[0]
    d = HD // H
    qc, qs = quantize_act(q, rule, False, stream=stream)
    kc, ks = quantize_act(k, rule, False, stream=stream)
    vc, vs = quantize_vt(v, rule, stream=stream)
    o = _out_bf16(Sq, HD, q.device) if out is None else out
    mxq_attention_mxfp4(qc, qs, kc, ks, vc, vs, Sq, Skv, H, d, rule, o.data_ptr(), o.stride(0), stream)
    return o


@_on_stream
def linear_w4a4(x: torch.Tensor, w_codes, w_sf, N: int, rule: int = MXQ_SCALE_OCP, hadamard128: bool = False,
                bias=None, stream=None) -> torch.Tensor:
    """The quantized linear layer: dynamic MXFP4 quantisation of X, then the W4A4 GEMM."""
    M, K = x.shape
    q, sf = quantize_act(x, rule, hadamard128, stream=stream)
    return gemm_w4a4(q, sf, w_codes, w_sf, M, N, K, 1.0, bias, stream=stream)


def linear_workspace(M: int, K: int, device) -> torch.Tensor:
    """A workspace for linear_w4a4_ws (the quantised activations)."""
    return torch.empty(mxq_linear_workspace_bytes(M, K), dtype=torch.uint8, device=device)


@_on_stream
def linear_w4a4_ws(x: torch.Tensor, w_codes, w_sf, N: int, rule: int = MXQ_SCALE_OCP, alpha: float = 1.0,
                   bias=None, workspace=None, out=None, stream=None) -> torch.Tensor:
    """The quantized linear layer in one call of the C ABI (quantised activations in `workspace`)."""
    x = _bf16_2d(x, "x")
    M, K = x.shape
    ws = linear_workspace(M, K, x.device) if workspace is None else workspace
    d = _out_bf16(M, N, x.device) if out is None else out
    mxq_linear_w4a4(x.data_ptr(), M, K, x.stride(0), rule, w_codes, w_sf, N, alpha, bias, ws, ws.numel(),
                    d.data_ptr(), d.stride(0), stream)
    return d


@_on_stream
def linear_w4a4_static(x: torch.Tensor, w_codes, w_sf, N: int, rule: int = MXQ_SCALE_OCP, alpha: float = 1.0,
                       bias=None, out=None, stream=None) -> torch.Tensor:
    """The quantized linear layer with the library's own fixed scratch (no allocation by the call)."""
    x = _bf16_2d(x, "x")
    M, K = x.shape
    d = _out_bf16(M, N, x.device) if out is None else out
    mxq_linear_w4a4_static(x.data_ptr(), M, K, x.stride(0), rule, w_codes, w_sf, N, alpha, bias, d.data_ptr(),
                           d.stride(0), stream)
    return d


@_on_stream
def linear_w4a8(x: torch.Tensor, act_scale: float, w_codes, w_sf, N: int, bias=None, stream=None) -> torch.Tensor:
    """The W4A8 layer: static FP8 quantisation of X, then the W4A8 GEMM."""
    M, K = x.shape
    q = quantize_act_fp8(x, act_scale, stream=stream)
    return gemm_w4a8(q, act_scale, w_codes, w_sf, M, N, K, bias, stream=stream)
