"""Shared helpers of the GPU parity tests: run both sides on the same BF16 inputs and
compare.  The oracle always quantises the inputs itself; nothing it consumes or
returns comes from the CUDA path."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import mxq

GEMM_TOL = 5e-3  # max|D - y_ref| / max|y_ref|, y_ref the unrounded FP64 oracle


def sample_rows(M: int, n: int = 256) -> np.ndarray:
    """Deterministic row sample: first rows, the last row, the tail tile, and rows
    spread with a stride across the whole range."""
    if M <= n:
        return np.arange(M, dtype=np.int64)
    rows = set(range(min(32, n // 4)))
    rows.add(M - 1)
    tail0 = (M - 1) // 128 * 128
    rows.update(range(tail0, min(M, tail0 + min(16, n // 8))))
    rows.update(np.linspace(0, M - 1, max(n - len(rows), 2), dtype=np.int64).tolist())
    return np.array(sorted(rows)[:n], dtype=np.int64)


def bias_bits(bias: torch.Tensor | None):
    if bias is None:
        return None
    return bias.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_w4a4(x: torch.Tensor, w: torch.Tensor, rows, rule_a=oracle.RULE_OCP, rule_w=oracle.RULE_OCP,
                hadamard=False, alpha=1.0, bias=None) -> np.ndarray:
    xc, wc = x.detach().cpu(), w.detach().cpu()
    M, K = xc.shape
    N = wc.shape[0]
    sel = xc[torch.as_tensor(rows)]
    a_codes, a_sl = oracle.quantize_mxfp4(sel, rule=rule_a, hadamard=hadamard)
    b_codes, b_sl = oracle.quantize_mxfp4(wc, rule=rule_w, hadamard=hadamard)
    a_sf = oracle.sf_swizzle(a_sl, len(rows), K)
    b_sf = oracle.sf_swizzle(b_sl, N, K)
    return oracle.gemm(a_codes, a_sf, b_codes, b_sf, len(rows), N, K, alpha=alpha, bias_bits=bias_bits(bias))


def oracle_w4a8(x: torch.Tensor, w: torch.Tensor, act_scale: float, rows, bias=None) -> np.ndarray:
    xc, wc = x.detach().cpu(), w.detach().cpu()
    K = xc.shape[1]
    N = wc.shape[0]
    sel = xc[torch.as_tensor(rows)]
    a8 = oracle.quantize_fp8(sel, act_scale)
    b_codes, b_sl = oracle.quantize_mxfp4(wc)
    b_sf = oracle.sf_swizzle(b_sl, N, K)
    return oracle.gemm(a8, None, b_codes, b_sf, len(rows), N, K, alpha=act_scale, bias_bits=bias_bits(bias),
                       a_fp8=True)


def gemm_rel_err(d: torch.Tensor, rows, y_ref: np.ndarray) -> float:
    got = d[torch.as_tensor(rows, device=d.device)].float().cpu().double().numpy()
    assert np.all(np.isfinite(got)), "non-finite output"
    denom = float(np.max(np.abs(y_ref)))
    return float(np.max(np.abs(got - y_ref))) / (denom if denom > 0 else 1.0)


def assert_status_clean():
    assert mxq.mxq_debug_poll() == 0, "a kernel reported a timeout"
