"""Per-layer (per-block) precision selection from output SQNR.

A block's precision is chosen from its whole-block output SQNR against the BF16 block,
measured under two conditions -- plain MXFP4 W4A4, and W4A4 with the fixed 128-point
Hadamard rotation followed by SmoothQuant -- through tiered thresholds: plain W4A4,
transform-enabled W4A4, W4A8 promotion, or BF16 fallback.
[AMD Quark adds native W4A8 mixed-precision for Wan2.2 video generation on MI350 --
 "Block-level SQNR calibration" and "Fixed rotation selector"]

Every quantised output comes from the library's kernels (quantiser, SmoothQuant
quantiser, block-scaled GEMM, SQNR sums); the BF16 reference layer is a plain cuBLAS
BF16 GEMM through torch.  The thresholds are not on the pages: they are parameters
(defaults 15 dB / 10 dB).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import mxq

NAMES = {mxq.MXQ_PREC_W4A4: "W4A4", mxq.MXQ_PREC_W4A4_TRANSFORM: "W4A4+rotation+SmoothQuant",
         mxq.MXQ_PREC_W4A8: "W4A8", mxq.MXQ_PREC_BF16: "BF16"}


@dataclass
class BlockPrecision:
    sqnr_plain_db: float
    sqnr_transform_db: float
    precision: int

    @property
    def name(self) -> str:
        return NAMES[self.precision]


def _accumulate(y: torch.Tensor, ref: torch.Tensor, acc: torch.Tensor, stream=None) -> None:
    M, N = ref.shape
    mxq.mxq_sqnr_accumulate(y.data_ptr(), y.stride(0), ref.data_ptr(), ref.stride(0), M, N, True, acc, stream)


def measure_block(layers, rule: int = mxq.MXQ_SCALE_OCP, alpha: float = 0.5, stream=None):
    """SQNR sums of a block of linear layers under both conditions.

    layers: iterable of (x [M][K], w [N][K]) BF16 CUDA tensors (calibration activations
    and weights).  Returns two FP64 device tensors [sum ref^2, sum (y - ref)^2]
    (plain, transform).  The transform needs K % 128 == 0; a layer without it counts
    with the plain layer's output under the transform condition as well."""
    dev = None
    acc_plain = acc_tr = None
    for x, w in layers:
        if dev is None:
            dev = x.device
            acc_plain = torch.zeros(2, dtype=torch.float64, device=dev)
            acc_tr = torch.zeros(2, dtype=torch.float64, device=dev)
        M, K = x.shape
        N = w.shape[0]
        ref = torch.matmul(x, w.t())  # the BF16 layer (cuBLAS)
        if N % 8:  # row stride a multiple of 8 elements for the 16-byte loads
            padded = torch.empty(M, (N + 7) // 8 * 8, dtype=torch.bfloat16, device=dev)[:, :N]
            ref = padded.copy_(ref)
        wc, wsf = mxq.pack_weight(w, mxq.MXQ_SCALE_OCP, False, stream=stream)
        y = mxq.linear_w4a4(x, wc, wsf, N, rule, False, stream=stream)
        _accumulate(y, ref, acc_plain, stream)
        if K % 128 == 0:
            lam, inv = mxq.smooth_factors(mxq.channel_absmax(x, True, stream=stream),
                                          mxq.channel_absmax(w, True, stream=stream), alpha, stream=stream)
            wc2, wsf2 = mxq.quantize_smooth(w, lam, mxq.MXQ_SCALE_OCP, True, stream=stream)
            q2, sf2 = mxq.quantize_smooth(x, inv, rule, True, stream=stream)
            y2 = mxq.gemm_w4a4(q2, sf2, wc2, wsf2, M, N, K, stream=stream)
            _accumulate(y2, ref, acc_tr, stream)
        else:
            _accumulate(y, ref, acc_tr, stream)
    return acc_plain, acc_tr


def select_block_precision(layers, high_db: float = 15.0, low_db: float = 10.0, rule: int = mxq.MXQ_SCALE_OCP,
                           alpha: float = 0.5, stream=None) -> BlockPrecision:
    """Measures both conditions on the block and applies the tiers."""
    acc_plain, acc_tr = measure_block(layers, rule, alpha, stream)
    p = acc_plain.cpu().tolist()
    t = acc_tr.cpu().tolist()
    sp, st = mxq.mxq_sqnr_db(p[0], p[1]), mxq.mxq_sqnr_db(t[0], t[1])
    return BlockPrecision(sp, st, mxq.mxq_select_precision(sp, st, high_db, low_db))
