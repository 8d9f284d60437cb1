"""Seeded synthetic inputs shaped like the linear layers the pages quantise.

This module holds only random-number recipes: it performs none of the
quantisation, rotation or GEMM arithmetic.  Both the CUDA path and the CPU oracle
consume the tensors it returns (the oracle after a copy to the host), so the two
sides always see identical BF16 inputs.

Shapes stand in for Wan2.2-T2V-A14B and FLUX.1-dev linear layers
([AMD Quark adds native W4A8 ... Wan2.2 video generation on MI350] and
[AMD Quark ... FLUX.1-dev MXFP4 on MI350 -- 1024x768 generation]); neither the
models' weights nor their evaluation data are used or needed.

Recipe (all draws FP32 from one ``torch.Generator``, then rounded to BF16 by
``.to(torch.bfloat16)``, which rounds to nearest even):
  * seeds: X = seed, W = seed + 1, calibration draw = seed + 2,
    outlier channel / token choice = seed + 3;
  * outlier counts are round(fraction * count), chosen by a seeded ``randperm``;
  * Student-t(3) = Z / sqrt(chi2_3 / 3) with chi2_3 the sum of three squared
    standard normals; per-channel lognormal(0, 0.5) = exp(0.5 * Z'), one factor per
    K channel.
"""

from __future__ import annotations

import torch

TINY = dict(M=128, K=512, N=512)
WAN_UP = dict(M=32760, K=5120, N=13824)
WAN_DOWN = dict(M=32760, K=13824, N=5120)
FLUX_QKV = dict(M=3584, K=3072, N=9216)
FLUX_MLP = dict(M=3584, K=3072, N=12288)
WAN_ATTN = dict(M=32760, K=5120, N=5120)
SWEEP_K, SWEEP_N = 5120, 13824
SWEEP_M = (16, 64, 256, 1024, 4096, 16384, 65536)

# Chunk (rows) for large draws, to bound the FP32 working set.
_CHUNK_ELEMS = 1 << 26


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(rows: int, cols: int, g: torch.Generator, device) -> torch.Tensor:
    return torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)


def normal_bf16(rows: int, cols: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) draw rounded to BF16."""
    g = _gen(seed, device)
    out = torch.empty(rows, cols, dtype=torch.bfloat16, device=device)
    step = max(1, _CHUNK_ELEMS // cols)
    for r in range(0, rows, step):
        n = min(step, rows - r)
        out[r:r + n] = (_randn(n, cols, g, device) * std).to(torch.bfloat16)
    return out


def _pick(count: int, fraction: float, seed: int, device) -> torch.Tensor:
    k = int(round(fraction * count))
    g = _gen(seed, "cpu")
    return torch.randperm(count, generator=g)[:k].to(device)


def outlier_channels_bf16(rows: int, cols: int, fraction: float, factor: float, seed: int,
                          device="cpu") -> torch.Tensor:
    """N(0,1) activations with round(fraction*cols) channels (K columns) scaled by factor."""
    g = _gen(seed, device)
    chans = _pick(cols, fraction, seed + 3, device)
    mult = torch.ones(cols, dtype=torch.float32, device=device)
    mult[chans] = factor
    out = torch.empty(rows, cols, dtype=torch.bfloat16, device=device)
    step = max(1, _CHUNK_ELEMS // cols)
    for r in range(0, rows, step):
        n = min(step, rows - r)
        out[r:r + n] = (_randn(n, cols, g, device) * mult).to(torch.bfloat16)
    return out


def heavy_tailed_bf16(rows: int, cols: int, seed: int, device="cpu", token_fraction: float = 0.0,
                      token_factor: float = 1.0) -> torch.Tensor:
    """Student-t(3) x per-channel lognormal(0, 0.5); optional per-token outliers
    (round(token_fraction*rows) rows scaled by token_factor)."""
    g = _gen(seed, device)
    chan_scale = torch.exp(0.5 * torch.randn(cols, generator=g, device=device, dtype=torch.float32))
    tok_mult = torch.ones(rows, dtype=torch.float32, device=device)
    if token_fraction > 0:
        tok_mult[_pick(rows, token_fraction, seed + 3, device)] = token_factor
    out = torch.empty(rows, cols, dtype=torch.bfloat16, device=device)
    step = max(1, _CHUNK_ELEMS // (4 * cols))
    for r in range(0, rows, step):
        n = min(step, rows - r)
        z = _randn(n, cols, g, device)
        chi2 = _randn(n, cols, g, device).square_()
        chi2 += _randn(n, cols, g, device).square_()
        chi2 += _randn(n, cols, g, device).square_()
        t3 = z / torch.sqrt(chi2 / 3.0)
        out[r:r + n] = (t3 * chan_scale * tok_mult[r:r + n, None]).to(torch.bfloat16)
    return out


# ---------------------------------------------------------------- named workloads
def tiny(seed: int = 0, device="cpu"):
    """128x512 activations, 1% of channels x20; 512x512 weights ~N(0, 0.02)."""
    x = outlier_channels_bf16(TINY["M"], TINY["K"], 0.01, 20.0, seed, device)
    w = normal_bf16(TINY["N"], TINY["K"], 0.02, seed + 1, device)
    return x, w


def wan_ffn(seed: int = 2000, device="cpu", which: str = "up", M: int | None = None):
    """Wan2.2-A14B FFN: up (5120->13824) or down (13824->5120) at M = 32760 tokens."""
    shp = dict(WAN_UP if which == "up" else WAN_DOWN)
    if M is not None:
        shp["M"] = M
    off = 0 if which == "up" else 10
    x = heavy_tailed_bf16(shp["M"], shp["K"], seed + off, device)
    w = normal_bf16(shp["N"], shp["K"], 0.02, seed + off + 1, device)
    return x, w


def flux_w4a8(seed: int = 3000, device="cpu", which: str = "qkv", M: int | None = None):
    """FLUX.1-dev-shaped W4A8 layer.  Returns (x, w, x_cal): x_cal is the seeded
    calibration draw (same outlier channels, fresh values) from which the static
    per-tensor FP8 scale is taken."""
    shp = dict(FLUX_QKV if which == "qkv" else FLUX_MLP)
    if M is not None:
        shp["M"] = M
    off = 0 if which == "qkv" else 10
    x = outlier_channels_bf16(shp["M"], shp["K"], 0.005, 30.0, seed + off, device)
    w = normal_bf16(shp["N"], shp["K"], 0.02, seed + off + 1, device)
    # Calibration: fresh values (seed + 2) on the same outlier channels (chosen by seed + 3).
    g = _gen(seed + off + 2, device)
    chans = _pick(shp["K"], 0.005, seed + off + 3, device)
    mult = torch.ones(shp["K"], dtype=torch.float32, device=device)
    mult[chans] = 30.0
    x_cal = (_randn(shp["M"], shp["K"], g, device) * mult).to(torch.bfloat16)
    return x, w, x_cal


def static_fp8_scale(x_cal: torch.Tensor) -> float:
    """The config's static per-tensor scale s = fl32(amax(x_cal) / 448), taken once
    from the calibration draw (offline, like weight packing)."""
    amax = x_cal.float().abs().max().item()
    return float(torch.tensor(amax, dtype=torch.float32) / torch.tensor(448.0, dtype=torch.float32))


def wan_attn(seed: int = 4000, device="cpu", M: int | None = None):
    """Wan2.2 attention projections, K = N = 5120: activations as the FFN recipe plus
    0.1% of tokens x50; four weights (Q, K, V, O)."""
    shp = dict(WAN_ATTN)
    if M is not None:
        shp["M"] = M
    x = heavy_tailed_bf16(shp["M"], shp["K"], seed, device, token_fraction=0.001, token_factor=50.0)
    ws = [normal_bf16(shp["N"], shp["K"], 0.02, seed + 1 + 10 * i, device) for i in range(4)]
    return x, ws


def m_sweep(M: int, seed: int = 5000, device="cpu"):
    """K = 5120 -> N = 13824 at the given M: X ~ N(0,1), W ~ N(0, 0.02)."""
    x = normal_bf16(M, SWEEP_K, 1.0, seed, device)
    w = normal_bf16(SWEEP_N, SWEEP_K, 0.02, seed + 1, device)
    return x, w
