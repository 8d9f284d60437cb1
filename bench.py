"""Benchmark of the MXFP4 quantized linear layer on B200.

One step = one pass of the hot path over one batch of the Wan2.2-A14B FFN workload
(M = 32760 tokens): dynamic MXFP4 quantisation of X_up [32760 x 5120] (OCP rule),
W4A4 GEMM against the packed W_up [13824 x 5120], dynamic quantisation of X_down
[32760 x 13824], W4A4 GEMM against W_down [5120 x 13824]; BF16 outputs.  Weights are
packed once before timing (offline, as the layer is deployed).

Metric: TFLOP/s including activation quantisation = 2*M*K*N per GEMM / step time.
Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a device
synchronize, CUDA events on the launching stream, max over ranks.  The per-step
traffic (> 2 GB) exceeds the 126 MB L2, so no extra flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxq|reference]

Under torchrun each rank runs its own replica of the layer on its own token batch
(weak scaling, no collective on the data path); ``value`` is the whole-job rate.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MXFP4 W4A4 GEMM TFLOPS incl. act-quant and % of B200 dense FP4 peak"
METRIC_W4A8 = "MXFP4 W4A8 GEMM TFLOPS incl. act-quant and % of B200 dense FP8 peak"
METRIC_QDQ = "MXFP4 quantise-dequantise + weight dequantisation GB/s (HBM-bound)"
METRIC_ATTN = "MXFP4 attention (UOS + PNQ) TFLOPS incl. Q/K/V quantisation and % of B200 dense FP4 peak"
METRIC_POLICY = "precision-selection pass (plain + rotation/SmoothQuant W4A4 vs BF16 SQNR), ms per Wan FFN block"
UNIT = "TFLOP/s"
NOMINAL_FP4_TFLOPS = 9000.0          # dense FP4, nominal
NOMINAL_FP8_TFLOPS = 4500.0          # dense FP8, nominal (kind::mxf8f6f4 runs at the FP8 rate)
FP4_PER_BF16 = 4.0                   # nominal FP4 : BF16 dense ratio (9 / 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0                   # nominal FP8 : BF16 dense ratio (4.5 / 2.25 PFLOP/s)
# DRAM traffic per launch of the dominant kernel, from an ncu capture (see profiles/); None if
# the kernel changed since the counters were taken.
# Wan FFN: mean of the up (256.9 + 867.8 MB) and down (326.8 + 313.8 MB) GEMM launches.
TRAFFIC = {"wan_ffn": (256.9e6 + 867.8e6 + 326.8e6 + 313.8e6) / 2}
# Packed weight bytes per workload (MXFP4 codes + scales), for the L2-residency decision.
W_BYTES = {"wan_ffn": 2 * 5120 * 13824 * 17 // 32, "wan_attn_hadamard": 4 * 5120 * 5120 * 17 // 32,
           "flux_w4a8": (9216 + 12288) * 3072 * 17 // 32, "m_sweep": 13824 * 5120 * 17 // 32, "qdq_wan_ffn": 0,
           "policy_wan_ffn": 0, "attn_wan": 0}
WORKLOAD = "Wan2.2-A14B FFN W4A4 (up 32760x5120->13824, down 32760x13824->5120), dynamic MXFP4 acts, OCP rule"
M_TOK, D_MODEL, D_FF = 32760, 5120, 13824


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["mxq", "reference"], default="mxq")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=40)
    p.add_argument("--m", type=int, default=0, help="token count (0: the workload's own)")
    p.add_argument("--workload", choices=["wan_ffn", "wan_attn_hadamard", "flux_w4a8", "m_sweep", "qdq_wan_ffn",
                                          "policy_wan_ffn", "attn_wan"],
                   default="wan_ffn")
    p.add_argument("--rule", choices=["ocp", "uos"], default=None,
                   help="activation scale rule (default: ocp; uos for the attention workload)")
    p.add_argument("--smooth", action="store_true",
                   help="SmoothQuant after the rotation (W4A4 workloads; factors calibrated before timing)")
    return p.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return pk, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks (read only)
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                mask = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU oracle baseline
def clock_matches_sustained(clock_summary, peaks) -> bool:
    """The sustained peak was measured at the power-capped clock: a fraction against it means
    something only for a run at about that clock."""
    ref = (peaks.get("clocks_under_load") or {}).get("sm_mhz_median")
    run = (clock_summary or {}).get("sm_mhz")
    return bool(ref and run and abs(run / ref - 1.0) <= 0.05)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_oracle_sample(x_up_rows, x_down_rows, w_up_q, w_down_q):
    """Times the oracle (as it stands) on a row sample of the same step: quantise the
    sampled activation rows, then the FP64 GEMM of those rows against the packed
    weights (packing is offline on both sides).  Returns (TFLOP/s, seconds, cores)."""
    import oracle
    cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    flops = 0.0
    for x, (bq, bsf, N) in ((x_up_rows, w_up_q), (x_down_rows, w_down_q)):
        R, K = x.shape
        aq, asl = oracle.quantize_mxfp4(x, nthreads=cores)
        oracle.gemm(aq, oracle.sf_swizzle(asl, R, K), bq, bsf, R, N, K, nthreads=cores)
        flops += 2.0 * R * N * K
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, dt, cores


def oracle_pack(w_cpu):
    import oracle
    N, K = w_cpu.shape
    bq, bsl = oracle.quantize_mxfp4(w_cpu)
    return bq, oracle.sf_swizzle(bsl, N, K), N


CPU_SAMPLE_ROWS = 24
CPU_SAMPLE_SECONDS = 10.0  # oracle time of the cpu_baseline leg


# ------------------------------------------------------------------ reference arm
REFERENCE_BUDGET_S = 120.0  # host time the whole --impl reference run may take


def run_reference(args, rank, world):
    """The oracle timed on the host cores, on a bounded sample of the same workload:
    CPU_SAMPLE_ROWS token rows against the first n_up rows of W_up and n_dn of W_down.
    A first full-width sample gives the cost; n_up and n_dn (multiples of 128) keep
    warm-up + steps within REFERENCE_BUDGET_S, since the oracle's cost grows with the
    weight rows it expands, not with the token rows."""
    if rank != 0:
        return
    import torch
    from mxfp4_block_scaled_mxq_b200 import inputs
    x_up, w_up = inputs.wan_ffn(which="up", M=CPU_SAMPLE_ROWS)
    x_dn, w_dn = inputs.wan_ffn(which="down", M=CPU_SAMPLE_ROWS)
    wq_up, wq_dn = oracle_pack(w_up), oracle_pack(w_dn)
    _, dt0, cores = cpu_oracle_sample(x_up, x_dn, wq_up, wq_dn)
    n_samples = max(1, args.warmup - 1 + args.steps)
    frac = min(1.0, REFERENCE_BUDGET_S / (dt0 * n_samples))
    n_up = max(128, int(D_FF * frac) // 128 * 128)
    n_dn = max(128, int(D_MODEL * frac) // 128 * 128)
    if n_up < D_FF:
        wq_up = oracle_pack(w_up[:n_up].contiguous())
    if n_dn < D_MODEL:
        wq_dn = oracle_pack(w_dn[:n_dn].contiguous())
    times = []
    for i in range(max(0, args.warmup - 1) + args.steps):
        _, dt, cores = cpu_oracle_sample(x_up, x_dn, wq_up, wq_dn)
        if i >= max(0, args.warmup - 1):
            times.append(dt)
    flops = 2.0 * CPU_SAMPLE_ROWS * (n_up * D_MODEL + n_dn * D_FF)
    total = sum(times)
    value = flops * len(times) / total / 1e12
    sample = (f"{CPU_SAMPLE_ROWS} token rows of X_up and X_down per step against the first {n_up} rows of "
              f"W_up and {n_dn} of W_down (quantise + FP64 GEMM)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_TOK, "parallelism": "replicas x1 (token batches, no collective)",
                   "timing": "oracle on the host cores; each step a bounded sample of the workload "
                             "(cpu_baseline.sample), wall clock"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu": cpu_model(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ------------------------------------------------------------------ multi-rank helpers
def rank_seed(rank: int) -> int:
    """Each rank draws its own token batch (weak scaling over independent replicas)."""
    return 2000 + 100 * rank


def max_over_ranks(x: float, dist, device) -> float:
    """The job's time is the slowest rank's (max over ranks, on the device for NCCL)."""
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """TFLOP/s of the whole job: every rank processes its own step of flops_per_step."""
    return world * flops_per_step * steps / (max_ms / 1e3) / 1e12


# ------------------------------------------------------------------ workloads
class Part:
    """One launch of the step: kind 'quant' (HBM-bound), 'gemm' (tensor-bound), 'lib' (a library
    kernel, e.g. the cuBLAS BF16 reference) or 'other' (small reductions)."""

    def __init__(self, label, kind, fn, flops=0.0, nbytes=0.0, peak_kind="fp4", launches=None):
        self.label, self.kind, self.fn, self.flops, self.nbytes, self.peak_kind = label, kind, fn, flops, nbytes, peak_kind
        # kernels of this library the part launches ("lib" parts run a library kernel)
        self.launches = launches if launches is not None else (0 if kind == "lib" else 1)


def gemm_bytes(M, N, K, a_bytes_per_elt=17 / 32):
    """Algorithmic bytes of one GEMM launch: A and B read once (MXFP4: 0.5 B per element +
    one scale byte per 32), D written once (BF16)."""
    return M * K * a_bytes_per_elt + N * K * 17 / 32 + 2.0 * M * N


def weight_copies(workload, working_set, w_bytes, l2):
    """How many copies of the weights the timed loop rotates over: 1 (no rotation) unless
    the M sweep's working set fits in 4x L2, then at least 4 and at least 2x L2 in total, so
    that every step streams its weights from HBM."""
    if workload != "m_sweep" or working_set >= 4 * l2 or w_bytes <= 0:
        return 1
    return max(4, -(-2 * l2 // w_bytes))


def quant_bytes(M, K, fp8=False):
    """Algorithmic bytes of one activation-quantiser launch: BF16 in, codes (+ scales) out."""
    return M * K * 2 + (M * K if fp8 else M * K // 2 + M * K // 32)


def build_workload(name, dev, M, seed, rule_name, smooth=False):
    """Returns (description, parts, inputs [(device tensor)], outputs [(device tensor)], flops per step)."""
    import torch
    from mxfp4_block_scaled_mxq_b200 import inputs, mxq

    rule = mxq.MXQ_SCALE_UOS if rule_name == "uos" else mxq.MXQ_SCALE_OCP

    def qbufs(rows, K):
        return (torch.empty(rows, K // 2, dtype=torch.uint8, device=dev),
                torch.empty(mxq.mxq_sf_bytes(rows, K), dtype=torch.uint8, device=dev))

    def out(rows, N):
        return torch.empty(rows, N, dtype=torch.bfloat16, device=dev)

    def w4a4_layer(label, x, w, hadamard, qb=None, share_quant=False, factors=None):
        """Parts for quantise(x) (unless shared) + GEMM against packed w.  With `smooth`,
        SmoothQuant factors (lambda, 1/lambda) -- given, or from the channel maxima of x and
        w (offline calibration) -- are applied after the rotation on both sides."""
        rows, K = x.shape
        N = w.shape[0]
        if smooth:
            lam, inv = factors if factors is not None else mxq.smooth_factors(
                mxq.channel_absmax(x, hadamard), mxq.channel_absmax(w, hadamard), 0.5)
            wc, wsf = mxq.quantize_smooth(w, lam, mxq.MXQ_SCALE_OCP, hadamard)
            quant = lambda: mxq.quantize_smooth(x, inv, rule, hadamard, out=qb)
        else:
            wc, wsf = mxq.pack_weight(w, mxq.MXQ_SCALE_OCP, hadamard)
            quant = lambda: mxq.quantize_act(x, rule, hadamard, out=qb)
        qb = qb if qb is not None else qbufs(rows, K)
        d = out(rows, N)
        parts = []
        if not share_quant:
            parts.append(Part(f"quant_{label}", "quant", quant, nbytes=quant_bytes(rows, K)))
        parts.append(Part(f"gemm_{label}", "gemm",
                          lambda: mxq.gemm_w4a4(qb[0], qb[1], wc, wsf, rows, N, K, out=d),
                          flops=2.0 * rows * N * K, nbytes=gemm_bytes(rows, N, K)))
        return parts, qb, d

    if name == "wan_ffn":
        x_up, w_up = inputs.wan_ffn(seed=seed, which="up", device=dev, M=M)
        x_dn, w_dn = inputs.wan_ffn(seed=seed, which="down", device=dev, M=M)
        p1, _, d1 = w4a4_layer("up", x_up, w_up, False)
        p2, _, d2 = w4a4_layer("down", x_dn, w_dn, False)
        rows = x_up.shape[0]
        desc = WORKLOAD if rows == M_TOK else WORKLOAD.replace("32760", str(rows))
        if rule_name == "uos":
            desc = desc.replace("OCP rule", "UOS rule")
        return desc, p1 + p2, [x_up, x_dn], [d1, d2], sum(p.flops for p in p1 + p2)

    if name == "wan_attn_hadamard":
        x, ws = inputs.wan_attn(seed=4000 + seed - 2000, device=dev, M=M)
        x_o = inputs.heavy_tailed_bf16(x.shape[0], x.shape[1], seed + 77, device=dev)
        f_qkv = None
        if smooth:  # Q, K and V share one quantised X: one lambda from the three weights' maxima
            aw = torch.maximum(torch.maximum(mxq.channel_absmax(ws[0], True), mxq.channel_absmax(ws[1], True)),
                               mxq.channel_absmax(ws[2], True))
            f_qkv = mxq.smooth_factors(mxq.channel_absmax(x, True), aw.contiguous(), 0.5)
        pq, qb, dq = w4a4_layer("q", x, ws[0], True, factors=f_qkv)
        pk, _, dk = w4a4_layer("k", x, ws[1], True, qb=qb, share_quant=True, factors=f_qkv)
        pv, _, dv = w4a4_layer("v", x, ws[2], True, qb=qb, share_quant=True, factors=f_qkv)
        po, _, do = w4a4_layer("o", x_o, ws[3], True)
        parts = pq + pk + pv + po
        desc = (f"Wan2.2 attention projections W4A4 with 128-point block-Hadamard"
                f"{' + SmoothQuant (alpha 0.5)' if smooth else ''}, Q/K/V/O "
                f"{x.shape[0]}x5120->5120, {rule_name.upper()} rule")
        return desc, parts, [x, x_o], [dq, dk, dv, do], sum(p.flops for p in parts)

    if name == "flux_w4a8":
        x, w_qkv, x_cal = inputs.flux_w4a8(which="qkv", device=dev, M=M)
        _, w_mlp, _ = inputs.flux_w4a8(which="mlp", device=dev, M=M)
        s = inputs.static_fp8_scale(x_cal)
        rows, K = x.shape
        q8 = torch.empty(rows, K, dtype=torch.uint8, device=dev)
        parts = [Part("quant_fp8", "quant", lambda: mxq.quantize_act_fp8(x, s, out=q8),
                      nbytes=quant_bytes(rows, K, fp8=True))]
        # The QKV and MLP input projections read the same X: their packed weights are stacked
        # (FLUX.1's single-stream blocks hold them as one linear layer) and run as one GEMM over
        # N = 9216 + 12288, output columns [0, 9216) QKV and [9216, 21504) MLP; every output
        # element is the same K-sum as in two launches.
        w = torch.cat([w_qkv, w_mlp], 0)
        N = w.shape[0]
        wc, wsf = mxq.pack_weight(w)
        d = out(rows, N)
        parts.append(Part("gemm_qkv_mlp", "gemm", lambda: mxq.gemm_w4a8(q8, s, wc, wsf, rows, N, K, out=d),
                          flops=2.0 * rows * N * K, nbytes=gemm_bytes(rows, N, K, 1.0), peak_kind="fp8"))
        desc = (f"FLUX.1-dev-shaped W4A8: M={rows}, QKV 3072->9216 and MLP 3072->12288 (stacked, one GEMM), "
                f"static FP8 E4M3 acts")
        return desc, parts, [x], [d], sum(p.flops for p in parts)

    if name == "m_sweep":
        x, w = inputs.m_sweep(M, seed=seed, device=dev)
        p, _, d = w4a4_layer("up", x, w, False)
        desc = f"M sweep W4A4: M={M}, 5120->13824, N(0,1) acts"
        return desc, p, [x], [d], sum(q.flops for q in p)

    if name == "qdq_wan_ffn":
        x, w = inputs.wan_ffn(seed=seed, which="up", device=dev, M=M)
        rows, K = x.shape
        N = w.shape[0]
        wc, wsf = mxq.pack_weight(w)
        d_x, d_w = out(rows, K), out(N, K)
        parts = [Part("qdq_x_up", "quant", lambda: mxq.qdq_act(x, rule=rule, out=d_x), nbytes=4.0 * rows * K),
                 Part("dequant_w_up", "quant", lambda: mxq.dequant_mxfp4(wc, wsf, K, out=d_w),
                      nbytes=N * K / 2 + N * K / 32 + 2.0 * N * K)]
        desc = (f"Wan2.2 FFN-up operands: fake-quantise X_up {rows}x{K} (MXFP4, {rule_name.upper()} rule) "
                f"and expand packed W_up {N}x{K} to BF16")
        return desc, parts, [x], [d_x, d_w], 0.0

    if name == "policy_wan_ffn":
        # One selection pass over the FFN block on a calibration batch: the BF16 layers
        # (cuBLAS), both conditions' weight packing, quantisation and W4A4 GEMMs, the
        # SmoothQuant calibration, and the SQNR sums.
        parts, xs, outs = [], [], []
        acc = torch.zeros(4, dtype=torch.float64, device=dev)
        flops = 0.0
        for label in ("up", "down"):
            x, w = inputs.wan_ffn(seed=seed, which=label, device=dev, M=M)
            rows, K = x.shape
            N = w.shape[0]
            xs.append(x)
            ref, y1, y2 = out(rows, N), out(rows, N), out(rows, N)
            outs += [ref, y1, y2]
            wq, q1, wq2, q2 = qbufs(N, K), qbufs(rows, K), qbufs(N, K), qbufs(rows, K)
            ax = torch.empty(K, dtype=torch.float32, device=dev)
            aw = torch.empty_like(ax)
            lam, inv = torch.empty_like(ax), torch.empty_like(ax)
            f = 2.0 * rows * N * K
            flops += 2 * f

            def sq(y, a):
                return lambda: mxq.mxq_sqnr_accumulate(y.data_ptr(), y.stride(0), ref.data_ptr(), ref.stride(0),
                                                       rows, N, True, a)
            parts += [
                Part(f"bf16_ref_{label}", "lib", lambda x=x, w=w, ref=ref: torch.matmul(x, w.t(), out=ref), flops=f),
                Part(f"pack_{label}", "quant", lambda w=w, wq=wq: mxq.mxq_pack_weight(
                    w.data_ptr(), N, K, K, mxq.MXQ_SCALE_OCP, False, wq[0], wq[1]), nbytes=quant_bytes(N, K)),
                Part(f"quant_{label}", "quant", lambda x=x, q1=q1: mxq.quantize_act(x, rule, out=q1),
                     nbytes=quant_bytes(rows, K)),
                Part(f"gemm_{label}", "gemm", lambda q1=q1, wq=wq, y1=y1: mxq.gemm_w4a4(
                    q1[0], q1[1], wq[0], wq[1], rows, N, K, out=y1), flops=f),
                Part(f"sqnr_plain_{label}", "other", sq(y1, acc[0:2])),
                Part(f"absmax_{label}", "other", lambda x=x, w=w, ax=ax, aw=aw: (
                    mxq.channel_absmax(x, True, out=ax), mxq.channel_absmax(w, True, out=aw)), launches=2),
                Part(f"factors_{label}", "other", lambda ax=ax, aw=aw, lam=lam, inv=inv: mxq.mxq_smooth_factors(
                    ax, aw, K, 0.5, lam, inv)),
                Part(f"pack_smooth_{label}", "quant", lambda w=w, lam=lam, wq2=wq2: mxq.quantize_smooth(
                    w, lam, mxq.MXQ_SCALE_OCP, True, out=wq2), nbytes=quant_bytes(N, K)),
                Part(f"quant_smooth_{label}", "quant", lambda x=x, inv=inv, q2=q2: mxq.quantize_smooth(
                    x, inv, rule, True, out=q2), nbytes=quant_bytes(rows, K)),
                Part(f"gemm_smooth_{label}", "gemm", lambda q2=q2, wq2=wq2, y2=y2: mxq.gemm_w4a4(
                    q2[0], q2[1], wq2[0], wq2[1], rows, N, K, out=y2), flops=f),
                Part(f"sqnr_transform_{label}", "other", sq(y2, acc[2:4])),
            ]
        desc = (f"selection pass on the Wan2.2 FFN block (up 5120->13824, down 13824->5120), calibration batch "
                f"M={M}: BF16 reference, plain and rotation+SmoothQuant W4A4, SQNR sums")
        return desc, parts, xs, outs, flops

    if name == "attn_wan":
        # Wan2.2 self-attention: 40 heads of 128 over the video tokens; Q, K, V quantised
        # (UOS by default), then one attention launch over all heads.
        H, d = 40, 128
        q = inputs.normal_bf16(M, H * d, 1.0, seed, device=dev)
        k = inputs.normal_bf16(M, H * d, 1.0, seed + 1, device=dev)
        v = inputs.heavy_tailed_bf16(M, H * d, seed + 2, device=dev)
        arule = mxq.MXQ_SCALE_OCP if rule_name == "ocp" else mxq.MXQ_SCALE_UOS
        qb, kb = qbufs(M, H * d), qbufs(M, H * d)
        Sp = mxq.mxq_attn_padded_keys(M)
        vb = (torch.empty(H * d, Sp // 2, dtype=torch.uint8, device=dev),
              torch.empty(mxq.mxq_sf_bytes(H * d, Sp), dtype=torch.uint8, device=dev))
        o = out(M, H * d)
        flops = 4.0 * M * M * d * H
        parts = [
            Part("quant_q", "quant", lambda: mxq.quantize_act(q, arule, out=qb), nbytes=quant_bytes(M, H * d)),
            Part("quant_k", "quant", lambda: mxq.quantize_act(k, arule, out=kb), nbytes=quant_bytes(M, H * d)),
            Part("quant_vt", "quant", lambda: mxq.quantize_vt(v, arule, out=vb), nbytes=quant_bytes(M, H * d)),
            Part("attention", "gemm", lambda: mxq.mxq_attention_mxfp4(qb[0], qb[1], kb[0], kb[1], vb[0], vb[1], M, M,
                                                                      H, d, arule, o.data_ptr(), o.stride(0)),
                 flops=flops),
        ]
        desc = (f"Wan2.2 self-attention, {M} tokens x {H} heads x d={d}, MXFP4 Q/K/V/P with "
                f"{'UOS' if arule == mxq.MXQ_SCALE_UOS else 'OCP'} scales and PNQ")
        return desc, parts, [q, k, v], [o], flops

    raise ValueError(f"unknown workload {name}")


# ------------------------------------------------------------------ our arm
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    from mxfp4_block_scaled_mxq_b200 import mxq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    mxq.lib()

    # Inputs (per rank its own token batch); weights packed once before timing.
    default_m = {"wan_ffn": M_TOK, "wan_attn_hadamard": M_TOK, "flux_w4a8": 3584, "m_sweep": 1024,
                 "qdq_wan_ffn": M_TOK, "policy_wan_ffn": 4096, "attn_wan": M_TOK}[args.workload]
    M = args.m if args.m else default_m
    rule = args.rule or ("uos" if args.workload == "attn_wan" else "ocp")
    desc, parts, x_in, d_out, flops_step = build_workload(args.workload, dev, M, rank_seed(rank), rule,
                                                          args.smooth)
    stream = torch.cuda.current_stream(dev)

    # Working sets that fit in L2: the M sweep rotates over copies of its weights (at least
    # 4, at least twice L2 in total) so that every step streams them from HBM, steps back to
    # back; the other workloads get an untimed L2 flush (a write of twice L2) before every
    # timed replay.
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    w_bytes = W_BYTES.get(args.workload, 0)
    working_set = sum(t.numel() * t.element_size() for t in x_in + d_out) + w_bytes
    copies = weight_copies(args.workload, working_set, w_bytes, l2)
    part_sets = [parts] + [build_workload(args.workload, dev, M, rank_seed(rank) + 7919 * i, rule, args.smooth)[1]
                           for i in range(1, copies)]
    flush = working_set < 4 * l2 and copies == 1
    scratch = torch.empty(2 * l2, dtype=torch.uint8, device=dev) if flush else None

    for _ in range(args.warmup):
        for ps in part_sets:
            for p in ps:
                p.fn()
    torch.cuda.synchronize(dev)
    if mxq.mxq_debug_poll() != 0:
        raise RuntimeError("a kernel reported a timeout during warm-up")

    # The step is captured once in a CUDA graph (one per weight copy) and replayed (no host
    # launch overhead).

    def capture(fns):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for f in fns:
                f()
        return g

    def time_graphs(gs, iters):
        """Device time of `iters` replays (ms), replay i of gs[i % len(gs)]: each flushed
        before, or all back to back."""
        if flush:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
            for i, (e0, e1) in enumerate(evs):
                scratch.zero_()
                e0.record(stream)
                gs[i % len(gs)].replay()
                e1.record(stream)
            torch.cuda.synchronize(dev)
            return sum(e0.elapsed_time(e1) for e0, e1 in evs)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(iters):
            gs[i % len(gs)].replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    # Steps of microseconds (the M sweep's few-token GEMMs rotating over weight copies) run
    # back to back inside ONE graph of all K steps, as consecutive layers do in a captured
    # model: one graph launch per step would add its launch gap to every step.
    if copies > 1:
        step_graphs = [capture([p.fn for i in range(args.steps) for p in part_sets[i % copies]])]
        timed_replays = 1
    else:
        step_graphs = [capture([p.fn for p in ps]) for ps in part_sets]
        timed_replays = args.steps
    for g in step_graphs:
        g.replay()
    torch.cuda.synchronize(dev)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        ms = time_graphs(step_graphs, timed_replays)
    if world > 1:
        dist.barrier()
        ms = max_over_ranks(ms, dist, dev)
    hbm_only = flops_step == 0.0
    time_metric = args.workload == "policy_wan_ffn"
    bytes_step = sum(p.nbytes for p in parts)
    if time_metric:  # ms per step (per block), the slowest rank's
        value = ms / args.steps
    elif hbm_only:  # GB/s: bytes per step instead of flops
        value = whole_job_rate(bytes_step, args.steps, world, ms) * 1e3
    else:
        value = whole_job_rate(flops_step, args.steps, world, ms)

    # Per-launch durations: each part captured alone and timed the same way.
    n_prof = max(5, min(20, args.steps))
    part_ms = []
    for j in range(len(parts)):
        if copies > 1:
            gs = [capture([part_sets[i % copies][j].fn for i in range(n_prof)])]
            reps = 1
        else:
            gs = [capture([ps[j].fn]) for ps in part_sets]
            reps = n_prof
        for g in gs:
            g.replay()
        part_ms.append(time_graphs(gs, reps) / n_prof)
    if mxq.mxq_debug_poll() != 0:
        raise RuntimeError("a kernel reported a timeout during timing")

    peaks, peak_kind = measured_peaks()
    # Denominator: the burst measured BF16 rate scaled by the nominal dtype ratio -- the
    # larger, more conservative choice.  A long step loop settles under the power cap (the
    # clocks line shows it), so the fraction of the sustained rate is reported beside it.
    peak_of = {"fp4": peaks["bf16_tflops"] * FP4_PER_BF16, "fp8": peaks["bf16_tflops"] * FP8_PER_BF16}
    bf16_sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    sustained_of = {"fp4": bf16_sustained * FP4_PER_BF16, "fp8": bf16_sustained * FP8_PER_BF16}
    parts_out = {}
    for p, t in zip(parts, part_ms):
        if p.kind in ("gemm", "lib"):
            parts_out[p.label] = {"ms": t, "tflops": p.flops / (t / 1e3) / 1e12}
        elif p.kind == "quant":
            parts_out[p.label] = {"ms": t, "gbs": p.nbytes / (t / 1e3) / 1e9}
        else:
            parts_out[p.label] = {"ms": t}
    gemm_t = sum(t for p, t in zip(parts, part_ms) if p.kind == "gemm")
    quant_t = sum(t for p, t in zip(parts, part_ms) if p.kind == "quant")
    gemm_parts = [p for p in parts if p.kind == "gemm"]
    quant_parts = [p for p in parts if p.kind == "quant"]
    gemm_kind = gemm_parts[0].peak_kind if gemm_parts else "fp4"
    achieved_g = sum(p.flops for p in gemm_parts) / (gemm_t / 1e3) / 1e12 if gemm_parts else None
    achieved_q = sum(p.nbytes for p in quant_parts) / (quant_t / 1e3) / 1e9 if quant_parts else None
    kernel_name = ("mx_gemm_pair_kernel" if M > 128 else "mx_gemm_swap_kernel") + (
        "<W4A8> (tcgen05 kind::mxf8f6f4)" if gemm_kind == "fp8" else "<W4A4> (tcgen05 kind::mxf4)")
    if args.workload == "attn_wan":
        kernel_name = "mx_attention_kernel (tcgen05 kind::mxf4 Q K^T and P V, PNQ softmax on the CUDA cores)"
    if hbm_only:
        top = max(zip(parts, part_ms), key=lambda pt: pt[1])
        top_gbs = top[0].nbytes / (top[1] / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": top[0].label, "achieved": top_gbs, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": top_gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
                    "traffic": None}
    elif gemm_t >= quant_t and M <= 128 and all(p.nbytes for p in gemm_parts):
        # few tokens: the GEMM streams its weights once, HBM-bound (ridge ~ M = 281)
        achieved_b = sum(p.nbytes for p in gemm_parts) / (gemm_t / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": kernel_name, "achieved": achieved_b, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved_b / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
                    "traffic": None,
                    "traffic_note": "algorithmic bytes per launch: packed weights + scales, A, D"}
    elif gemm_t >= quant_t:
        roofline = {"bound": "tensor", "kernel": kernel_name, "achieved": achieved_g, "peak": peak_of[gemm_kind],
                    "unit": "TFLOP/s", "frac": achieved_g / peak_of[gemm_kind],
                    "peak_source": f"{peak_kind} bf16_tflops (burst) x "
                                   f"{FP4_PER_BF16 if gemm_kind == 'fp4' else FP8_PER_BF16} (nominal ratio)",
                    "peak_sustained": sustained_of[gemm_kind],
                    "frac_sustained": (achieved_g / sustained_of[gemm_kind]
                                       if clock_matches_sustained(clocks.summary(), peaks) else None),
                    "frac_sustained_note": "only for a run whose median SM clock is within 5 % of the clock the "
                                           "sustained peak was measured at (the power-capped clock)",
                    "traffic": TRAFFIC.get(args.workload) if M == M_TOK else None,
                    "traffic_note": "DRAM bytes per GEMM launch, mean over the step's launches (ncu)"}
    else:
        roofline = {"bound": "hbm", "kernel": "quantize_act", "achieved": achieved_q, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved_q / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
                    "traffic": None}
    nominal = NOMINAL_FP4_TFLOPS if gemm_kind == "fp4" else NOMINAL_FP8_TFLOPS
    result = {
        "metric": (METRIC_POLICY if time_metric else METRIC_QDQ if hbm_only else METRIC_ATTN
                   if args.workload == "attn_wan" else
                   METRIC if args.workload in ("wan_ffn", "m_sweep", "wan_attn_hadamard") else METRIC_W4A8),
        "value": value, "unit": "ms" if time_metric else "GB/s" if hbm_only else UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": not time_metric, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 <-> mxfp4 (e2m1 x e8m0)" if hbm_only else "mxfp4 (e2m1 x e8m0, fp32 accumulate)"
                 if gemm_kind == "fp4"
                 else "e4m3 x mxfp4 (e8m0 scales, fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": desc, "M": M, "parallelism": f"replicas x{world} (token batches, no collective)",
                   "l2": (f"working set {working_set / 1e6:.0f} MB < 4x L2: L2 flushed (untimed) before every "
                          f"timed step" if flush else
                          f"weights {w_bytes / 1e6:.0f} MB fit in L2: {copies} weight copies "
                          f"({copies * w_bytes / 1e6:.0f} MB >= 2x L2) rotated, the K steps back to back in "
                          f"one graph"
                          if copies > 1 else f"working set {working_set / 1e9:.2f} GB > L2, steps back to back"),
                   "timing": ("the K steps captured back to back in one CUDA graph, replayed once"
                              if copies > 1 else "step captured in one CUDA graph, replayed") +
                             "; CUDA events on the launching stream"},
        "pct_of_dense_peak": None if hbm_only or time_metric else 100.0 * value / world / nominal,
        "roofline": roofline,
        "gemm": None if hbm_only else {"achieved": achieved_g, "unit": "TFLOP/s", "peak": peak_of[gemm_kind],
                                       "frac": achieved_g / peak_of[gemm_kind]},
        "quantizer": ({"achieved": achieved_q, "unit": "GB/s", "peak": peaks["hbm_gbs"],
                       "frac": achieved_q / peaks["hbm_gbs"]} if quant_parts else None),
        "parts": parts_out,
        "gpu_launches": sum(p.launches for p in parts) * args.steps,
        "clocks": clocks.summary(),
    }

    # End to end through the public API: pinned host inputs in, outputs back, every step.
    # Pipelined over two buffer sets: the host-to-device copy of step k+1 (copy stream) and
    # the device-to-host copy of step k (second copy stream) overlap step k's kernels.
    if not args.no_e2e:
        second = build_workload(args.workload, dev, M, rank_seed(rank), rule, args.smooth)
        sets = [(parts, x_in, d_out), (second[1], second[2], second[3])]
        hin = [x.cpu().pin_memory() for x in x_in]
        hout = [[torch.empty(d.shape, dtype=d.dtype, pin_memory=True) for d in ds] for _, _, ds in sets]
        s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_run(n_steps, start_event):
            computed, copied_out = [None, None], [None, None]
            s_h2d.wait_event(start_event)
            for k in range(n_steps):
                b = k % 2
                ps, xs, ds = sets[b]
                with torch.cuda.stream(s_h2d):  # inputs of set b: free once step k-2 consumed them
                    if computed[b] is not None:
                        s_h2d.wait_event(computed[b])
                    for x, h in zip(xs, hin):
                        x.copy_(h, non_blocking=True)
                    loaded = torch.cuda.Event()
                    loaded.record(s_h2d)
                stream.wait_event(loaded)
                if copied_out[b] is not None:  # outputs of set b: free once step k-2's copy-out is done
                    stream.wait_event(copied_out[b])
                for p in ps:
                    p.fn()
                computed[b] = torch.cuda.Event()
                computed[b].record(stream)
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(computed[b])
                    for d, h in zip(ds, hout[b]):
                        h.copy_(d, non_blocking=True)
                    copied_out[b] = torch.cuda.Event()
                    copied_out[b].record(s_d2h)
            for ev in copied_out:
                if ev is not None:
                    stream.wait_event(ev)

        warm = torch.cuda.Event()
        warm.record(stream)
        e2e_run(2, warm)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(args.e2e_steps, e0)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems = e0.elapsed_time(e1)
        if world > 1:
            ems = max_over_ranks(ems, dist, dev)
        e2e_value = (ems / args.e2e_steps if time_metric else
                     whole_job_rate(bytes_step, args.e2e_steps, world, ems) * 1e3 if hbm_only
                     else whole_job_rate(flops_step, args.e2e_steps, world, ems))
        result["e2e"] = {"value": e2e_value, "unit": "ms" if time_metric else "GB/s" if hbm_only else UNIT,
                         "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h in hin),
                         "d2h_bytes_per_step": sum(h.numel() * h.element_size() for h in hout[0]),
                         "steps": args.e2e_steps,
                         "pipelined": "H2D of step k+1 and D2H of step k overlap step k's kernels (2 buffer sets)"}

    if rank == 0 and not args.no_cpu_baseline and args.workload == "wan_ffn":
        from mxfp4_block_scaled_mxq_b200 import inputs
        x_up, w_up = inputs.wan_ffn(which="up", M=CPU_SAMPLE_ROWS)
        x_dn, w_dn = inputs.wan_ffn(which="down", M=CPU_SAMPLE_ROWS)
        wq = (oracle_pack(w_up), oracle_pack(w_dn))
        # the sample repeated until about CPU_SAMPLE_SECONDS of oracle time (a bounded count)
        v, dt, cores = cpu_oracle_sample(x_up, x_dn, *wq)
        reps = [dt]
        while sum(reps) < CPU_SAMPLE_SECONDS and len(reps) < 20:
            reps.append(cpu_oracle_sample(x_up, x_dn, *wq)[1])
        v = v * dt * len(reps) / sum(reps)  # same FLOPs per repetition
        result["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "cpu": cpu_model(), "kind": "oracle",
                                  "sample": f"{len(reps)} x {CPU_SAMPLE_ROWS} token rows of X_up and X_down (quantise "
                                            f"+ FP64 GEMM vs all N), {sum(reps):.1f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


if __name__ == "__main__":
    main()
