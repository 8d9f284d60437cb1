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
UNIT = "TFLOP/s"
NOMINAL_FP4_TFLOPS = 9000.0          # dense FP4, nominal
FP4_PER_BF16 = 4.0                   # nominal FP4 : BF16 dense ratio (9 / 2.25 PFLOP/s)
WORKLOAD = "Wan2.2-A14B FFN W4A4 (up 32760x5120->13824, down 32760x13824->5120), dynamic MXFP4 acts, OCP rule"
M_TOK, D_MODEL, D_FF = 32760, 5120, 13824


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["mxq", "reference"], default="mxq")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--m", type=int, default=M_TOK, help="token count (profiling of smaller cases)")
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


# ------------------------------------------------------------------ reference arm
def run_reference(args, rank, world):
    """The oracle timed on the host cores, on a bounded row sample of the same workload."""
    if rank != 0:
        return
    import torch
    from mxfp4_block_scaled_mxq_b200 import inputs
    x_up, w_up = inputs.wan_ffn(which="up", M=CPU_SAMPLE_ROWS)
    x_dn, w_dn = inputs.wan_ffn(which="down", M=CPU_SAMPLE_ROWS)
    wq_up, wq_dn = oracle_pack(w_up), oracle_pack(w_dn)
    times, vals = [], []
    for i in range(args.warmup + args.steps):
        v, dt, cores = cpu_oracle_sample(x_up, x_dn, wq_up, wq_dn)
        if i >= args.warmup:
            times.append(dt)
            vals.append(v)
    flops = 2.0 * CPU_SAMPLE_ROWS * (D_MODEL * D_FF) * 2
    total = sum(times)
    value = flops * len(times) / total / 1e12
    sample = f"{CPU_SAMPLE_ROWS} token rows of X_up and X_down per step (quantise + FP64 GEMM vs all N)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD + " -- row sample", "rows_per_step": CPU_SAMPLE_ROWS},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


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
    from mxfp4_block_scaled_mxq_b200 import inputs, mxq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    mxq.lib()

    # Inputs (per rank its own token batch), weights packed once before timing.
    seed = 2000 + 100 * rank
    x_up, w_up = inputs.wan_ffn(seed=seed, which="up", device=dev, M=args.m)
    x_dn, w_dn = inputs.wan_ffn(seed=seed, which="down", device=dev, M=args.m)
    wc_up, wsf_up = mxq.pack_weight(w_up)
    wc_dn, wsf_dn = mxq.pack_weight(w_dn)
    M = x_up.shape[0]
    q_up = (torch.empty(M, D_MODEL // 2, dtype=torch.uint8, device=dev),
            torch.empty(mxq.mxq_sf_bytes(M, D_MODEL), dtype=torch.uint8, device=dev))
    q_dn = (torch.empty(M, D_FF // 2, dtype=torch.uint8, device=dev),
            torch.empty(mxq.mxq_sf_bytes(M, D_FF), dtype=torch.uint8, device=dev))
    d_up = torch.empty(M, D_FF, dtype=torch.bfloat16, device=dev)
    d_dn = torch.empty(M, D_MODEL, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        mxq.quantize_act(x_up, mxq.MXQ_SCALE_OCP, False, out=q_up)
        if ev is not None:
            ev[1].record(stream)
        mxq.gemm_w4a4(q_up[0], q_up[1], wc_up, wsf_up, M, D_FF, D_MODEL, out=d_up)
        if ev is not None:
            ev[2].record(stream)
        mxq.quantize_act(x_dn, mxq.MXQ_SCALE_OCP, False, out=q_dn)
        if ev is not None:
            ev[3].record(stream)
        mxq.gemm_w4a4(q_dn[0], q_dn[1], wc_dn, wsf_dn, M, D_MODEL, D_FF, out=d_dn)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if mxq.mxq_debug_poll() != 0:
        raise RuntimeError("a kernel reported a timeout during warm-up")

    # Whole-step timing (events only at the boundaries).
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(stop)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    flops_gemm = 2.0 * M * D_MODEL * D_FF
    flops_step = 2 * flops_gemm
    value = world * flops_step * args.steps / (ms / 1e3) / 1e12

    # Per-kernel durations (a second, separately timed pass with events between launches).
    n_prof = max(5, min(20, args.steps))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_prof)]
    for e in evs:
        step(e)
    torch.cuda.synchronize(dev)
    seg = [[e[i].elapsed_time(e[i + 1]) for e in evs] for i in range(4)]
    quant_up_ms, gemm_up_ms, quant_dn_ms, gemm_dn_ms = (statistics.mean(s) for s in seg)
    if mxq.mxq_debug_poll() != 0:
        raise RuntimeError("a kernel reported a timeout during timing")

    peaks, peak_kind = measured_peaks()
    fp4_peak = peaks["bf16_tflops_sustained"] * FP4_PER_BF16
    gemm_ms = (gemm_up_ms + gemm_dn_ms) / 2
    achieved = flops_gemm / (gemm_ms / 1e3) / 1e12
    quant_bytes = lambda K: M * K * 2 + M * K // 2 + M * K // 32
    q_gbs_up = quant_bytes(D_MODEL) / (quant_up_ms / 1e3) / 1e9
    q_gbs_dn = quant_bytes(D_FF) / (quant_dn_ms / 1e3) / 1e9

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "mxfp4 (e2m1 x e8m0, fp32 accumulate)", "data": "synthetic",
        "config": {"workload": WORKLOAD if M == M_TOK else WORKLOAD.replace("32760", str(M)), "M": M,
                   "d_model": D_MODEL, "d_ff": D_FF,
                   "parallelism": f"replicas x{world} (token batches, no collective)",
                   "l2": "inputs larger than L2 (> 2 GB of traffic per step), no explicit flush"},
        "pct_of_dense_fp4_peak": 100.0 * value / world / NOMINAL_FP4_TFLOPS,
        "roofline": {"bound": "tensor", "kernel": "mx_gemm_kernel<W4A4> (tcgen05 kind::mxf4)",
                     "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                     "peak_source": f"{peak_kind} bf16_tflops_sustained x {FP4_PER_BF16} (nominal FP4:BF16)",
                     "traffic": None},
        "parts_ms": {"quant_up": quant_up_ms, "gemm_up": gemm_up_ms, "quant_down": quant_dn_ms,
                     "gemm_down": gemm_dn_ms},
        "quantizer": {"bound": "hbm", "achieved_up": q_gbs_up, "achieved_down": q_gbs_dn, "unit": "GB/s",
                      "peak": peaks["hbm_gbs"], "frac_up": q_gbs_up / peaks["hbm_gbs"],
                      "frac_down": q_gbs_dn / peaks["hbm_gbs"]},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks.summary(),
    }

    # End to end through the public API: pinned host X in, D back to the host, every step.
    if not args.no_e2e:
        xh_up = x_up.cpu().pin_memory()
        xh_dn = x_dn.cpu().pin_memory()
        dh_up = torch.empty(d_up.shape, dtype=d_up.dtype, pin_memory=True)
        dh_dn = torch.empty(d_dn.shape, dtype=d_dn.dtype, pin_memory=True)

        def e2e_step():
            x_up.copy_(xh_up, non_blocking=True)
            x_dn.copy_(xh_dn, non_blocking=True)
            step()
            dh_up.copy_(d_up, non_blocking=True)
            dh_dn.copy_(d_dn, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems = e0.elapsed_time(e1)
        if world > 1:
            t = torch.tensor([ems], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        result["e2e"] = {"value": world * flops_step * args.e2e_steps / (ems / 1e3) / 1e12, "unit": UNIT,
                         "h2d_bytes_per_step": xh_up.numel() * 2 + xh_dn.numel() * 2,
                         "d2h_bytes_per_step": dh_up.numel() * 2 + dh_dn.numel() * 2,
                         "steps": args.e2e_steps}

    if rank == 0 and not args.no_cpu_baseline:
        rows = slice(0, CPU_SAMPLE_ROWS)
        v, dt, cores = cpu_oracle_sample(x_up[rows].cpu(), x_dn[rows].cpu(), oracle_pack(w_up.cpu()),
                                         oracle_pack(w_dn.cpu()))
        result["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                  "sample": f"{CPU_SAMPLE_ROWS} token rows of X_up and X_down (quantise + FP64 "
                                            f"GEMM vs all N), {dt:.1f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


if __name__ == "__main__":
    main()
