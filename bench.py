"""Benchmark of the smoothed, outlier-split W4A4 linear layer on B200.

One step = one pass of the hot path over one batch of synthetic tokens:
quantize_act (smooth, split, MXFP4-encode) followed by dual_gemm (block-
scaled MXFP4 tcgen05 MMAs + BF16 outlier MMAs into one TMEM accumulator),
with inputs resident in HBM. Default workload: the Wan-like FFN
up-projection, 4096 tokens x 5120 -> 13824, alpha 0.6, k = 128 outliers,
128x1 weight stripes, FP32 output.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload up|down|long|tiny]

Multi-GPU (torchrun, one rank per GPU): tokens are data-parallel, each rank
runs its own batch with no collective on the data path (weak scaling); the
step time is the max over ranks. `--impl reference` times the CPU oracle
(the only reference implementation of this method) on a bounded sample of
the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FP4_PER_BF16 = 4.0          # nominal dense ratio FP4 : BF16 (9 : 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_SPEC_TFLOPS = 9000.0    # published dense FP4 peak, context only


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workloads():
    from outlier_split_mixed_b200 import synth
    return {"up": synth.UP, "down": synth.DOWN, "long": synth.LONG, "tiny": synth.TINY}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock, max clock and throttle reasons via NVML every
    `period` seconds on a background thread (nvidia-smi's data source)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period: float = 0.01):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        names = [n for n, b in self.REASONS.items() if self.reasons & b]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ oracle arm

def oracle_sample_throughput(cfg, rows_per_step: int, steps: int, warmup: int):
    """Time the CPU oracle (quantize_act + dual-branch product) on
    `rows_per_step` tokens of the workload per step. Weights are packed
    offline, outside the timed region, as on the GPU path."""
    import oracle
    from outlier_split_mixed_b200 import synth
    M_s = rows_per_step * (steps + warmup)
    X = cfg.make_x(min(cfg.M, max(M_s, 256)))
    W = cfg.make_w()
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, O = oracle.calibrate(amax, wmax, cfg.alpha, cfg.k)
    wc, wsc, wh = oracle.pack_weights(W, s, O, cfg.wmode)
    times = []
    for i in range(steps + warmup):
        lo = (i * rows_per_step) % max(1, X.shape[0] - rows_per_step)
        xr = X[lo:lo + rows_per_step]
        t0 = time.perf_counter()
        ac, asc, ah = oracle.quantize_act(xr, inv_s, O)
        oracle.dual_gemm_rows(ac, asc, ah, np.arange(rows_per_step), wc, wsc, wh)
        t1 = time.perf_counter()
        if i >= warmup:
            times.append(t1 - t0)
    t = float(np.mean(times))
    flops = 2.0 * rows_per_step * cfg.N * cfg.K
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return flops / t / 1e12, t, cores


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return 0
    rows = max(1, args.ref_rows)
    tflops, t, cores = oracle_sample_throughput(cfg, rows, args.steps, args.warmup)
    line = {
        "impl": "reference",
        "metric": "dual-branch W4A4 GEMM effective TFLOP/s (+act quantize)",
        "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (oracle)", "data": "synthetic",
        "config": {"workload": cfg.name, "M": cfg.M, "K": cfg.K, "N": cfg.N, "k": cfg.k, "alpha": cfg.alpha,
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} of {cfg.M} tokens per step, weights packed offline"},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import outlier_split_mixed_b200 as osm
    from outlier_split_mixed_b200 import dist as odist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    M, K, N = cfg.M, cfg.K, cfg.N
    epi = osm.EPI_BF16 if cfg.out_bf16 else osm.EPI_F32

    # synthetic batch (each rank its own tokens: data-parallel shards)
    X = cfg.make_x() if rank == 0 else cfg.make_x()  # same recipe; shards are independent batches
    W = cfg.make_w()
    Xd = torch.from_numpy(X.view(np.int16)).to(dev).view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)

    # offline: calibrate (statistics all-reduced over ranks), plan, pack
    amax = torch.zeros(K, dtype=torch.float32, device=dev)
    wmax = torch.empty(K, dtype=torch.float32, device=dev)
    osm.act_amax_accumulate(Xd, amax)
    osm.weight_amax(Wd, wmax)
    s, inv_s, O = odist.calibrate_from_local_stats(amax, wmax, cfg.alpha, cfg.k)
    plan = osm.Plan(K, N, cfg.k, s, O, cfg.wmode)
    wc, wsc, wh = plan.alloc_packed(N, dev)
    osm.pack_weights(plan, Wd, wc, wsc, wh)
    ac, asc, ah = plan.alloc_packed(M, dev)
    Y = torch.empty((M, N), dtype=torch.float32 if epi == osm.EPI_F32 else torch.bfloat16, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > 126 MB L2

    def step():
        osm.quantize_act(plan, Xd, ac, asc, ah)
        osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y, epi=epi)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()

    n = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(n):
            flush.fill_(float(i))                    # evict L2 between timed steps (untimed)
            ev[i][0].record(stream)
            osm.quantize_act(plan, Xd, ac, asc, ah)
            ev[i][1].record(stream)
            osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y, epi=epi)
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if plan.status() != 0:
        raise RuntimeError("device status reports a timeout during the timed region")
    t_q = np.array([ev[i][0].elapsed_time(ev[i][1]) for i in range(n)]) * 1e-3
    t_g = np.array([ev[i][1].elapsed_time(ev[i][2]) for i in range(n)]) * 1e-3
    t_step = t_q + t_g
    loc = torch.tensor([t_step.mean(), t_g.mean(), t_q.mean()], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(loc, op=dist.ReduceOp.MAX)
    step_s, gemm_s, quant_s = (float(x) for x in loc.cpu())

    # end-to-end through the host entry point: pinned X in, Y out
    Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((M, N), dtype=Y.dtype).pin_memory()
    ws = torch.empty(osm.linear_workspace_size(plan, M, epi), dtype=torch.uint8, device=dev)
    e2e_steps = max(3, min(20, n))
    for _ in range(2):
        osm.linear_host(plan, Xh, M, wc, wsc, wh, Yh, ws, epi=epi)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        osm.linear_host(plan, Xh, M, wc, wsc, wh, Yh, ws, epi=epi)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_t = torch.tensor([e0.elapsed_time(e1) * 1e-3 / e2e_steps], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)
    e2e_s = float(e2e_t.item())

    if rank == 0:
        peaks, peak_src = load_peaks()
        flops = 2.0 * M * N * K
        value = world * flops / step_s / 1e12
        # roofline of the dominant kernel (dual_gemm): bound by the tensor pipe.
        # Peak blended over the two branches at their own dtypes: FP4 = measured
        # BF16 burst x 4 (nominal ratio), BF16 = measured BF16 burst.
        p16 = peaks["bf16_tflops"]
        p4 = p16 * FP4_PER_BF16
        t_ideal = 2.0 * M * N * plan.Kb / (p4 * 1e12) + 2.0 * M * N * plan.k / (p16 * 1e12)
        peak_blend = flops / t_ideal / 1e12
        achieved = flops / gemm_s / 1e12
        cb, sb, hb = plan.sizes(M)
        q_bytes = M * K * 2 + cb + sb + hb
        q_gbs = q_bytes / quant_s / 1e9
        line = {
            "metric": "dual-branch W4A4 GEMM effective TFLOP/s (+act quantize)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": n, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "mxfp4(e2m1,e8m0)+bf16, fp32 accumulate", "data": "synthetic",
            "config": {"workload": cfg.name, "M_per_gpu": M, "K": K, "N": N, "k": cfg.k, "alpha": cfg.alpha,
                       "wscale": {0: "1x32", 1: "32x32", 2: "128x1"}[cfg.wmode],
                       "out": "bf16" if cfg.out_bf16 else "f32",
                       "l2": "flushed between timed steps (256 MiB write, untimed)",
                       "parallelism": f"dp{world} (token shards, no data-path collective)"},
            "pct_fp4_spec_peak": 100.0 * value / world / FP4_SPEC_TFLOPS,
            "kernels": {
                "dual_gemm": {"ms": gemm_s * 1e3, "tflops": achieved,
                              "pct_fp4_spec_peak": 100.0 * achieved / FP4_SPEC_TFLOPS},
                "quantize_act": {"ms": quant_s * 1e3, "gbs": q_gbs, "bytes": q_bytes,
                                 "frac_hbm": q_gbs / peaks["hbm_gbs"]},
            },
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_blend, "unit": "TFLOP/s",
                         "frac": achieved / peak_blend, "traffic": None, "kernel": "dual_gemm",
                         "peak_source": f"{peak_src}: bf16 burst {p16} x4 for the FP4 share, x1 for the "
                                        f"BF16 share (k={plan.k} of K={K})"},
            "e2e": {"value": world * flops / e2e_s / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * Y.element_size(),
                    "api": "osm_linear_host"},
            "gpu_launches": 2 * n,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            tf, t, cores = oracle_sample_throughput(cfg, args.cpu_rows, 2, 1)
            line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                    "sample": f"{args.cpu_rows} of {M} tokens per step (2 steps), weights "
                                              f"packed offline"}
        print(json.dumps(line), flush=True)
    plan.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["up", "down", "long", "tiny"], default="up")
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--ref-rows", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = workloads()[args.workload]

    if args.impl == "reference":
        return run_reference(args, cfg, rank, world)

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_ours(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
