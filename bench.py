"""Benchmark of the smoothed, outlier-split W4A4 linear layer on B200.

One step = one pass of the hot path over one batch of synthetic tokens,
with inputs resident in HBM. Default workload (the largest single-GPU
configuration): four Wan-like FFN blocks of 32760 tokens, each
quantize_act (smooth, split, MXFP4-encode), the up-projection 5120 -> 13824
(block-scaled MXFP4 tcgen05 MMAs + BF16 outlier MMAs into one TMEM
accumulator) with GELU, the down-projection's smoothing and its MXFP4
requantisation fused into the epilogue, then the down-projection
13824 -> 5120 to BF16 -- one osm_ffn_block call per block.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload ffn|up|down|long|tiny|refresh|search|errk]

The single-layer workloads (`up` 4096 x 5120 -> 13824, `down` 32760 x
13824 -> 5120, `long` 75600 x 5120 -> 13824, `tiny`) time quantize_act +
dual_gemm of one layer; `errk` reports the layer's relative error against
the unquantised product for k in {0, 16, 64, 128, 256}.

Multi-GPU: `--gpus N` without a torchrun environment starts N ranks itself
(torch.distributed.run, one rank per GPU, NCCL); tokens are data-parallel,
each rank runs its own batch with no collective on the data path (weak
scaling; calibration statistics are all-reduced with MAX), and the step
time is the max over ranks. `--impl reference` times the CPU oracle (the
only reference implementation of this method) on a bounded sample of the
same workload, on rank 0 only.
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
    return {"up": synth.UP, "down": synth.DOWN, "long": synth.LONG, "tiny": synth.TINY, "ffn": synth.FFN}


METRIC = "dual-branch W4A4 GEMM effective TFLOP/s (+act quantize)"


WSCALE_NAMES = {0: "1x32", 1: "32x32", 2: "128x1"}

# streams that consecutive end-to-end steps rotate over (copies of one step
# overlap the kernels of another)
E2E_STREAMS = 3

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one dual_gemm
# launch, from one ncu capture of the current kernel on the full-size
# workload (one pass), per (workload, kernel); a workload or kernel without a
# capture of the current code reports null.
DUAL_GEMM_TRAFFIC = {
    ("wan_ffn_block_x4_32760x5120x13824", "up_gelu_requant"): 380.74e6,
    ("wan_ffn_block_x4_32760x5120x13824", "down_bf16"): 723.50e6,
    ("wan_ffn_up_4096x5120x13824", "mxfp4"): 292.47e6,
}


def workload_config(cfg):
    if hasattr(cfg, "layers"):
        return {"workload": cfg.name, "layers": cfg.layers, "M": cfg.M, "d_model": cfg.d_model, "d_ff": cfg.d_ff,
                "k_up": cfg.k_up, "k_down": cfg.k_down, "alpha_up": cfg.alpha_up, "alpha_down": cfg.alpha_down,
                "wscale_up": WSCALE_NAMES[cfg.wmode_up], "wscale_down": WSCALE_NAMES[cfg.wmode_down],
                "calib_tokens": cfg.calib_tokens}
    return {"workload": cfg.name, "M": cfg.M, "K": cfg.K, "N": cfg.N, "k": cfg.k, "alpha": cfg.alpha}


def fmt_config(args, cfg):
    """The 4-bit format and weight-scale mode a layer workload runs with."""
    if getattr(args, "nvfp4", False):
        return {"format": "nvfp4", "wscale": "1x16"}
    return {"format": "mxfp4", "wscale": WSCALE_NAMES[cfg.wmode]} if hasattr(cfg, "wmode") else {"format": "mxfp4"}


def blended_peak(peaks, parts, sustained: bool = False):
    """Tensor-pipe peak for a mix of FP4 and BF16 MMAs: parts is a list of
    (fp4_flops, bf16_flops); FP4 runs at the measured BF16 rate x 4 (the
    nominal dense ratio), BF16 at the measured BF16 rate -- the burst rate
    for a kernel timed alone, the sustained (power-capped) rate for a kernel
    timed inside a long step."""
    p16 = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    p4 = p16 * FP4_PER_BF16
    f4 = sum(a for a, _ in parts)
    f16 = sum(b for _, b in parts)
    t_ideal = f4 / (p4 * 1e12) + f16 / (p16 * 1e12)
    return (f4 + f16) / t_ideal / 1e12, p16


# ------------------------------------------------------------------ L2 flush

L2_NOTE = ("flushed between timed steps (untimed): a 256 MiB write, then a 256 MiB read so that the "
           "written lines are evicted before the step")


class L2Flush:
    """Between timed steps: write a 256 MiB buffer (twice the 126 MB L2), then
    read another 256 MiB buffer, so that the step starts with none of its
    inputs in L2 and without dirty lines of the flush still to be written back
    (which would otherwise be charged to the step's first kernel)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def __call__(self, v: float = 1.0):
        self.w.fill_(v)
        self._sink = self.r.sum()


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

def oracle_sample_throughput(cfg, rows_per_step: int, steps: int, warmup: int, nv: bool = False):
    """Time the CPU oracle (quantize_act + dual-branch product, MXFP4 or
    NVFP4) on `rows_per_step` tokens of the workload per step. Weights are
    packed offline, outside the timed region, as on the GPU path."""
    import oracle
    from outlier_split_mixed_b200 import synth
    M_s = rows_per_step * (steps + warmup)
    X = cfg.make_x(min(cfg.M, max(M_s, 256)))
    W = cfg.make_w()
    amax, wmax = oracle.act_amax(X), oracle.weight_amax(W)
    s, inv_s, O = oracle.calibrate(amax, wmax, cfg.alpha, cfg.k)
    if nv:
        ga, gw = oracle.nvfp4_plan_exponents(amax, wmax, s, inv_s, O)
        wc, wsc, wh = oracle.pack_weights_nv(W, s, O, gw)
    else:
        wc, wsc, wh = oracle.pack_weights(W, s, O, cfg.wmode)
    times = []
    for i in range(steps + warmup):
        lo = (i * rows_per_step) % max(1, X.shape[0] - rows_per_step)
        xr = X[lo:lo + rows_per_step]
        t0 = time.perf_counter()
        if nv:
            ac, asc, ah = oracle.quantize_act_nv(xr, inv_s, O, ga)
            oracle.dual_gemm_rows_nv(ac, asc, ah, np.arange(rows_per_step), wc, wsc, wh, ga, gw)
        else:
            ac, asc, ah = oracle.quantize_act(xr, inv_s, O)
            oracle.dual_gemm_rows(ac, asc, ah, np.arange(rows_per_step), wc, wsc, wh)
        t1 = time.perf_counter()
        if i >= warmup:
            times.append(t1 - t0)
    t = float(np.mean(times))
    flops = 2.0 * rows_per_step * cfg.N * cfg.K
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return flops / t / 1e12, t, cores


def oracle_ffn_throughput(cfg, rows_per_step: int, steps: int, warmup: int, calib_rows: int = 64):
    """Time the CPU oracle on the FFN chain: per block quantize (up),
    dual-branch product, GELU to BF16, quantize (down), dual-branch product,
    on `rows_per_step` tokens per block per step. Calibration (on the first
    `calib_rows` tokens of each block's calibration batch; down-projection
    statistics from the unquantised GELU(X W_up)) and weight packing are
    offline, outside the timed region."""
    import oracle
    preps = []
    for l in range(cfg.layers):
        Xc = cfg.make_calib(l)[:calib_rows]
        Wu, Wd = cfg.make_w_up(l), cfg.make_w_down(l)
        s_u, inv_u, O_u = oracle.calibrate(oracle.act_amax(Xc), oracle.weight_amax(Wu), cfg.alpha_up, cfg.k_up)
        allc = np.arange(cfg.d_model, dtype=np.int32)
        ones = np.ones(cfg.d_model, np.float32)
        fa = oracle.quantize_act(Xc, ones, allc)
        fw = oracle.pack_weights(Wu, ones, allc, cfg.wmode_up)
        y, _ = oracle.dual_gemm_rows(*fa, np.arange(Xc.shape[0]), *fw)
        Hc = oracle.gelu_bf16(y)
        s_d, inv_d, O_d = oracle.calibrate(oracle.act_amax(Hc), oracle.weight_amax(Wd), cfg.alpha_down, cfg.k_down)
        preps.append(dict(inv_u=inv_u, O_u=O_u, wu=oracle.pack_weights(Wu, s_u, O_u, cfg.wmode_up),
                          inv_d=inv_d, O_d=O_d, wd=oracle.pack_weights(Wd, s_d, O_d, cfg.wmode_down),
                          X=cfg.make_x(l, max(256, rows_per_step * (steps + warmup)))))
    times = []
    r = np.arange(rows_per_step)
    for i in range(steps + warmup):
        t0 = time.perf_counter()
        for pr in preps:
            lo = (i * rows_per_step) % max(1, pr["X"].shape[0] - rows_per_step)
            a = oracle.quantize_act(pr["X"][lo:lo + rows_per_step], pr["inv_u"], pr["O_u"])
            y, _ = oracle.dual_gemm_rows(*a, r, *pr["wu"])
            h = oracle.gelu_bf16(y)
            a2 = oracle.quantize_act(h, pr["inv_d"], pr["O_d"])
            oracle.dual_gemm_rows(*a2, r, *pr["wd"])
        t1 = time.perf_counter()
        if i >= warmup:
            times.append(t1 - t0)
    t = float(np.mean(times))
    flops = cfg.layers * 2.0 * 2.0 * rows_per_step * cfg.d_model * cfg.d_ff
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return flops / t / 1e12, t, cores


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return 0
    is_ffn = hasattr(cfg, "layers")
    rows = max(1, args.ref_rows if not is_ffn else max(1, args.ref_rows // 8))
    if is_ffn:
        tflops, t, cores = oracle_ffn_throughput(cfg, rows, args.steps, args.warmup)
    else:
        tflops, t, cores = oracle_sample_throughput(cfg, rows, args.steps, args.warmup, nv=args.nvfp4)
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (oracle)", "data": "synthetic",
        "config": dict(workload_config(cfg), sample_rows_per_step=rows, **fmt_config(args, cfg)),
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
    plan = osm.Plan(K, N, cfg.k, s, O, osm.WSCALE_1x32 if args.nvfp4 else cfg.wmode, hp_fp16=args.hp_fp16)
    if args.nvfp4:
        plan.set_format(osm.FMT_NVFP4, *odist.nvfp4_exponents_from_local_stats(amax, wmax, s, inv_s, O))
    wc, wsc, wh = plan.alloc_packed(N, dev)
    osm.pack_weights(plan, Wd, wc, wsc, wh)
    ac, asc, ah = plan.alloc_packed(M, dev)
    Y = torch.empty((M, N), dtype=torch.float32 if epi == osm.EPI_F32 else torch.bfloat16, device=dev)
    flush = L2Flush(dev)

    def step():
        osm.quantize_act(plan, Xd, ac, asc, ah)
        osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y, epi=epi)

    for _ in range(args.warmup):
        flush(1.0)
        step()
    torch.cuda.synchronize()

    # The timed region: K steps with events at the step boundaries only (an
    # event between the two kernels would stop dual_gemm's dependent launch
    # from overlapping quantize_act's tail). The kernel split comes from the
    # same K steps run again with an event between the kernels.
    n = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(n):
            flush(float(i))                          # evict L2 between timed steps (untimed)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        for i in range(n):
            flush(float(i))
            evs[i][0].record(stream)
            osm.quantize_act(plan, Xd, ac, asc, ah)
            evs[i][1].record(stream)
            osm.dual_gemm(plan, ac, asc, ah, M, wc, wsc, wh, Y, epi=epi)
            evs[i][2].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if plan.status() != 0:
        raise RuntimeError("device status reports a timeout during the timed region")
    t_step = np.array([ev[i][0].elapsed_time(ev[i][1]) for i in range(n)]) * 1e-3
    t_q = np.array([evs[i][0].elapsed_time(evs[i][1]) for i in range(n)]) * 1e-3
    t_g = np.array([evs[i][1].elapsed_time(evs[i][2]) for i in range(n)]) * 1e-3
    loc = torch.tensor([t_step.mean(), t_g.mean(), t_q.mean()], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(loc, op=dist.ReduceOp.MAX)
    step_s, gemm_s, quant_s = (float(x) for x in loc.cpu())

    # end-to-end through the host entry point: pinned X in, Y out, every
    # step. Consecutive steps rotate over E2E_STREAMS streams (each with its
    # own workspace and host Y), so one step's copy in, another's kernels
    # and a third's copy out overlap, as a serving loop would run them.
    Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
    streams = [torch.cuda.Stream(device=dev) for _ in range(E2E_STREAMS)]
    Yhs = [torch.empty((M, N), dtype=Y.dtype).pin_memory() for _ in streams]
    wss = [torch.empty(osm.linear_workspace_size(plan, M, epi), dtype=torch.uint8, device=dev) for _ in streams]
    e2e_steps = max(3 * E2E_STREAMS, min(24, n))
    for j in range(E2E_STREAMS):
        osm.linear_host(plan, Xh, M, wc, wsc, wh, Yhs[j], wss[j], epi=epi, stream=streams[j])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for st in streams:
        st.wait_event(e0)
    for i in range(e2e_steps):
        j = i % E2E_STREAMS
        osm.linear_host(plan, Xh, M, wc, wsc, wh, Yhs[j], wss[j], epi=epi, stream=streams[j])
    for st in streams:
        stream.wait_stream(st)
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
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": n, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("nvfp4(e2m1,ue4m3 per 16,2^g per tensor)" if args.nvfp4 else "mxfp4(e2m1,e8m0)")
                     + "+bf16, fp32 accumulate", "data": "synthetic",
            "config": {"workload": cfg.name, "M_per_gpu": M, "K": K, "N": N, "k": cfg.k, "alpha": cfg.alpha,
                       **fmt_config(args, cfg), "g": [plan.g_act, plan.g_w] if args.nvfp4 else None,
                       "out": "bf16" if cfg.out_bf16 else "f32",
                       "outlier_branch": "fp16" if args.hp_fp16 else "bf16",
                       "l2": L2_NOTE,
                       "parallelism": f"dp{world} (token shards, no data-path collective)"},
            "pct_fp4_spec_peak": 100.0 * value / world / FP4_SPEC_TFLOPS,
            "kernels": {
                "dual_gemm": {"ms": gemm_s * 1e3, "tflops": achieved,
                              "pct_fp4_spec_peak": 100.0 * achieved / FP4_SPEC_TFLOPS},
                "quantize_act": {"ms": quant_s * 1e3, "gbs": q_gbs, "bytes": q_bytes,
                                 "frac_hbm": q_gbs / peaks["hbm_gbs"]},
            },
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_blend, "unit": "TFLOP/s",
                         "frac": achieved / peak_blend,
                         "traffic": None if args.hp_fp16 else DUAL_GEMM_TRAFFIC.get((cfg.name,
                                                                                    fmt_config(args, cfg)["format"])),
                         "traffic_unit": "bytes per launch", "kernel": "dual_gemm",
                         "pct_fp4_spec_peak": 100.0 * achieved / FP4_SPEC_TFLOPS,
                         "peak_source": f"derived from {peak_src} peaks: BF16 burst {p16} TFLOP/s x4 (nominal "
                                        f"FP4:BF16 dense ratio) for the FP4 share, x1 for the BF16 share "
                                        f"(k={plan.k} of K={K}); FP4 itself is not measured"},
            "e2e": {"value": world * flops / e2e_s / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * Y.element_size(),
                    "api": f"osm_linear_host, steps rotated over {E2E_STREAMS} streams"},
            "gpu_launches": 2 * n,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            tf, t, cores = oracle_sample_throughput(cfg, args.cpu_rows, 2, 1, nv=args.nvfp4)
            line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                    "sample": f"{args.cpu_rows} of {M} tokens per step (2 steps), weights "
                                              f"packed offline"}
        print(json.dumps(line), flush=True)
    plan.close()
    return 0


def run_ffn(args, cfg, rank, world, local_rank):
    """Four FFN blocks on one stream, each one call of osm_ffn_block:
    quantize_act of the block input for the up-projection; dual_gemm up with
    the fused GELU + smoothing + MXFP4 requantisation epilogue, writing the
    down-projection's packed activations; dual_gemm down to BF16."""
    import torch
    import torch.distributed as dist

    import outlier_split_mixed_b200 as osm
    from outlier_split_mixed_b200 import dist as odist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    M, D, F = cfg.M, cfg.d_model, cfg.d_ff

    def to_dev(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    blocks = []
    for l in range(cfg.layers):
        Xc, Wu, Wd = to_dev(cfg.make_calib(l)), to_dev(cfg.make_w_up(l)), to_dev(cfg.make_w_down(l))
        # up-projection statistics
        amax = torch.zeros(D, dtype=torch.float32, device=dev)
        wmax = torch.empty(D, dtype=torch.float32, device=dev)
        osm.act_amax_accumulate(Xc, amax)
        osm.weight_amax(Wu, wmax)
        s_u, _, O_u = odist.calibrate_from_local_stats(amax, wmax, cfg.alpha_up, cfg.k_up)
        # down-projection statistics from the unquantised GELU(Xc W_up): k = K, s = 1
        full = osm.Plan(D, F, D, np.ones(D, np.float32), np.arange(D, dtype=np.int32), cfg.wmode_up)
        fa = full.alloc_packed(Xc.shape[0], dev)
        fw = full.alloc_packed(F, dev)
        osm.quantize_act(full, Xc, *fa)
        osm.pack_weights(full, Wu, *fw)
        Hc = torch.empty((Xc.shape[0], F), dtype=torch.bfloat16, device=dev)
        osm.dual_gemm(full, *fa, Xc.shape[0], *fw, Hc, epi=osm.EPI_GELU_BF16)
        amax_d = torch.zeros(F, dtype=torch.float32, device=dev)
        wmax_d = torch.empty(F, dtype=torch.float32, device=dev)
        osm.act_amax_accumulate(Hc, amax_d)
        osm.weight_amax(Wd, wmax_d)
        s_d, _, O_d = odist.calibrate_from_local_stats(amax_d, wmax_d, cfg.alpha_down, cfg.k_down)
        full.close()
        del fa, fw, Hc
        up = osm.Plan(D, F, cfg.k_up, s_u, O_u, cfg.wmode_up, hp_fp16=args.hp_fp16)
        down = osm.Plan(F, D, cfg.k_down, s_d, O_d, cfg.wmode_down, hp_fp16=args.hp_fp16)
        wu = up.alloc_packed(F, dev)
        osm.pack_weights_for_next(up, down, Wu, *wu)
        wd = down.alloc_packed(D, dev)
        osm.pack_weights(down, Wd, *wd)
        del Wu, Wd, Xc
        blocks.append(dict(up=up, down=down, wu=wu, wd=wd, X=cfg.make_x(l)))
    # the device workspace (both layers' packed activations) is shared by the
    # blocks, which run one after another; each block has its own input and output
    ws = torch.empty(max(osm.ffn_workspace_size(b["up"], b["down"], M) for b in blocks), dtype=torch.uint8,
                     device=dev)
    for b in blocks:
        b["Xd"] = to_dev(b["X"])
        b["Y"] = torch.empty((M, D), dtype=torch.bfloat16, device=dev)
    # the same buffers split per kernel, for the pass with events between kernels
    a_up = blocks[0]["up"].alloc_packed(M, dev)
    a_dn = blocks[0]["down"].alloc_packed(M, dev)
    flush = L2Flush(dev)

    def block(b):
        osm.ffn_block(b["up"], b["down"], b["Xd"], b["wu"], b["wd"], b["Y"], ws)

    def block_split(b, ev):
        ev[0].record(stream)
        osm.quantize_act(b["up"], b["Xd"], *a_up)
        ev[1].record(stream)
        osm.dual_gemm(b["up"], *a_up, M, *b["wu"], None, epi=osm.EPI_GELU_REQUANT, next_plan=b["down"],
                      next_buffers=a_dn)
        ev[2].record(stream)
        osm.dual_gemm(b["down"], *a_dn, M, *b["wd"], b["Y"], epi=osm.EPI_BF16)
        ev[3].record(stream)

    for _ in range(args.warmup):
        flush(1.0)
        for b in blocks:
            block(b)
    torch.cuda.synchronize()

    # The timed region: K steps of the four blocks with events at the step
    # boundaries only (events between kernels would stop each dual_gemm's
    # dependent launch); the kernel split comes from the same K steps run
    # again with events between the kernels.
    n = args.steps
    L = cfg.layers
    evt = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(L)] for _ in range(n)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(n):
            flush(float(i))                          # evict L2 between timed steps (untimed)
            evt[i][0].record(stream)
            for b in blocks:
                block(b)
            evt[i][1].record(stream)
        torch.cuda.synchronize()
        for i in range(n):
            flush(float(i))
            for l, b in enumerate(blocks):
                block_split(b, ev[i][l])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    for b in blocks:
        if b["up"].status() != 0 or b["down"].status() != 0:
            raise RuntimeError("device status reports a timeout during the timed region")
    t = np.array([[[ev[i][l][j].elapsed_time(ev[i][l][j + 1]) * 1e-3 for j in range(3)] for l in range(L)]
                  for i in range(n)])  # [step][block][quantize, up, down]
    t_step = np.array([evt[i][0].elapsed_time(evt[i][1]) * 1e-3 for i in range(n)])
    loc = torch.tensor([t_step.mean(), t[:, :, 0].sum(1).mean(), t[:, :, 1].sum(1).mean(), t[:, :, 2].sum(1).mean()],
                       dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(loc, op=dist.ReduceOp.MAX)
    step_s, quant_s, up_s, down_s = (float(x) for x in loc.cpu())

    # End to end through the host entry point osm_ffn_block_host: every block
    # input copied in from pinned host memory and every block output copied
    # out, inside the timed region. Each block runs on its own stream with its
    # own device workspace, so one block's copies overlap another's kernels.
    Xh = [torch.from_numpy(b["X"].view(np.int16)).view(torch.bfloat16).pin_memory() for b in blocks]
    Yh = [torch.empty((M, D), dtype=torch.bfloat16).pin_memory() for _ in blocks]
    streams = [torch.cuda.Stream(device=dev) for _ in blocks]
    wss = [torch.empty(osm.ffn_host_workspace_size(b["up"], b["down"], M), dtype=torch.uint8, device=dev)
           for b in blocks]

    def e2e_step():
        for b, xh, yh, st, w in zip(blocks, Xh, Yh, streams, wss):
            osm.ffn_block_host(b["up"], b["down"], xh, b["wu"], b["wd"], yh, w, stream=st)

    e2e_steps = max(3, min(10, n))
    e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for st in streams:
        st.wait_event(e0)
    for _ in range(e2e_steps):
        e2e_step()
    for st in streams:
        stream.wait_stream(st)
    e1.record(stream)
    torch.cuda.synchronize()
    for b in blocks:
        if b["up"].status() != 0 or b["down"].status() != 0:
            raise RuntimeError("device status reports a timeout during the end-to-end region")
    e2e_t = torch.tensor([e0.elapsed_time(e1) * 1e-3 / e2e_steps], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)
    e2e_s = float(e2e_t.item())
    del wss

    if rank == 0:
        peaks, peak_src = load_peaks()
        flops = cfg.flops
        value = world * flops / step_s / 1e12
        up0, dn0 = blocks[0]["up"], blocks[0]["down"]
        f_up = L * 2.0 * M * F * D
        f_dn = L * 2.0 * M * D * F
        # the dominant kernel: the up-projection with the fused epilogue
        # the kernels run back to back for the whole ~10 ms step (and the
        # clocks settle under the power cap), so the sustained BF16 rate sets
        # the peak
        peak_up, p16 = blended_peak(peaks, [(2.0 * M * F * up0.Kb, 2.0 * M * F * up0.k)], sustained=True)
        peak_dn, _ = blended_peak(peaks, [(2.0 * M * D * dn0.Kb, 2.0 * M * D * dn0.k)], sustained=True)
        ach_up = f_up / up_s / 1e12
        ach_dn = f_dn / down_s / 1e12
        cb, sb, hb = up0.sizes(M)
        q_bytes = L * (M * D * 2 + cb + sb + hb)
        traffic = None if args.hp_fp16 else DUAL_GEMM_TRAFFIC.get((cfg.name, "up_gelu_requant"))
        # algorithmic bytes of one launch: packed activations in, packed weights, output out
        cd_, sd_, hd_ = dn0.sizes(M)
        cwu, swu, hwu = up0.sizes(F)
        cwd, swd, hwd = dn0.sizes(D)
        alg_up = (cb + sb + hb) + (cwu + swu + hwu) + (cd_ + sd_ + hd_)
        alg_dn = (cd_ + sd_ + hd_) + (cwd + swd + hwd) + M * D * 2
        line = {
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": n, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "mxfp4(e2m1,e8m0)+bf16, fp32 accumulate", "data": "synthetic",
            "config": dict(workload_config(cfg), l2=L2_NOTE,
                           parallelism=f"dp{world} (token shards, no data-path collective)",
                           outlier_branch="fp16" if args.hp_fp16 else "bf16",
                           step="osm_ffn_block per block (quantize_act, up with fused GELU requant, down to BF16)"),
            "pct_fp4_spec_peak": 100.0 * value / world / FP4_SPEC_TFLOPS,
            "kernels": {
                "dual_gemm_up_gelu_requant": {"ms": up_s * 1e3, "tflops": ach_up, "frac": ach_up / peak_up,
                                              "pct_fp4_spec_peak": 100.0 * ach_up / FP4_SPEC_TFLOPS},
                "dual_gemm_down_bf16": {"ms": down_s * 1e3, "tflops": ach_dn, "frac": ach_dn / peak_dn,
                                        "pct_fp4_spec_peak": 100.0 * ach_dn / FP4_SPEC_TFLOPS,
                                        "traffic": None if args.hp_fp16 else
                                        DUAL_GEMM_TRAFFIC.get((cfg.name, "down_bf16")),
                                        "algorithmic_bytes": alg_dn},
                "quantize_act": {"ms": quant_s * 1e3, "gbs": q_bytes / quant_s / 1e9, "bytes": q_bytes,
                                 "frac_hbm": q_bytes / quant_s / 1e9 / peaks["hbm_gbs"]},
            },
            "roofline": {"bound": "tensor", "achieved": ach_up, "peak": peak_up, "unit": "TFLOP/s",
                         "frac": ach_up / peak_up, "traffic": traffic, "traffic_unit": "bytes per launch",
                         "algorithmic_bytes": alg_up,
                         "kernel": "dual_gemm up-projection, fused GELU + smoothing + MXFP4 requantisation",
                         "pct_fp4_spec_peak": 100.0 * ach_up / FP4_SPEC_TFLOPS,
                         "peak_source": f"derived from {peak_src} peaks: sustained BF16 {p16} TFLOP/s x4 "
                                        f"(nominal FP4:BF16 dense ratio) for the FP4 share, x1 for the BF16 share "
                                        f"(k={up0.k} of K={D}); FP4 itself is not measured"},
            "e2e": {"value": world * flops / e2e_s / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": L * M * D * 2, "d2h_bytes_per_step": L * M * D * 2,
                    "copies_declared": True,
                    "api": "osm_ffn_block_host per block (pinned X in, Y out); each block on its own stream"},
            "gpu_launches": 3 * L * n,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            rows = max(1, args.cpu_rows // 4)
            tf, t1, cores = oracle_ffn_throughput(cfg, rows, 2, 1)
            line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                    "sample": f"{rows} of {M} tokens per block per step (2 steps), calibration "
                                              f"on 64 tokens, weights packed offline"}
        print(json.dumps(line), flush=True)
    for b in blocks:
        b["up"].close()
        b["down"].close()
    return 0


def run_refresh(args, cfg, rank, world, local_rank):
    """Dynamic outlier set: one step re-calibrates the layer on the device
    from the current batch (activation maxima, osm_plan_refresh) and packs
    the weights again for the new s and O; inputs resident in HBM."""
    import torch
    import outlier_split_mixed_b200 as osm

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    M, K, N = cfg.M, cfg.K, cfg.N
    X, W = cfg.make_x(), cfg.make_w()
    Xd = torch.from_numpy(X.view(np.int16)).to(dev).view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
    wmax = torch.empty(K, dtype=torch.float32, device=dev)
    osm.weight_amax(Wd, wmax)
    amax = torch.zeros(K, dtype=torch.float32, device=dev)
    plan = osm.Plan(K, N, cfg.k, np.ones(K, np.float32), np.arange(cfg.k, dtype=np.int32), cfg.wmode)
    wc, wsc, wh = plan.alloc_packed(N, dev)
    flush = L2Flush(dev)

    score = torch.empty(K, dtype=torch.float32, device=dev) if args.percentile else None

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        amax.zero_()
        osm.act_amax_accumulate(Xd, amax)
        if score is not None:
            osm.act_percentile(Xd, args.percentile, score)
        if ev is not None:
            ev[1].record(stream)
        if score is not None:
            plan.refresh_scored(amax, score, wmax, cfg.alpha)
        else:
            plan.refresh(amax, wmax, cfg.alpha)
        if ev is not None:
            ev[2].record(stream)
        osm.pack_weights(plan, Wd, wc, wsc, wh)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        flush(1.0)
        step()
    torch.cuda.synchronize()
    n = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    with ClockSampler(local_rank) as clk:
        for i in range(n):
            flush(float(i))
            step(ev[i])
        torch.cuda.synchronize()
    if plan.status() != 0:
        raise RuntimeError("plan status reports an error")
    t = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) * 1e-3 for j in range(3)] for i in range(n)]).mean(0)
    step_s = float(t.sum())
    if rank == 0:
        peaks, _ = load_peaks()
        cb, sb, hb = plan.sizes(N)
        pack_bytes = K * N * 2 + cb + sb + hb
        line = {
            "metric": "dynamic re-calibration time per step (activation statistics + plan refresh + weight repack)",
            "value": step_s * 1e6, "unit": "us", "n_gpus": world, "steps": n, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 in, mxfp4+bf16 out", "data": "synthetic",
            "config": dict(workload_config(cfg), l2=L2_NOTE,
                           channel_score=f"percentile {args.percentile}" if args.percentile else "maximum"),
            "kernels": {
                "act_stats": {"us": t[0] * 1e6, "gbs": M * K * 2 * (2 if args.percentile else 1) / t[0] / 1e9},
                "plan_refresh": {"us": t[1] * 1e6},
                "pack_weights": {"us": t[2] * 1e6, "gbs": pack_bytes / t[2] / 1e9, "bytes": pack_bytes,
                                 "frac_hbm": pack_bytes / t[2] / 1e9 / peaks["hbm_gbs"]},
            },
            "gpu_launches": 4 * n,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    plan.close()
    return 0


def run_search(args, cfg, rank, world, local_rank):
    """Per-layer alpha / k search on a calibration batch: wall time per
    candidate (host calibration and plan, device pack + quantize + GEMM +
    error norms) over a 4 x 4 grid."""
    import torch
    from outlier_split_mixed_b200.search import search_alpha_k

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    T = min(cfg.M, 2048)
    X = cfg.make_x(T)
    Xd = torch.from_numpy(X.view(np.int16)).to(dev).view(torch.bfloat16)
    Wd = torch.from_numpy(cfg.make_w().view(np.int16)).to(dev).view(torch.bfloat16)
    alphas, ks = [0.4, 0.5, 0.6, 0.7], [0, 64, 128, 256]
    search_alpha_k(Xd, Wd, alphas[:1], ks[:1], wmode=cfg.wmode)  # warm-up
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    r = search_alpha_k(Xd, Wd, alphas, ks, wmode=cfg.wmode)
    torch.cuda.synchronize()
    t = (time.perf_counter() - t0) / len(r.table)
    if rank == 0:
        line = {
            "metric": "per-layer alpha/k search time per candidate (wall clock)",
            "value": t * 1e3, "unit": "ms", "n_gpus": 1, "steps": len(r.table), "warmup": 1,
            "ms_per_step": t * 1e3, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 in, mxfp4+bf16 path, fp64 error norms", "data": "synthetic",
            "config": dict(workload_config(cfg), calibration_tokens=T, alphas=alphas, ks=ks),
            "best": {"alpha": r.alpha, "k": r.k, "rel_err": r.rel_err},
            "table": [{"alpha": a, "k": k, "rel_err": e} for a, k, e in r.table],
        }
        print(json.dumps(line), flush=True)
    return 0


def run_errk(args, cfg, rank, world, local_rank):
    """The paper's Eq. (5) argument measured on the CUDA path: relative
    Frobenius error of the layer output against the unquantised product of
    the same BF16 operands (PyTorch FP32 matmul) for k in {0, 16, 64, 128,
    256} outlier channels, on the layer workload's synthetic batch."""
    import torch
    import outlier_split_mixed_b200 as osm

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    X, W = cfg.make_x(), cfg.make_w()
    Xd = torch.from_numpy(X.view(np.int16)).to(dev).view(torch.bfloat16)
    Wd = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
    ref = Xd.float() @ Wd.float()
    table = []
    for k in (0, 16, 64, 128, 256):
        s, _, O, _, _ = osm.calibrate([Xd], Wd, cfg.alpha, k)
        plan = osm.Plan(cfg.K, cfg.N, k, s, O, cfg.wmode)
        wc, wsc, wh = plan.alloc_packed(cfg.N, dev)
        osm.pack_weights(plan, Wd, wc, wsc, wh)
        ac, asc, ah = plan.alloc_packed(cfg.M, dev)
        osm.quantize_act(plan, Xd, ac, asc, ah)
        Y = torch.empty((cfg.M, cfg.N), dtype=torch.float32, device=dev)
        osm.dual_gemm(plan, ac, asc, ah, cfg.M, wc, wsc, wh, Y)
        e, nrm = osm.error_norms(Y, ref)
        if plan.status() != 0:
            raise RuntimeError("plan status reports an error")
        plan.close()
        table.append({"k": k, "rel_err": float(np.sqrt(e / nrm))})
    if rank == 0:
        rel = [r["rel_err"] for r in table]
        line = {
            "metric": "relative Frobenius error of Y against the unquantised FP32 XW, by outlier count k",
            "value": rel[-1], "unit": "relative error at k=256", "n_gpus": 1, "steps": len(table), "warmup": 0,
            "higher_is_better": False, "vs_baseline": None, "dtype": "mxfp4(e2m1,e8m0)+bf16, fp32 accumulate",
            "data": "synthetic", "config": dict(workload_config(cfg), wscale=WSCALE_NAMES[cfg.wmode]),
            "error_vs_k": table,
            "falls_monotonically": all(b <= a for a, b in zip(rel, rel[1:])),
        }
        print(json.dumps(line), flush=True)
    return 0


def relaunch_ranks(n: int) -> int:
    """Start n ranks of this same command under torch.distributed.run (one
    process per GPU, rendezvous on 127.0.0.1) and return its exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["ffn", "up", "down", "long", "tiny", "refresh", "search", "errk"],
                    default="ffn")
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--ref-rows", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (small cases for profiler captures)")
    ap.add_argument("--blocks", type=int, default=0, help="override the number of FFN blocks (ffn workload)")
    ap.add_argument("--hp-fp16", action="store_true", help="outlier branch in FP16 instead of BF16")
    ap.add_argument("--nvfp4", action="store_true",
                    help="layer workloads: NVFP4 bulk format (16-blocks, UE4M3 scales) instead of MXFP4")
    ap.add_argument("--percentile", type=float, default=0.0,
                    help="refresh workload: score channels by this percentile of |x| (0: by the maximum)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.nvfp4 and (args.workload in ("ffn", "refresh", "search") or args.hp_fp16):
        ap.error("--nvfp4 applies to the layer workloads (up, down, long, tiny) with the BF16 outlier branch")

    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return relaunch_ranks(args.gpus)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started {world} ranks")
    cfg = workloads()[args.workload if args.workload not in ("refresh", "search", "errk") else "up"]
    if args.tokens or args.blocks:
        import dataclasses
        changes = {}
        if args.tokens:
            changes["M"] = args.tokens
        if args.blocks and hasattr(cfg, "layers"):
            changes["layers"] = args.blocks
        changes["name"] = cfg.name + "".join(f"_{k}{v}" for k, v in sorted(changes.items()))
        cfg = dataclasses.replace(cfg, **changes)

    if args.impl == "reference":
        return run_reference(args, cfg, rank, world)

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.workload == "ffn":
            return run_ffn(args, cfg, rank, world, local_rank)
        if args.workload == "refresh":
            return run_refresh(args, cfg, rank, world, local_rank)
        if args.workload == "search":
            return run_search(args, cfg, rank, world, local_rank)
        if args.workload == "errk":
            return run_errk(args, cfg, rank, world, local_rank)
        return run_ours(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
