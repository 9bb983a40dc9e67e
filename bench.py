#!/usr/bin/env python
"""Benchmark of the QLoRA hot path on B200: NF4 + DQ quantize, standalone dequant, fused
QLoRA linear forward + backward.

One step = the whole path over one batch of synthetic input for the seven linears of a
LLaMA-13B decoder block (q, k, v, o 5120x5120; gate, up 13824x5120; down 5120x13824), 8192
tokens per GPU, LoRA r = 64, alpha = 16: for each linear, quantize its bf16 weight (absmax,
nearest NF4 level, packing, double quantization), dequantize it to bf16 (the standalone HBM
stream), then the fused forward and the backward (dX, dA, dB).  With N > 1 GPUs each rank
runs its own 8192-token batch (data parallel, weak scaling) and the adapter gradients are
summed across ranks with NCCL after each backward.

value = algorithmic fwd+bwd flops of all ranks (4MNK + 6MKr + 6MNr per linear) / step time
(max over ranks), so quantize and dequant time count against it.  Per-row rates, the
roofline of the dominant kernel (timed live with CUDA events around its launches), the CPU
oracle baseline, an end-to-end run through host buffers and the SM clocks seen during the
timed region are reported on the same JSON line.

Extra rows on the same line (rank 0, one GPU): the LLaMA-7B block at 512 tokens, the
quantize / dequant sweep over the 80-layer 65B-shaped stack (bytes per weight, GB/s), and the
robust 4000x3000 weight over ranks r in {8, 64, 256} and token counts M in {1, 16, 512, 16384}
(with the HBM roofline where M <= 16).

--gpus N (N > 1) without a launcher re-executes itself under torch.distributed.run with N
ranks on this node; under a launcher the world size must equal N.
--impl reference times the CPU oracle (oracle/) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4 dequant GB/s, % of B200 roofline"
WORKLOAD = "llama13b_block_8192tok"
R = 64
ALPHA = 16.0
M_TOKENS = 8192
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Algorithmic bytes per weight: quantize reads bf16 (2 B) and writes codes (0.5 B), scale
# codes (1/64 B) and group constants (4/(64*256) B); dequant reads the latter and writes bf16.
CODEC_BYTES_PER_WEIGHT = 2.0 + 0.5 + 1.0 / 64 + 4.0 / (64 * 256)
# float64 fused multiply-add peak of one B200, derived from unit counts and clock: 148 SMs x 64
# float64 FMA per cycle per SM (ncu's peak_sustained for sm__sass_thread_inst_executed_op_dfma)
# x 2 flops x 1.965 GHz (clocks.max.sm).  No measured figure exists for it.
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12
# kernels one nf4_quantize_dq call launches
QUANTIZE_LAUNCHES = 2


def linears():
    import synth
    return synth.LLAMA13B


def linear_flops(M, N, K, r):
    return 4 * M * N * K + 6 * M * K * r + 6 * M * N * r


def step_flops(M=M_TOKENS, r=R):
    return sum(linear_flops(M, l.N, l.K, r) for l in linears())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def pick_bf16_peak(peaks: dict, clocks: dict):
    """The bf16 tensor peak a kernel timed in this run is measured against.

    MEASURED_PEAKS.json holds a burst figure (a short matmul at full clock) and a sustained
    one (a seconds-long loop that settles under the power cap at a lower clock).  The peak
    that applies is the one whose clock the timed region actually ran at: the burst figure
    when the median SM clock sampled during the timed region is within 10 % of the maximum
    (or was not sampled), else the sustained figure."""
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm is None or not smax or sm >= 0.9 * smax:
        return peaks["bf16_tflops"], "burst"
    return peaks["bf16_tflops_sustained"], "sustained"


# ------------------------------------------------------------------------------------------
# DRAM traffic of the fused GEMMs
# ------------------------------------------------------------------------------------------
# Bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum), averaged over the 14 launches
# of the two timed steps, from one single-pass capture of this script's own run:
#   ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum
#       --clock-control none -k regex:"qlora_gemm|nf4_quant_stream|dq_mean|nf4_dequant|lowrank" -c 189
#       python bench.py --steps 2 --warmup 1 --no-e2e --no-cpu-baseline --no-extra
# They hold only for the kernel sources they were taken on: once any of FUSED_SOURCES changes
# the traffic is reported as null.
FUSED_SOURCES = ("gemm.cuh", "gemm.h", "common.cuh", "nf4_device.cuh", "qlora_nf4.cu")
FUSED_TRAFFIC = {"sources_sha256": "68512cc91b958081e192f4913f8c2c36b265cf18605a62b42be2d733325411d6",
                 "fwd": 285568603, "dx": 311298395}


def fused_traffic(which: str):
    import hashlib
    csrc = os.path.join(ROOT, "bit_nf4_quantized_dq_b200", "csrc")
    h = hashlib.sha256()
    for f in FUSED_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return FUSED_TRAFFIC[which] if h.hexdigest() == FUSED_TRAFFIC["sources_sha256"] else None


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    smax.append(float(p[2]))
                except ValueError:
                    continue
                for n, v in zip(names, p[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


class NvmlClockSampler:
    """SM clock and clock-event reasons every `period_s` through NVML, in a background thread
    (nvidia-smi needs over 100 ms before its first sample, longer than a short timed region).
    The device is found by its PCI bus id; falls back to ClockSampler when NVML is missing."""
    BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, torch_device_index: int, period_s: float = 0.005):
        self.idx = torch_device_index
        self.period = period_s
        self.fallback = None
        self.samples = []
        self.thread = None
        self.stop_flag = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.idx)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            dev = getattr(props, "pci_device_id", 0)
            return pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0".encode())
        return pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def start(self):
        import threading
        try:
            import pynvml
            h = self._handle()
            reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.fallback = ClockSampler(self.idx)
            self.fallback.start()
            return
        self.stop_flag = threading.Event()

        def run():
            while not self.stop_flag.is_set():
                try:
                    self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), reasons_fn(h)))
                except Exception:
                    pass
                self.stop_flag.wait(self.period)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self) -> dict:
        if self.fallback is not None:
            return self.fallback.stop()
        self.stop_flag.set()
        self.thread.join(timeout=5)
        sm = [float(c) for c, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, b in self.BITS.items() if r & b})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": float(self.smax),
                "reasons": reasons, "samples": len(sm), "source": "nvml"}


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------
class LinearBufs:
    """Device buffers of one linear, preallocated so the timed region allocates nothing."""

    def __init__(self, lin, M, r, seed, dev):
        import torch
        import synth
        import bit_nf4_quantized_dq_b200 as q
        self.N, self.K, self.M, self.r = lin.N, lin.K, M, r
        self.s = ALPHA / r
        self.W = synth.normal_bf16((lin.N, lin.K), 0.02, seed, device=dev)
        inp = synth.linear_inputs(M, lin.N, lin.K, r, seed, device=dev)
        self.x, self.A, self.B, self.dY = inp["x"], inp["A"], inp["B"], inp["dY"]
        numel = lin.N * lin.K
        nb = (numel + 63) // 64
        ng = (nb + 255) // 256
        u8, f32, bf = torch.uint8, torch.float32, torch.bfloat16
        self.Q = q.NF4Tensor(torch.empty(32 * nb, dtype=u8, device=dev), torch.empty(nb, dtype=u8, device=dev),
                             torch.empty(ng, dtype=f32, device=dev), torch.empty(1, dtype=f32, device=dev),
                             (lin.N, lin.K))
        L = q.lib()
        self.ws_q = torch.empty(L.nf4_quantize_workspace_bytes(numel), dtype=u8, device=dev)
        self.ws_f = torch.empty(max(256, L.qlora_linear_fwd_workspace_bytes(M, lin.K, lin.N, r)), dtype=u8,
                                device=dev)
        self.ws_b = torch.empty(max(256, L.qlora_linear_bwd_workspace_bytes(M, lin.K, lin.N, r)), dtype=u8,
                                device=dev)
        self.y = torch.empty((M, lin.N), dtype=bf, device=dev)
        self.t = torch.empty((M, r), dtype=f32, device=dev)
        self.dX = torch.empty((M, lin.K), dtype=bf, device=dev)
        self.dA = torch.empty((r, lin.K), dtype=bf, device=dev)
        self.dB = torch.empty((lin.N, r), dtype=bf, device=dev)
        self.plan = q.linear_plan(M, lin.K, lin.N, r)


def _p(t):
    import ctypes
    return ctypes.c_void_p(t.data_ptr())


def run_linear(L, b: LinearBufs, wdq, stream, ev=None):
    """quantize -> dequant -> forward -> backward of one linear through the C ABI."""
    import ctypes
    import bit_nf4_quantized_dq_b200 as q
    st = ctypes.c_void_p(stream)

    def chk(rc, what):
        if rc != 0:
            raise RuntimeError(f"{what}: {rc} {L.qnf4_last_error().decode()}")

    numel = b.N * b.K
    if ev:
        ev["q0"].record()
    chk(L.nf4_quantize_dq(_p(b.W), numel, _p(b.Q.codes), _p(b.Q.scale_codes), _p(b.Q.c2), _p(b.Q.mean),
                          _p(b.ws_q), b.ws_q.numel(), st), "quantize")
    if ev:
        ev["q1"].record()
    chk(L.nf4_dequant(_p(b.Q.codes), _p(b.Q.scale_codes), _p(b.Q.c2), _p(b.Q.mean), numel, _p(wdq), st),
        "dequant")
    if ev:
        ev["d1"].record()
        q.set_timing_events(ev["fwd"])
    chk(L.qlora_linear_fwd(_p(b.x), b.M, b.K, b.N, _p(b.Q.codes), _p(b.Q.scale_codes), _p(b.Q.c2), _p(b.Q.mean),
                           _p(b.A), _p(b.B), b.r, ctypes.c_float(b.s), _p(b.y), _p(b.t), _p(b.ws_f),
                           b.ws_f.numel(), st), "fwd")
    if ev:
        q.set_timing_events(ev["bwd"])
    chk(L.qlora_linear_bwd(_p(b.dY), _p(b.x), _p(b.t), b.M, b.K, b.N, _p(b.Q.codes), _p(b.Q.scale_codes),
                           _p(b.Q.c2), _p(b.Q.mean), _p(b.A), _p(b.B), b.r, ctypes.c_float(b.s), _p(b.dX),
                           _p(b.dA), _p(b.dB), _p(b.ws_b), b.ws_b.numel(), st), "bwd")
    if ev:
        q.set_timing_events(None)


def make_events(n_linears):
    """Timing events of one step.  torch only reports elapsed time between events it has
    recorded itself, so every event is recorded once here (outside any timed region); the
    library's stage marks then re-record the same handles at the stage boundaries."""
    import torch

    def E():
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        return e
    return [{"q0": E(), "q1": E(), "d1": E(), "fwd": [E() for _ in range(3)], "bwd": [E() for _ in range(6)]}
            for _ in range(n_linears)]


class CudaTimer:
    """Device time between two CUDA events on the current stream."""

    def __init__(self):
        import torch
        self.t0 = torch.cuda.Event(enable_timing=True)
        self.t1 = torch.cuda.Event(enable_timing=True)

    def start(self):
        self.t0.record()

    def stop(self):
        self.t1.record()

    def elapsed_ms(self) -> float:
        return self.t0.elapsed_time(self.t1)


def timed_region(step, steps: int, warmup: int, dist, sync, timer, reduce_max, on_start=None, on_stop=None):
    """The rank orchestration of every timed run: `warmup` untimed steps, a barrier and a
    synchronize, `steps` timed steps (step(k) gets the step index), a synchronize and a
    barrier, then the elapsed time reduced to its maximum over the ranks.  Every rank takes
    the same collective calls in the same order.  `dist` is None on one rank."""
    for _ in range(warmup):
        step(None)
    sync()
    if dist is not None:
        dist.barrier()
    sync()
    if on_start:
        on_start()
    timer.start()
    for k in range(steps):
        step(k)
    timer.stop()
    sync()
    if on_stop:
        on_stop()
    if dist is not None:
        dist.barrier()
    return reduce_max(timer.elapsed_ms())


def make_reduce_max(dist, device):
    """Max over ranks of a host float, through a one-element tensor on `device`."""
    def reduce_max(v: float) -> float:
        if dist is None:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return reduce_max


def ours(args, rank, world, dev_index):
    import torch
    import bit_nf4_quantized_dq_b200 as q

    dev = torch.device("cuda", dev_index)
    torch.cuda.set_device(dev)
    L = q.lib()
    lins = linears()
    bufs = [LinearBufs(l, M_TOKENS, R, 3000 + 100 * rank + i, dev) for i, l in enumerate(lins)]
    wdq = torch.empty(max(l.N * l.K for l in lins), dtype=torch.bfloat16, device=dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
    from bit_nf4_quantized_dq_b200.dp import allreduce_adapter_grads

    stream = torch.cuda.current_stream().cuda_stream
    ev_steps = [make_events(len(bufs)) for _ in range(args.steps)]

    def step(k):
        evs = ev_steps[k] if k is not None else None
        for i, b in enumerate(bufs):
            run_linear(L, b, wdq, stream, evs[i] if evs else None)
            if dist is not None:
                allreduce_adapter_grads([b.dA, b.dB])

    # ------------------------------------------------ device-timed run (inputs resident in HBM)
    clocks = NvmlClockSampler(dev_index)
    clock_info = {}

    def stop_clocks():
        clock_info.update(clocks.stop())

    elapsed_ms = timed_region(step, args.steps, args.warmup, dist, torch.cuda.synchronize, CudaTimer(),
                              make_reduce_max(dist, dev), on_start=clocks.start, on_stop=stop_clocks)
    q.check_device_error()
    ms_per_step = elapsed_ms / args.steps

    # per-stage totals over the timed steps
    acc = {k: 0.0 for k in ("quantize", "dequant", "fwd_down", "fwd_fused", "bwd_prep", "bwd_up", "dx_fused",
                            "dA", "dB")}
    for evs in ev_steps:
        for e in evs:
            acc["quantize"] += e["q0"].elapsed_time(e["q1"])
            acc["dequant"] += e["q1"].elapsed_time(e["d1"])
            f, b = e["fwd"], e["bwd"]
            acc["fwd_down"] += f[0].elapsed_time(f[1])
            acc["fwd_fused"] += f[1].elapsed_time(f[2])
            acc["bwd_prep"] += b[0].elapsed_time(b[1])
            acc["bwd_up"] += b[1].elapsed_time(b[2])
            acc["dx_fused"] += b[2].elapsed_time(b[3])
            acc["dA"] += b[3].elapsed_time(b[4])
            acc["dB"] += b[4].elapsed_time(b[5])
    K = args.steps
    weights = sum(l.N * l.K for l in lins)
    fused_fwd_flops = sum(2 * M_TOKENS * l.N * l.K + 2 * M_TOKENS * l.N * R for l in lins)
    fused_dx_flops = sum(2 * M_TOKENS * l.N * l.K + 2 * M_TOKENS * l.K * R for l in lins)
    peaks, peak_src = load_peaks()
    rows = {
        "quantize_gbs": weights * CODEC_BYTES_PER_WEIGHT * K / (acc["quantize"] * 1e6),
        "dequant_gbs": weights * (CODEC_BYTES_PER_WEIGHT) * K / (acc["dequant"] * 1e6),
        "fwd_fused_tflops": fused_fwd_flops * K / (acc["fwd_fused"] * 1e9),
        "dx_fused_tflops": fused_dx_flops * K / (acc["dx_fused"] * 1e9),
        "ms_per_step_by_stage": {k: v / K for k, v in acc.items()},
    }
    rows["quantize_frac_hbm"] = rows["quantize_gbs"] / peaks["hbm_gbs"]
    rows["dequant_frac_hbm"] = rows["dequant_gbs"] / peaks["hbm_gbs"]
    linear_ms = sum(acc[k] for k in ("fwd_down", "fwd_fused", "bwd_prep", "bwd_up", "dx_fused", "dA", "dB")) / K
    rows["linear_fwd_bwd_tflops"] = step_flops() / (linear_ms * 1e9)
    peak, which = pick_bf16_peak(peaks, clock_info)
    rows["fwd_fused_frac"] = rows["fwd_fused_tflops"] / peak
    rows["dx_fused_frac"] = rows["dx_fused_tflops"] / peak
    rows["linear_fwd_bwd_frac"] = rows["linear_fwd_bwd_tflops"] / peak
    # dominant kernel: the fused dequant GEMM with the larger total time
    if acc["fwd_fused"] >= acc["dx_fused"]:
        dom, dom_flops, dom_ms = "fused forward GEMM (NF4 dequant producer + tcgen05)", fused_fwd_flops, acc["fwd_fused"]
        traffic = fused_traffic("fwd")
    else:
        dom, dom_flops, dom_ms = "fused dX GEMM (NF4 dequant producer + tcgen05)", fused_dx_flops, acc["dx_fused"]
        traffic = fused_traffic("dx")
    launches_per_linear = [b.plan["fwd_launches"] + b.plan["bwd_launches"] + QUANTIZE_LAUNCHES + 1 for b in bufs]
    achieved = dom_flops / (dom_ms / K) / 1e9
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "peak_source": (f"{peak_src} bf16 {which} (median SM clock {clock_info.get('sm_mhz')} MHz of "
                                f"{clock_info.get('sm_max_mhz')} during the timed region)"),
                "frac_vs_burst": achieved / peaks["bf16_tflops"],
                "frac_vs_sustained": achieved / peaks["bf16_tflops_sustained"],
                "traffic": traffic, "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                "launches_per_step": len(lins), "avg_launch_ms": dom_ms / K / len(lins),
                "algorithmic_flops_per_launch": dom_flops / len(lins)}

    # ------------------------------------------------ end to end through host buffers
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(args, bufs, wdq, L, dist, dev)

    extra = {}
    if world == 1 and not args.no_extra:
        del ev_steps
        extra = extra_rows(args, L, dev, peaks, peak)

    flops_all = step_flops() * world
    value = flops_all / (ms_per_step / 1e3) / 1e12
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "model": "LLaMA-13B decoder block, 7 linears (random init)",
                   "tokens_per_gpu": M_TOKENS, "global_batch_tokens": M_TOKENS * world, "r": R, "alpha": ALPHA,
                   "parallelism": f"dp{world}", "l2": "inputs larger than L2 (weights + activations, about 3 GB)",
                   "step": "per linear: quantize W, dequant W, fused fwd, bwd (dX, dA, dB)"},
        "rows": rows, "roofline": roofline, "gpu_launches": sum(launches_per_linear) * K, "clocks": clock_info,
    }
    if extra:
        out["rows"].update(extra)
    if e2e is not None:
        out["e2e"] = e2e
    return out


def end_to_end(args, bufs, wdq, L, dist, dev):
    """The same step through the C ABI with the inputs copied in from pinned host buffers and
    the outputs copied back every step.  Host-to-device copies run on one stream, the
    compute on the current stream and device-to-host copies on a third, ordered per linear
    by events, so that linear i+1's inputs and linear i-1's outputs move while linear i
    computes."""
    import torch
    from bit_nf4_quantized_dq_b200.dp import allreduce_adapter_grads
    host_in, host_out = [], []
    h2d = d2h = 0
    for b in bufs:
        hi = {k: getattr(b, k).to("cpu").pin_memory() for k in ("W", "x", "A", "B", "dY")}
        ho = {k: torch.empty(getattr(b, k).shape, dtype=getattr(b, k).dtype, pin_memory=True)
              for k in ("y", "dX", "dA", "dB")}
        host_in.append(hi)
        host_out.append(ho)
        h2d += sum(v.numel() * v.element_size() for v in hi.values())
        d2h += sum(v.numel() * v.element_size() for v in ho.values())
    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(bufs)
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_done = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]

    def step(_k):
        for i, (b, hi, ho) in enumerate(zip(bufs, host_in, host_out)):
            s_in.wait_event(ev_done[i])          # the previous step's linear i no longer reads them
            with torch.cuda.stream(s_in):
                for k, v in hi.items():
                    getattr(b, k).copy_(v, non_blocking=True)
            ev_in[i].record(s_in)
            compute.wait_event(ev_in[i])
            compute.wait_event(ev_out[i])        # the previous step's outputs of linear i are copied out
            run_linear(L, b, wdq, compute.cuda_stream)
            if dist is not None:
                allreduce_adapter_grads([b.dA, b.dB])
            ev_done[i].record(compute)
            s_out.wait_event(ev_done[i])
            with torch.cuda.stream(s_out):
                for k, v in ho.items():
                    v.copy_(getattr(b, k), non_blocking=True)
            ev_out[i].record(s_out)
        for i in range(n):
            compute.wait_event(ev_out[i])        # the step ends when its last output is on the host

    ms = timed_region(step, args.steps, 1, dist, torch.cuda.synchronize, CudaTimer(), make_reduce_max(dist, dev))
    world = dist.get_world_size() if dist is not None else 1
    value = step_flops() * world / (ms / args.steps / 1e3) / 1e12
    return {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / args.steps,
            "copies": "pinned host buffers; H2D, compute and D2H on three streams, overlapped across linears"}


# ------------------------------------------------------------------------------------------
# extra rows: the 512-token LLaMA-7B block, the 65B stack codec sweep, the robust weight
# ------------------------------------------------------------------------------------------
def _time_calls(fn, reps: int, warmup: int = 2) -> float:
    """Mean device time in ms of fn() over `reps` calls on the current stream."""
    import torch
    for _ in range(warmup):
        fn()
    t = CudaTimer()
    torch.cuda.synchronize()
    t.start()
    for _ in range(reps):
        fn()
    t.stop()
    torch.cuda.synchronize()
    return t.elapsed_ms() / reps


def rows_llama7b_512(L, dev, peak):
    """The seven linears of a LLaMA-7B block at 512 tokens (r = 64): the same step as the
    headline (quantize, dequant, fwd, bwd per linear)."""
    import torch
    import synth
    lins = synth.LLAMA7B
    M = 512
    bufs = [LinearBufs(l, M, R, 2000 + i, dev) for i, l in enumerate(lins)]
    wdq = torch.empty(max(l.N * l.K for l in lins), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream().cuda_stream

    def step():
        for b in bufs:
            run_linear(L, b, wdq, stream)

    ms = _time_calls(step, 10, 3)
    flops = sum(linear_flops(M, l.N, l.K, R) for l in lins)
    return {"workload": "llama7b_block_512tok", "ms_per_step": ms, "tflops": flops / (ms * 1e9),
            "frac": flops / (ms * 1e9) / peak,
            "note": "step = quantize + dequant + fwd + bwd of the 7 linears; flops = 4MNK + 6MKr + 6MNr"}


def rows_stack65b(L, dev, hbm_gbs, layers: int):
    """Quantize and dequant, layer by layer, of `layers` layers of the 65B-shaped stack (each
    layer: 4 x 8192x8192, 3 x 22016x8192, W ~ N(0, 0.015^2) drawn per layer on the GPU)."""
    import torch
    import synth
    import bit_nf4_quantized_dq_b200 as q
    shapes = synth.STACK65B_LAYER
    big = max(l.N * l.K for l in shapes)
    W = torch.empty(big, dtype=torch.bfloat16, device=dev)
    out = torch.empty(big, dtype=torch.bfloat16, device=dev)
    nb_big = (big + 63) // 64
    codes = torch.empty(32 * nb_big, dtype=torch.uint8, device=dev)
    sc = torch.empty(nb_big, dtype=torch.uint8, device=dev)
    c2 = torch.empty((nb_big + 255) // 256, dtype=torch.float32, device=dev)
    mean = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(L.nf4_quantize_workspace_bytes(big), dtype=torch.uint8, device=dev)
    st = _stream_arg()
    g = torch.Generator(device=dev)
    tq = td = 0.0
    nweights = nbytes = 0
    for layer in range(layers):
        for j, l in enumerate(shapes):
            numel = l.N * l.K
            g.manual_seed(synth.seed_for(4, layer * 7 + j))
            Wv = W[:numel]
            Wv.copy_(torch.randn(numel, generator=g, device=dev) * 0.015)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record()
            rc = L.nf4_quantize_dq(_p(Wv), numel, _p(codes), _p(sc), _p(c2), _p(mean), _p(ws), ws.numel(), st)
            e[1].record()
            rc |= L.nf4_dequant(_p(codes), _p(sc), _p(c2), _p(mean), numel, _p(out), st)
            e[2].record()
            if rc != 0:
                raise RuntimeError(L.qnf4_last_error().decode())
            torch.cuda.synchronize()
            tq += e[0].elapsed_time(e[1])
            td += e[1].elapsed_time(e[2])
            nb = (numel + 63) // 64
            nweights += numel
            nbytes += 32 * nb + nb + 4 * ((nb + 255) // 256) + 4
    q.check_device_error()
    gb = nweights * CODEC_BYTES_PER_WEIGHT / 1e9
    return {"workload": "stack65b_codec", "layers_timed": layers, "layers_in_stack": 80, "weights": nweights,
            "stored_bits_per_weight": nbytes * 8 / nweights,
            "stored_bits_per_weight_expected": 4.126953125, "stack_stored_gb_80_layers": nbytes * 80 / layers / 1e9,
            "quantize_gbs": gb / (tq / 1e3), "dequant_gbs": gb / (td / 1e3),
            "quantize_frac_hbm": gb / (tq / 1e3) / hbm_gbs, "dequant_frac_hbm": gb / (td / 1e3) / hbm_gbs,
            "note": "algorithmic bytes 2.51587 per weight for each of quantize and dequant"}


def _stream_arg():
    import ctypes
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def linear_hbm_bytes(M, N, K, r):
    """Algorithmic HBM bytes of one fwd + bwd: activations, codes + scales, adapters, outputs."""
    codec = N * K * (0.5 + 1.0 / 64 + 4.0 / (64 * 256))
    fwd = 2 * M * K + codec + 2 * r * K + 2 * N * r + 2 * M * N + 4 * M * r
    bwd = 2 * M * N + codec + 2 * M * K + 2 * M * K + 2 * (2 * r * K + 2 * N * r) + 4 * M * r
    return fwd + bwd


def rows_robust(L, dev, peaks, peak):
    """fwd + bwd on the robust 4000x3000 weight (Student-t, outlier columns, exact zeros) for
    r in {8, 64, 256} and M in {1, 16, 512, 16384}; M <= 16 is reported against HBM."""
    import torch
    import synth
    import bit_nf4_quantized_dq_b200 as q
    N, K = 4000, 3000
    W = synth.robust_weight_bf16(N, K, synth.seed_for(5, 0)).to(dev)
    Q = q.nf4_quantize_dq(W)
    out = []
    for r in (8, 64, 256):
        for M in (1, 16, 512, 16384):
            inp = synth.linear_inputs(M, N, K, r, synth.seed_for(5, 10 + r + M), device=str(dev))
            s = ALPHA / r
            wsf = torch.empty(max(256, L.qlora_linear_fwd_workspace_bytes(M, K, N, r)), dtype=torch.uint8, device=dev)
            wsb = torch.empty(max(256, L.qlora_linear_bwd_workspace_bytes(M, K, N, r)), dtype=torch.uint8, device=dev)
            x, A, B, dY = inp["x"], inp["A"], inp["B"], inp["dY"]

            def fb():
                y, t = q.qlora_linear_fwd(x, Q, A, B, s, workspace=wsf)
                q.qlora_linear_bwd(dY, x, t, Q, A, B, s, workspace=wsb)

            ms = _time_calls(fb, 20 if M <= 512 else 5)
            flops = linear_flops(M, N, K, r)
            row = {"r": r, "M": M, "ms": ms, "tflops": flops / (ms * 1e9), "frac_tensor": flops / (ms * 1e9) / peak}
            hb = linear_hbm_bytes(M, N, K, r)
            row["gbs"] = hb / (ms * 1e6)
            if M <= 16:
                row["frac_hbm"] = row["gbs"] / peaks["hbm_gbs"]
                # the same calls replayed from a CUDA graph: the host-side cost of the Python
                # calls (larger than the kernels at these sizes) leaves the timed region
                try:
                    torch.cuda.synchronize()
                    side = torch.cuda.Stream()
                    side.wait_stream(torch.cuda.current_stream())
                    with torch.cuda.stream(side):
                        fb()
                    torch.cuda.current_stream().wait_stream(side)
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        fb()
                    mg = _time_calls(g.replay, 50)
                    row["ms_graph"] = mg
                    row["gbs_graph"] = hb / (mg * 1e6)
                    row["frac_hbm_graph"] = row["gbs_graph"] / peaks["hbm_gbs"]
                    del g
                except Exception as exc:   # capture is a measurement aid; report why it is missing
                    row["graph_error"] = str(exc)[:120]
            out.append(row)
    q.check_device_error()
    return {"workload": "robust_4000x3000", "points": out,
            "note": "fwd + bwd through the Python binding (allocating outputs); M <= 16 is HBM-bound, and is "
                    "also timed as CUDA-graph replays of the same calls (ms_graph)"}


def rows_variants(dev, peaks, peak):
    """Code books and scale formats on the 13B q linear (5120 x 5120, 8192 tokens, r = 64):
    stored bits per weight, quantize / dequant GB/s (algorithmic bytes: bf16 in, codes and
    scales out, or the reverse) and the fused forward + backward TFLOP/s; then the adapter
    merge + re-quantization and one paged AdamW step over the block's adapters."""
    import torch
    import synth
    import bit_nf4_quantized_dq_b200 as q
    N = K = 5120
    M = M_TOKENS
    W = synth.normal_bf16((N, K), 0.02, 3000, device=str(dev))
    inp = synth.linear_inputs(M, N, K, R, 3000, device=str(dev))
    x, A, B, dY = inp["x"], inp["A"], inp["B"], inp["dY"]
    s = ALPHA / R
    L = q.lib()
    wsf = torch.empty(max(256, L.qlora_linear_fwd_workspace_bytes(M, K, N, R)), dtype=torch.uint8, device=dev)
    wsb = torch.empty(max(256, L.qlora_linear_bwd_workspace_bytes(M, K, N, R)), dtype=torch.uint8, device=dev)
    out = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    numel = N * K
    points = []
    for cb in ("nf4", "fp4_e2m1", "int4"):
        for dq in (True, False):
            Q = q.quantize(W, codebook=cb, double_quant=dq)
            bits = Q.nbytes() * 8 / numel
            codec_bytes = numel * (2 + bits / 8)
            tq = _time_calls(lambda: q.quantize(W, codebook=cb, double_quant=dq), 10)
            td = _time_calls(lambda: q.nf4_dequant(Q, out=out), 20)

            def fb():
                y, t = q.qlora_linear_fwd(x, Q, A, B, s, workspace=wsf)
                q.qlora_linear_bwd(dY, x, t, Q, A, B, s, workspace=wsb)

            tl = _time_calls(fb, 5)
            fl = linear_flops(M, N, K, R)
            points.append({"codebook": cb, "double_quant": dq, "bits_per_weight": bits,
                           "quantize_gbs": codec_bytes / (tq * 1e6), "dequant_gbs": codec_bytes / (td * 1e6),
                           "dequant_frac_hbm": codec_bytes / (td * 1e6) / peaks["hbm_gbs"],
                           "linear_fwd_bwd_tflops": fl / (tl * 1e9), "linear_frac": fl / (tl * 1e9) / peak})
    Q = q.nf4_quantize_dq(W)
    Ab, Bb = A, B * 20
    tm = _time_calls(lambda: q.merge_requantize(Q, Ab, Bb, s), 5)
    fp64 = numel * R * 2 / (tm * 1e9)
    merge = {"shape": "5120x5120 r=64 NF4+DQ", "ms": tm, "gweights_per_s": numel / (tm * 1e6),
             "fp64_tflops": fp64, "bound": "alu", "fp64_peak_tflops": FP64_PEAK_TFLOPS,
             "frac_fp64": fp64 / FP64_PEAK_TFLOPS,
             "note": "W'' = bf16(W' + s B A): float64 rank-r sum (2 r flops per weight), then re-quantized"}
    lins = linears()
    sizes = [R * l.K + l.N * R for l in lins]
    params = [torch.zeros(n, dtype=torch.float32, device=dev) for n in sizes]
    grads = [torch.zeros(n, dtype=torch.bfloat16, device=dev) for n in sizes]
    nparam = sum(sizes)
    adam = {"params": nparam, "bytes_per_param": 26,
            "note": "AdamW step over the 13B block's adapters (7 tensors, one launch each); 26 B per parameter "
                    "(fp32 p, m, v read and written, bf16 g read); 'device': states in plain device memory, "
                    "'paged': states in managed memory, prefetched to the device before every step"}
    for mode in ("device", "paged"):
        opt = q.PagedAdamW(params, None, lr=1e-4, paged=(mode == "paged"))
        ta = _time_calls(lambda: opt.step(grads), 10)
        opt.close()
        adam[mode] = {"ms": ta, "gbs": nparam * 26 / (ta * 1e6), "frac_hbm": nparam * 26 / (ta * 1e6) / peaks["hbm_gbs"]}
    return {"variants_13b_q": points, "merge_13b_q": merge, "adamw_13b_block": adam}


def extra_rows(args, L, dev, peaks, peak):
    import torch
    torch.cuda.empty_cache()
    rows = {"llama7b_512": rows_llama7b_512(L, dev, peak),
            "stack65b": rows_stack65b(L, dev, peaks["hbm_gbs"], args.stack_layers),
            "robust": rows_robust(L, dev, peaks, peak)}
    torch.cuda.empty_cache()
    rows.update(rows_variants(dev, peaks, peak))
    return rows


# ------------------------------------------------------------------------------------------
# the CPU oracle on a bounded sample of the same workload
# ------------------------------------------------------------------------------------------
def oracle_sample(codec_weights=1 << 21, tokens=128):
    """Time the oracle on a sample: the codec (quantize + dequant) on `codec_weights` weights of
    each linear's weight, and the linear forward + backward of every linear on `tokens` tokens.
    The per-step time is extrapolated linearly in weights (codec) and in tokens (linear)."""
    import numpy as np
    import torch
    import synth
    from oracle import linear as olin
    from oracle import nf4 as onf4

    t_codec = t_lin = 0.0
    codec_done = 0
    lin_flops = 0
    for i, l in enumerate(linears()):
        W = synth.normal_bf16((l.N, l.K), 0.02, 3000 + i).float().numpy()
        sub = W.ravel()[:codec_weights]
        c0 = time.perf_counter()
        qd = onf4.quantize_nf4_dq(sub)
        onf4.dequant_nf4_dq(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], sub.size)
        t_codec += time.perf_counter() - c0
        codec_done += sub.size
        inp = synth.linear_inputs(tokens, l.N, l.K, R, 3000 + i)
        f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
        x, A, B, dY = (f64(inp[k]) for k in ("x", "A", "B", "dY"))
        Wd = W.astype(np.float64)          # stands in for W' (same shape; the codec is timed above)
        c0 = time.perf_counter()
        olin.qlora_forward(x, Wd, A, B, ALPHA / R)
        olin.qlora_backward(dY, x, Wd, A, B, ALPHA / R)
        t_lin += time.perf_counter() - c0
        lin_flops += linear_flops(tokens, l.N, l.K, R)
    weights = sum(l.N * l.K for l in linears())
    est_step_s = t_codec * (weights / codec_done) + t_lin * (step_flops() / lin_flops)
    cores = len(os.sched_getaffinity(0))
    return {
        "value": step_flops() / est_step_s / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
        "sample": (f"codec on the first {codec_weights} weights of each of the 7 weights, fwd+bwd of all 7 "
                   f"linears on {tokens} of the 8192 tokens (float64 numpy, BLAS threads = {cores}); "
                   f"step time extrapolated linearly: {est_step_s:.1f} s"),
        "measured_s": t_codec + t_lin,
    }


def reference(args, rank, world):
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_sample(codec_weights=1 << 16, tokens=16)
    vals, runs = [], []
    for _ in range(args.steps):
        r = oracle_sample(codec_weights=1 << 19, tokens=64)
        vals.append(r["value"])
        runs.append(r)
    v = statistics.median(vals)
    last = runs[-1]
    ms = step_flops() / (v * 1e12) * 1e3
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "model": "LLaMA-13B decoder block, 7 linears (random init)",
                   "tokens_per_gpu": M_TOKENS, "r": R, "alpha": ALPHA, "parallelism": "oracle on host cores"},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


CASES = ("fwd", "bwd", "quantize", "dequant")


def single_case(args):
    """One linear of the block (`--linear`, default q: 5120x5120) at 8192 tokens; runs only the
    calls of `--case` (after one quantize), `--warmup` + `--steps` times.  Small enough (about
    0.2-0.6 GB on the device, more than L2) for profiler captures of one kernel family."""
    import ctypes
    import torch
    import bit_nf4_quantized_dq_b200 as q

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L = q.lib()
    lin = {l.name: l for l in linears()}[args.linear]
    b = LinearBufs(lin, M_TOKENS, R, 3000, dev)
    wdq = torch.empty(lin.N * lin.K, dtype=torch.bfloat16, device=dev)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    numel = lin.N * lin.K

    def quantize():
        assert L.nf4_quantize_dq(_p(b.W), numel, _p(b.Q.codes), _p(b.Q.scale_codes), _p(b.Q.c2), _p(b.Q.mean),
                                 _p(b.ws_q), b.ws_q.numel(), st) == 0

    def fwd():
        assert L.qlora_linear_fwd(_p(b.x), b.M, b.K, b.N, _p(b.Q.codes), _p(b.Q.scale_codes), _p(b.Q.c2),
                                  _p(b.Q.mean), _p(b.A), _p(b.B), b.r, ctypes.c_float(b.s), _p(b.y), _p(b.t),
                                  _p(b.ws_f), b.ws_f.numel(), st) == 0

    def bwd():
        assert L.qlora_linear_bwd(_p(b.dY), _p(b.x), _p(b.t), b.M, b.K, b.N, _p(b.Q.codes), _p(b.Q.scale_codes),
                                  _p(b.Q.c2), _p(b.Q.mean), _p(b.A), _p(b.B), b.r, ctypes.c_float(b.s), _p(b.dX),
                                  _p(b.dA), _p(b.dB), _p(b.ws_b), b.ws_b.numel(), st) == 0

    def dequant():
        assert L.nf4_dequant(_p(b.Q.codes), _p(b.Q.scale_codes), _p(b.Q.c2), _p(b.Q.mean), numel, _p(wdq), st) == 0

    quantize()
    if args.case == "bwd":
        fwd()
    fn = {"fwd": fwd, "bwd": bwd, "quantize": quantize, "dequant": dequant}[args.case]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    q.check_device_error()
    ms = t0.elapsed_time(t1) / args.steps
    print(json.dumps({"case": args.case, "linear": args.linear, "tokens": M_TOKENS, "ms_per_call": ms}), flush=True)


def launcher_command(args, argv):
    """torch.distributed.run command that starts `args.gpus` ranks of this script on this node."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def check_world(args, env) -> tuple:
    """(rank, world, local rank) from the launcher's environment; the world size must match
    --gpus (a silent one-rank run of `--gpus 8` would report the wrong n_gpus)."""
    world = int(env.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but the launcher started {world} rank(s)")
    return int(env.get("RANK", "0")), world, int(env.get("LOCAL_RANK", "0"))


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end run")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the oracle sample")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the extra rows (512-token block, 65B stack sweep, robust weight)")
    ap.add_argument("--stack-layers", type=int, default=80, help="layers of the 65B stack in the codec sweep")
    ap.add_argument("--case", choices=CASES, default=None,
                    help="run one call family on one linear only (profiling aid; prints its own line)")
    ap.add_argument("--linear", default="q", help="linear of the block used by --case")
    args = ap.parse_args(argv)
    if args.case:
        single_case(args)
        return 0
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return subprocess.call(launcher_command(args, argv))
    rank, world, local = check_world(args, os.environ)
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)

    if args.impl == "reference":
        out = reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        out = ours(args, rank, world, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cb = oracle_sample()
            out["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
