#!/usr/bin/env python3
"""Benchmark of the W8A8 / W4A8 quantized linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one call of the linear (activation quant + tcgen05 GEMM with the
fused dequant epilogue) on one batch of synthetic input already resident in
HBM.  The default workload is the DiT MLP projection W8A8 linear,
x [16384, 3072] bf16 -> y [16384, 12288] bf16 (1% outlier channels x20, bias).
Rank 0 prints one JSON line.  On one GPU the default run also carries
  - `int8_peak_probe`: the INT8 tensor-pipe rate measured on the device by the
    library's probe (the GEMM's tcgen05 kind::i8 MMA stream on shared-memory
    operands), burst and sustained, with clocks -- the roofline denominator;
  - `sustained`: the headline call back to back for two seconds, with clocks;
  - `workloads`: every other configuration (tiny, the DiT attention
    projection, the M = 2048 sweep, W4A8 at M = 1 / 8 / 16 / 4096, the
    quick-start matmul, the gated epilogue, the INT8 attention), each with its
    per-call time, throughput, the dominant kernel alone and its roofline
    fraction;
  - `cpu_baseline`: the oracle on the host cores, one thread and all cores.
Under torchrun each rank is an independent replica (the path needs no
collective): per-GPU work is fixed, the value is the sum over ranks divided by
the slowest rank's time ("scaling": "weak").

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and torch.cuda.synchronize(), CUDA events on the launching stream, max over
ranks.  Inputs rotate over two full input sets (x and Wq), so every step reads
its operands from HBM (x 100.7 MB + Wq 37.7 MB per set, y 402.7 MB written per
step; more than the 126 MB L2).  SM clocks and throttle reasons are sampled
with NVML during the timed region.

`--impl reference` times the CPU oracle (oracle/, plain C, OpenMP over rows)
on all host cores for the same metric, one bounded sample of the workload per
step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 linear TOPS incl. act quant at DiT shapes; % of B200 INT8 peak"
INT8_SPEC_TOPS = 4500.0  # dense INT8, B200 datasheet
L2_BYTES = 126 * 1024 * 1024

WORKLOADS = {
    "dit_mlp": ("DIT_MLP", None),
    "dit_mlp_gated": ("DIT_MLP", None),
    "dit_mlp_fused": ("DIT_MLP", None),
    "dit_attn_fused": ("DIT_ATTN", None),
    "quickstart_w8a8_fused": ("QUICKSTART", 0),
    "dit_attn": ("DIT_ATTN", None),
    "sweep_4096x4096": ("SWEEP", 0),
    "sweep_4096x12288": ("SWEEP", 1),
    "sweep_12288x4096": ("SWEEP", 2),
    "sweep_thin_5120x48": ("SWEEP", 3),
    "tiny": ("TINY", None),
    "w4a8_m1": ("W4A8", 0),
    "w4a8_m8": ("W4A8", 1),
    "w4a8_m16": ("W4A8", 2),
    "w4a8_m4096": ("W4A8", 3),
    "quickstart_w8a8": ("QUICKSTART", 0),
    "quickstart_w4a8": ("QUICKSTART", 1),
    "w4a8_m4096_prepared": ("W4A8", 3),
    "quickstart_w4a8_prepared": ("QUICKSTART", 1),
    "sage_attn": ("SAGE_QUICKSTART", None),
}
ATTN_METRIC = "INT8 attention TFLOP/s (4 B H L^2 D ops) at DiT shapes"


def get_case(name):
    from w4a8_quantized_gemm_token_b200 import synthetic

    attr, idx = WORKLOADS[name]
    obj = getattr(synthetic, attr)
    return obj if idx is None else obj[idx]


def is_w4(name):
    return "w4a8" in name


def is_attention(name):
    return name.startswith("sage")


def is_fused(name):
    """The W8A8 linear as one kernel (qk_w8a8_linear_fused)."""
    return name.endswith("_fused")


def is_prepared(name):
    """The W4A8 linear on a prepared weight (qk_w4a8_prepare once, then
    qk_w4a8_linear_prepared): the digit planes are not rebuilt per call."""
    return name.endswith("_prepared")


def is_gated(name):
    """The W8A8 linear with the gated residual epilogue y = r + gate * linear."""
    return name.endswith("_gated")


# ------------------------------------------------------------ peaks / clocks

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}


class ClockSampler:
    """Samples SM clock, power and clock-event reasons with NVML every `period` s."""

    def __init__(self, torch_device: int, period: float = 0.02):
        self.period = period
        self.samples = []
        self.handle = None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            self.nv = pynvml
            bus = None
            props = torch.cuda.get_device_properties(torch_device)
            if hasattr(props, "pci_bus_id"):
                bus = f"{getattr(props, 'pci_domain_id', 0):08x}:{props.pci_bus_id:02x}:" \
                      f"{getattr(props, 'pci_device_id', 0):02x}.0"
            if bus is not None:
                try:
                    self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
                except Exception:
                    self.handle = None
            if self.handle is None:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(torch_device)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.handle = None
            self.max_mhz = None

    def _one(self):
        nv = self.nv
        try:
            sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            pw = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
            self.samples.append((sm, rs, pw))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._one()
            time.sleep(self.period)

    def __enter__(self):
        if self.handle is not None:
            self._one()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.handle is not None:
            self._stop.set()
            self._t.join()
            self._one()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, rs, _ in self.samples:
            for bit, name in REASON_BITS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": float(statistics.median(s[0] for s in self.samples)),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "power_w_max": round(max(s[2] for s in self.samples), 1),
                "samples": len(self.samples)}


def traffic_from_profile(kernel_tag: str, src_path: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel (matched by a hash of the .cu file) and
    on this workload (the summary's `workload:` line)."""
    import hashlib

    prof = os.path.join(ROOT, "profiles", f"{kernel_tag}.txt")
    try:
        digest = hashlib.sha256(open(src_path, "rb").read()).hexdigest()[:16]
        fields = {}
        for line in open(prof):
            if ":" in line:
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
        if fields.get("source_sha256_16") != digest or fields.get("workload") != workload:
            return None
        return float(fields["dram_bytes_per_launch_full_workload"])
    except (OSError, KeyError, ValueError):
        return None


# ------------------------------------------------------------ distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of `value` over ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def whole_job_value(ops_per_step: float, steps: int, world: int, max_seconds: float) -> float:
    """Aggregate throughput over all ranks in tera-ops/s (each rank does the same work)."""
    return ops_per_step * steps * world / max_seconds / 1e12


# ------------------------------------------------------------ our arm

def graph_runner(fn, steps):
    """Capture `steps` calls of fn(i) into one CUDA graph; returns its replay.
    Used where a step lasts only microseconds, so host launch cost would
    otherwise be timed instead of the kernels."""
    import torch

    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for i in range(steps):
                fn(i)
    torch.cuda.current_stream().wait_stream(side)
    # The first replay of a graph also uploads it to the device; replay once
    # here (untimed, as warm-up) so the timed replay measures the kernels only.
    g.replay()
    torch.cuda.synchronize()
    return g.replay


def event_ms(run, stream):
    """Milliseconds of run() between two CUDA events on `stream` (synchronized
    on both sides)."""
    import torch

    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def csrc(name):
    return os.path.join(ROOT, "w4a8_quantized_gemm_token_b200", "csrc", name)


class LinearRun:
    """One W8A8 / W4A8 linear workload resident on the device: rotating input
    sets (enough that one pass over them exceeds twice the L2), quantized
    weights, a workspace and the output."""

    def __init__(self, name, dev, sets=0):
        import torch

        from w4a8_quantized_gemm_token_b200 import binding as qk
        from w4a8_quantized_gemm_token_b200 import synthetic

        self.qk, self.name, self.dev = qk, name, dev
        self.case = case = get_case(name)
        M, K, N = self.M, self.K, self.N = case.M, case.K, case.N
        self.w4, self.gated = is_w4(name), is_gated(name)
        self.prepared = None
        xb, W, b, _ = case.draw()
        self.x_host = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
        del xb
        if self.gated:
            gate_np, res_bits = synthetic.gated_inputs(case)
            self.gate = torch.from_numpy(gate_np).to(dev)
            self.res_host = torch.from_numpy(res_bits.view(np.int16)).view(torch.bfloat16)
            self.res = self.res_host.to(dev)
            del res_bits
        W_dev = torch.from_numpy(W).to(dev)
        del W
        self.bias = torch.from_numpy(b).to(dev) if b is not None else None
        w4 = self.w4
        self.per_set = M * K * 2 + (N * K // 2 + N * (K // 64) * 4 if w4 else N * K + 4 * N)
        self.nsets = sets or int(min(32, max(2, -(-2 * L2_BYTES // self.per_set))))
        self.xs = [self.x_host.to(dev) for _ in range(self.nsets)]
        if w4:
            self.weights = [qk.qk_quantize_weights_int4(W_dev) for _ in range(self.nsets)]
            wsz = qk.qk_w4a8_workspace_size(M, K)
            self.prepared = ([qk.qk_w4a8_prepare(*wt)[0] for wt in self.weights]
                             if is_prepared(name) else None)
        else:
            self.weights = [qk.qk_quantize_weights_int8(W_dev) for _ in range(self.nsets)]
            wsz = qk.qk_w8a8_workspace_size(M, K)
        del W_dev
        self.ws = torch.empty(wsz, dtype=torch.uint8, device=dev)
        self.y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        self.ops = 2.0 * M * N * K
        self.xq_sets = None

    def step(self, i):
        qk, wt, x = self.qk, self.weights[i % self.nsets], self.xs[i % self.nsets]
        if self.w4 and self.prepared is not None:
            qk.qk_w4a8_linear_prepared(x, *wt, self.prepared[i % self.nsets], self.bias, y=self.y,
                                       workspace=self.ws)
        elif self.w4:
            qk.qk_w4a8_linear(x, *wt, self.bias, y=self.y, workspace=self.ws)
        elif self.gated:
            qk.qk_w8a8_linear_gated(x, *wt, self.bias, self.gate, self.res, y=self.y,
                                    workspace=self.ws)
        else:
            qk.qk_w8a8_linear(x, *wt, self.bias, y=self.y, workspace=self.ws,
                              fused=is_fused(self.name))

    def kstep(self, i):
        """The dominant kernel alone: the product on pre-quantized activations
        (the gated linear has no such entry: its call is timed)."""
        qk = self.qk
        if self.gated or (is_fused(self.name) and self.N > 64):
            return self.step(i)  # the call is the kernel (gated: no split entry)
        if self.xq_sets is None:
            self.xq_sets = [qk.qk_quantize_activations(x, with_xsum=self.w4) for x in self.xs]
        xq, sx, xsum = self.xq_sets[i % self.nsets]
        wt = self.weights[i % self.nsets]
        if self.w4 and self.prepared is not None:
            qk.qk_w4a8_gemm_prepared(xq, sx, xsum, *wt, self.prepared[i % self.nsets], self.bias,
                                     y=self.y)
        elif self.w4:
            route = qk.QK_ROUTE_GEMV if self.M <= 16 else qk.QK_ROUTE_GEMM
            qk.qk_w4a8_gemm(xq, sx, xsum, *wt, self.bias, y=self.y, route=route)
        else:
            qk.qk_w8a8_gemm(xq, sx, *wt, self.bias, y=self.y)

    def kernel(self):
        """(kernel tag, source file, bound, algorithmic bytes per launch)."""
        M, K, N = self.M, self.K, self.N
        if self.w4 and M <= 16:
            G = K // 64
            kbytes = N * K / 2 + 4 * N * G + M * K + 4 * M + 4 * M * G + 2 * M * N
            one = M == 1 and K % 1024 == 0 and K <= 4096   # the dp4a one-token kernel
            return (("w4a8_gemv1_kernel", "gemv1_w4a8.cu") if one else
                    ("w4a8_gemv_kernel", "gemv_w4a8.cu")) + ("hbm", kbytes)
        if not self.w4 and N <= 64 and M <= 8192:           # thin outputs: split-K route
            return ("w8a8_skinny_kernel", "gemm_w8a8_skinny.cu", "hbm",
                    M * K + N * K + 2 * M * N + 4 * (M + 2 * N))
        if self.w4:
            # the GEMM route: plane count, plane build, gated fold, byte-plane GEMM
            return ("w4a8_planes_kernel", "gemm_w4a8_planes.cu", "tensor", None)
        return ("w8a8_gemm_kernel", "gemm_w8a8.cu", "tensor", None)


def launches_per_call(M, K, N, w4, gated, qk, fused=False, prepared=False):
    """Kernels one call of the linear launches: the W8A8 linear is the
    quantization kernel + the GEMM (qk_w8a8_linear_fused: one kernel, except
    for thin outputs, N <= 64); the W4A8 linear follows its plan
    (qk_w4a8_linear_plan); its GEMM route is four kernels (the plane count,
    the plane build, the per-group fold that computes only when the byte
    planes cannot, and the byte-plane GEMM), two on a prepared weight."""
    if w4:
        plan = qk.qk_w4a8_linear_plan(M, K, N)
        return {qk.QK_PLAN_GEMV_QUANT: 1, qk.QK_PLAN_QUANT_GEMV: 2}.get(plan, 3 if prepared else 5)
    if gated or not fused or (N <= 64 and M <= 8192):
        return 2
    return 1


def int8_peak_source(peaks, int8):
    if int8 is not None:
        return int8["burst"]["tops"], ("measured in this run: the tcgen05 kind::i8 probe "
                                       "(qk_debug_int8_peak, the GEMM's MMA stream on "
                                       "shared-memory operands), burst")
    return peaks["bf16"] * 2.0, (f"{peaks['source']} bf16_tflops (burst) x 2, the nominal "
                                 "int8/bf16 ratio (4.5 / 2.25 POPS)")


def roofline(run, k_ms, peaks, int8, workload):
    tag, src, bound, kbytes = run.kernel()
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": kbytes / (k_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "peak_source": f"{peaks['source']} hbm_gbs (copy)",
                "algorithmic_bytes": kbytes}
    else:
        peak, psrc = int8_peak_source(peaks, int8)
        roof = {"bound": "tensor", "achieved": run.ops / (k_ms / 1e3) / 1e12, "peak": peak,
                "unit": "TFLOP/s", "peak_source": psrc + "; int8 ops counted as 2*M*N*K",
                "algorithmic_ops": run.ops}
    roof["kernel"] = tag
    roof["traffic"] = traffic_from_profile(tag, csrc(src), workload)
    if run.gated:
        roof["kernel"] = "w8a8_gemm_kernel (gated) with its activation quant: the timed call"
        roof["traffic"] = None  # the committed summary covers the plain epilogue
    elif is_fused(workload) and run.N > 64:
        roof["kernel"] = "w8a8_gemm_kernel with fused activation quantization: the timed call"
        roof["traffic"] = None
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel_ms"] = k_ms
    return roof


def time_linear(run, steps, warmup, local, graph="auto"):
    """Time `steps` calls (after `warmup`), then the dominant kernel alone.
    Returns (ms per call, kernel ms, clock summary, timing label)."""
    import torch

    stream = torch.cuda.current_stream()
    for i in range(warmup):
        run.step(i)
    torch.cuda.synchronize()
    run.qk.qk_check_device_error()
    use_graph = graph == "on" or (graph == "auto" and run.M <= 256)
    run_steps = graph_runner(run.step, steps) if use_graph else \
        (lambda: [run.step(i) for i in range(steps)])
    sampler = ClockSampler(local)
    barrier(run.dev)
    torch.cuda.synchronize()
    with sampler:
        ms = event_ms(run_steps, stream)
    barrier(run.dev)
    run.qk.qk_check_device_error()
    for i in range(warmup):
        run.kstep(i)
    torch.cuda.synchronize()
    run_k = graph_runner(run.kstep, steps) if use_graph else \
        (lambda: [run.kstep(i) for i in range(steps)])
    k_ms = event_ms(run_k, stream) / steps
    run.qk.qk_check_device_error()
    return ms, k_ms, sampler.summary(), \
        ("CUDA graph of the timed calls" if use_graph else "eager launches")


def measure_int8_peak(local, burst_ms=20.0, sustained_s=2.0):
    """INT8 tensor-pipe rate of the device from qk_debug_int8_peak: a burst
    (one ~20 ms launch, best of 3) and a sustained run (~50 ms launches back to
    back for `sustained_s`), with the SM clocks sampled during each."""
    import torch

    from w4a8_quantized_gemm_token_b200 import binding as qk

    stream = torch.cuda.current_stream()
    qk.qk_debug_int8_peak(256)
    torch.cuda.synchronize()
    cal = 4096
    ops_cal = [0.0]
    ms = event_ms(lambda: ops_cal.__setitem__(0, qk.qk_debug_int8_peak(cal)), stream)
    iters = int(max(256, min(1 << 22, cal * burst_ms / max(ms, 1e-3))))
    best = None
    sampler = ClockSampler(local, period=0.005)
    with sampler:
        for _ in range(3):
            ops = [0.0]
            ms = event_ms(lambda: ops.__setitem__(0, qk.qk_debug_int8_peak(iters)), stream)
            tops = ops[0] / (ms / 1e3) / 1e12
            best = tops if best is None else max(best, tops)
    burst = {"tops": best, "iters_per_launch": iters, "clocks": sampler.summary()}
    per = int(max(256, min(1 << 22, iters * 50.0 / burst_ms)))
    n = int(max(1, sustained_s * 1e3 / 50.0))
    total = [0.0]

    def chain():
        for _ in range(n):
            total[0] += qk.qk_debug_int8_peak(per)

    sampler = ClockSampler(local)
    with sampler:
        ms = event_ms(chain, stream)
    qk.qk_check_device_error()
    sustained = {"tops": total[0] / (ms / 1e3) / 1e12, "seconds": ms / 1e3, "launches": n,
                 "clocks": sampler.summary()}
    return {"burst": burst, "sustained": sustained,
            "shape": "tcgen05.mma.cta_group::2.kind::i8 256x256x32, one CTA pair per two SMs"}


def measure_sustained(run, local, seconds, int8, peaks):
    """The call back to back for `seconds` (thermal / power steady state)."""
    import torch

    stream = torch.cuda.current_stream()
    ms1 = event_ms(lambda: [run.step(i) for i in range(10)], stream) / 10
    steps = int(max(20, seconds * 1e3 / max(ms1, 1e-3)))
    sampler = ClockSampler(local)
    with sampler:
        ms = event_ms(lambda: [run.step(i) for i in range(steps)], stream)
    run.qk.qk_check_device_error()
    value = run.ops * steps / (ms / 1e3) / 1e12
    out = {"seconds": ms / 1e3, "steps": steps, "ms_per_step": ms / steps, "value": value,
           "unit": "TOPS", "clocks": sampler.summary(),
           "frac_of_bf16_sustained_x2": value / (2.0 * peaks["bf16_sustained"])}
    if int8 is not None:
        out["frac_of_int8_probe_sustained"] = value / int8["sustained"]["tops"]
    return out


# Workloads of the `workloads` record of the default run: every configuration
# of the target (tiny, DiT attention projection, the M = 2048 sweep, the DiT
# MLP, W4A8 at M = 1 / 8 / 16 / 4096), the README's quick-start matmul, the
# gated residual epilogue and the INT8 attention.
TABLE = ["tiny", "dit_attn", "sweep_4096x4096", "sweep_4096x12288", "sweep_12288x4096",
         "sweep_thin_5120x48", "w4a8_m1", "w4a8_m8", "w4a8_m16", "w4a8_m4096",
         "quickstart_w8a8", "quickstart_w4a8", "w4a8_m4096_prepared", "quickstart_w4a8_prepared",
         "dit_mlp_gated", "sage_attn",
         "dit_mlp_fused", "dit_attn_fused", "quickstart_w8a8_fused"]


def table_entry(name, local, dev, peaks, int8):
    """One workload of the `workloads` record: per-call time and throughput,
    the dominant kernel alone and its roofline fraction."""
    import torch

    if is_attention(name):
        rec = attention_entry(name, local, dev, peaks, steps=5, warmup=3)
        torch.cuda.empty_cache()
        return rec
    run = LinearRun(name, dev)
    # size the timed region: graph-replayed small calls 200, else ~25 ms
    if run.M <= 256:
        steps = 200
    else:
        for i in range(3):
            run.step(i)
        est = event_ms(lambda: [run.step(i) for i in range(3)],
                       torch.cuda.current_stream()) / 3
        steps = int(max(10, min(400, 25.0 / max(est, 1e-3))))
    ms, k_ms, clocks, timing = time_linear(run, steps, 3, local)
    roof = roofline(run, k_ms, peaks, int8, name)
    per = ms / steps
    rec = {"config": run.case.name + ("_gated_residual" if run.gated else "")
                     + ("_one_kernel" if is_fused(name) else "")
                     + ("_prepared_weight" if is_prepared(name) else ""),
           "M": run.M, "K": run.K, "N": run.N, "steps": steps, "timing": timing,
           "ms_per_call": per, "value": run.ops / (per / 1e3) / 1e12, "unit": "TOPS",
           "pct_of_int8_spec": 100.0 * run.ops / (per / 1e3) / 1e12 / INT8_SPEC_TOPS,
           "kernel": roof["kernel"], "kernel_ms": k_ms,
           "roofline": {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                             "traffic")},
           "sm_mhz": clocks["sm_mhz"], "reasons": clocks["reasons"]}
    if run.w4 and run.M > 16 and roof["bound"] == "tensor":
        # the GEMM route runs int8 GEMMs on the digit rows of the weight: P per
        # weight row in tiles of 256 / P rows (64 for P = 3), or in the mixed
        # layout 256 digit rows per tile of 120 weight rows; the tensor pipe
        # does (digit rows / N) times the product's 2 M N K operations
        from w4a8_quantized_gemm_token_b200 import binding as qk

        _, s16, o16 = run.weights[0]
        planes, mixed = qk.qk_debug_w4a8_plane_count(s16, o16, run.K, with_mixed=True)
        rec["planes"] = planes
        rec["mixed_layout"] = bool(mixed)
        if 1 <= planes <= 3:
            tile = 120 if mixed else {1: 256, 2: 128, 3: 64}[planes]
            rows = (256 if mixed else planes * tile) * (-(-run.N // tile))
            rec["digit_rows"] = rows
            rec["tensor_ops_per_call"] = rows / run.N * run.ops
            rec["tensor_frac"] = rows / run.N * roof["achieved"] / roof["peak"]
    del run
    torch.cuda.empty_cache()
    return rec


def attention_entry(name, local, dev, peaks, steps, warmup, e2e_steps=0):
    """The INT8 attention (qk_sage_attention) on the quick-start shape."""
    import torch

    from w4a8_quantized_gemm_token_b200 import binding as qk

    case = get_case(name)
    B, H, L, D = case.B, case.H, case.L, case.D
    qb, kb, vb = case.draw()
    hosts = [torch.from_numpy(t.view(np.int16)).view(torch.bfloat16) for t in (qb, kb, vb)]
    del qb, kb, vb
    q, k, v = (t.to(dev) for t in hosts)  # 3 x 144 MB: each step reads more than the L2
    out = torch.empty_like(q)
    ws = torch.empty(qk.qk_sage_attention_workspace_size(B, H, L), dtype=torch.uint8, device=dev)
    flops = 4.0 * B * H * L * L * D
    stream = torch.cuda.current_stream()

    def step(i):
        qk.qk_sage_attention(q, k, v, out=out, workspace=ws)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    qk.qk_check_device_error()
    sampler = ClockSampler(local)
    barrier(dev)
    torch.cuda.synchronize()
    with sampler:
        ms = event_ms(lambda: [step(i) for i in range(steps)], stream)
    barrier(dev)
    qk.qk_check_device_error()
    # Roofline: Q K^T at the INT8 rate, P V at the bf16 rate (measured bf16 x 2 and
    # measured bf16); the bound is the sum of the two times.
    t_bound = (flops / 2) / (2 * peaks["bf16"] * 1e12) + (flops / 2) / (peaks["bf16"] * 1e12)
    per = ms / steps
    achieved = flops / (per / 1e3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": flops / t_bound / 1e12,
            "unit": "TFLOP/s",
            "peak_source": f"{peaks['source']} bf16_tflops (burst): Q K^T at x2 (INT8), P V at x1",
            "kernel": "sage_attn_kernel with its q/k quantization and v transpose (the call)",
            "traffic": None, "kernel_ms": per}
    roof["frac"] = roof["achieved"] / roof["peak"]
    rec = {"config": case.name, "B": B, "H": H, "L": L, "D": D, "steps": steps,
           "timing": "eager launches", "ms_per_call": per, "value": achieved,
           "unit": "TFLOP/s", "kernel": roof["kernel"], "kernel_ms": per,
           "roofline": {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                             "traffic")},
           "sm_mhz": sampler.summary()["sm_mhz"], "reasons": sampler.summary()["reasons"],
           "_roof": roof, "_clocks": sampler.summary(), "_ms": ms}
    if e2e_steps:
        pins = [t.pin_memory() for t in hosts]
        o_pin = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            for dst, src in zip((q, k, v), pins):
                dst.copy_(src, non_blocking=True)
            qk.qk_sage_attention(q, k, v, out=out, workspace=ws)
            o_pin.copy_(out, non_blocking=True)

        e2e_step()
        e_ms = event_ms(lambda: [e2e_step() for _ in range(e2e_steps)], stream)
        rec["_e2e_ms"] = e_ms
        rec["_e2e"] = {"h2d_bytes_per_step": 3 * q.numel() * 2,
                       "d2h_bytes_per_step": out.numel() * 2}
    return rec


def run_attention(args, world, rank, local):
    """`--workload sage_attn`: the INT8 attention as the bench line."""
    import torch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    n_e2e = 0 if args.no_e2e else max(3, min(args.steps, 5))
    rec = attention_entry(args.workload, local, dev, peaks, args.steps, args.warmup,
                          e2e_steps=n_e2e)
    case = get_case(args.workload)
    flops = 4.0 * case.B * case.H * case.L * case.L * case.D
    max_ms = reduce_max(rec["_ms"], dev)
    value = whole_job_value(flops, args.steps, world, max_ms / 1e3)
    e2e = None
    if n_e2e:
        e_ms = reduce_max(rec["_e2e_ms"], dev)
        e2e = {"value": whole_job_value(flops, n_e2e, world, e_ms / 1e3), "unit": "TFLOP/s",
               **rec["_e2e"], "steps": n_e2e, "ms_per_step": e_ms / n_e2e}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = attention_cpu_baseline(case, args.cpu_seconds)
    if rank == 0:
        line = {
            "metric": ATTN_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8 scores, bf16 P V", "data": "synthetic",
            "config": {"workload": case.name, "B": case.B, "H": case.H, "L": case.L,
                       "D": case.D,
                       "l2": "q, k, v of 144 MB each: every step reads more than the L2",
                       "timing": "eager launches",
                       "parallelism": f"replicas x{world} (no collective)"},
            "roofline": rec["_roof"], "e2e": e2e, "cpu_baseline": cpu, "clocks": rec["_clocks"],
            "gpu_launches": 4 * args.steps,
        }
        print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import torch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    run = LinearRun(args.workload, dev, args.sets)
    M, K, N, w4, gated = run.M, run.K, run.N, run.w4, run.gated
    peaks = load_peaks()

    # ---- the headline: `steps` calls, max over ranks
    ms, k_ms, clocks, timing = time_linear(run, args.steps, args.warmup, local, args.graph)
    max_ms = reduce_max(ms, dev)
    value = whole_job_value(run.ops, args.steps, world, max_ms / 1e3)

    # ---- the INT8 tensor-pipe probe (roofline denominator), burst right after;
    # the probe, the sustained record and the per-configuration record are
    # one-GPU measurements: replicas under torchrun skip them
    single = world == 1
    int8 = None
    if single and not args.no_peak_probe and not (w4 and M <= 16):
        int8 = measure_int8_peak(local, sustained_s=0.0 if args.no_sustained else 2.0)
    roof = roofline(run, k_ms, peaks, int8, args.workload)

    # ---- end to end through the public call, host buffers in and out
    e2e = None
    e2e_step = None
    if not args.no_e2e:
        stream = torch.cuda.current_stream()
        x_pin = run.x_host.pin_memory()
        y_pin = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
        x_dev = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        n_e2e = max(3, min(args.steps, args.e2e_steps))
        r_pin = run.res_host.pin_memory() if gated else None

        def e2e_step(i):
            x_dev.copy_(x_pin, non_blocking=True)
            wt = run.weights[i % run.nsets]
            if w4:
                run.qk.qk_w4a8_linear(x_dev, *wt, run.bias, y=run.y, workspace=run.ws)
            elif gated:
                run.res.copy_(r_pin, non_blocking=True)
                run.qk.qk_w8a8_linear_gated(x_dev, *wt, run.bias, run.gate, run.res, y=run.y,
                                            workspace=run.ws)
            else:
                run.qk.qk_w8a8_linear(x_dev, *wt, run.bias, y=run.y, workspace=run.ws)
            y_pin.copy_(run.y, non_blocking=True)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(dev)
        e_ms = reduce_max(event_ms(lambda: [e2e_step(i) for i in range(n_e2e)], stream), dev)
        e2e = {"value": whole_job_value(run.ops, n_e2e, world, e_ms / 1e3), "unit": "TOPS",
               "h2d_bytes_per_step": M * K * 2 + (M * N * 2 if gated else 0),
               "d2h_bytes_per_step": M * N * 2,
               "steps": n_e2e, "ms_per_step": e_ms / n_e2e}

    # ---- the same call back to back for seconds (power-capped steady state)
    sustained = None
    if single and not args.no_sustained and not w4 and M > 256:
        sustained = measure_sustained(run, local, 2.0, int8, peaks)
    launches = launches_per_call(M, K, N, w4, gated, run.qk, is_fused(args.workload),
                                 is_prepared(args.workload))
    config = {"workload": run.case.name + ("_gated_residual" if gated else "")
                          + ("_prepared_weight" if is_prepared(args.workload) else ""),
              "M": M, "K": K, "N": N,
              "weights": "W4 affine g64" if w4 else "W8 per-channel",
              "bias": run.bias is not None,
              "activations": "bf16 N(0,1)" + (", 1% channels x20" if run.case.outlier_frac else ""),
              "l2": f"{run.nsets} rotating input sets of {run.per_set / 1e6:.1f} MB; "
                    "one pass over them exceeds twice the 126 MB L2",
              "timing": timing, "parallelism": f"replicas x{world} (no collective)"}
    del run, e2e_step
    torch.cuda.empty_cache()

    # ---- every other configuration, each with its dominant kernel alone
    workloads = None
    if single and args.workload == "dit_mlp" and not args.no_workloads:
        workloads = {}
        for name in TABLE:
            try:
                workloads[name] = table_entry(name, local, dev, peaks, int8)
            except Exception as exc:  # reported in the line; the headline stands
                workloads[name] = {"error": f"{type(exc).__name__}: {exc}"}
                torch.cuda.empty_cache()
                continue
            for k in [k for k in workloads[name] if k.startswith("_")]:
                del workloads[name][k]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(get_case(args.workload), seconds=args.cpu_seconds, gated=gated)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8", "data": "synthetic", "config": config,
            "pct_of_int8_spec": 100.0 * value / world / INT8_SPEC_TOPS,
            "roofline": roof, "e2e": e2e, "cpu_baseline": cpu, "clocks": clocks,
            "gpu_launches": launches * args.steps,
            "int8_peak_probe": int8, "sustained": sustained, "workloads": workloads,
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ oracle legs

def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


class OracleSample:
    """Inputs for bounded oracle samples of a workload (same recipe as the GPU
    arm; only the first rows of x are drawn, since a sample never uses more)."""

    def __init__(self, case, w4, max_rows=1024, gated=False):
        import dataclasses

        import oracle
        from w4a8_quantized_gemm_token_b200 import synthetic

        self.case, self.w4, self.gated = case, w4, gated
        small = dataclasses.replace(case, M=min(case.M, max_rows))
        self.xb, W, self.b, _ = small.draw()
        if gated:
            self.gate, self.res = synthetic.gated_inputs(case, rows=small.M)
        if w4:
            self.Wp, self.s16, self.o16 = oracle.quant_w4(W)
        else:
            self.Wq, self.sw = oracle.quant_w8(W)

    @property
    def rows(self):
        return self.xb.shape[0]

    def run(self, rows, ncols):
        """Quantize `rows` activation rows and compute their outputs for the first
        `ncols` output channels.  Returns (seconds, ops)."""
        import oracle

        t0 = time.perf_counter()
        xq, sx = oracle.quant_act(self.xb[:rows])
        if self.w4:
            xsum = oracle.group_sums(xq)
            acc = oracle.w4a8_group_acc(xq, self.Wp[:ncols])
            oracle.w4a8_dequant(acc, xsum, sx, self.s16[:ncols], self.o16[:ncols], None)
        elif self.gated:
            acc = oracle.w8a8_acc(xq, self.Wq[:ncols])
            oracle.w8a8_gated(acc, sx, self.sw[:ncols], None if self.b is None else self.b[:ncols],
                              self.gate[:ncols], self.res[:rows, :ncols])
        else:
            acc = oracle.w8a8_acc(xq, self.Wq[:ncols])
            oracle.w8a8_dequant(acc, sx, self.sw[:ncols],
                                None if self.b is None else self.b[:ncols])
        return time.perf_counter() - t0, 2.0 * rows * ncols * self.case.K


def _oracle_leg(smp, seconds, threads):
    """Time the oracle over about `seconds` of rows with `threads` OpenMP
    threads (one row per thread to calibrate).  Returns (rows, s, ops, threads)."""
    import oracle

    got = oracle.set_threads(threads)
    try:
        probe = max(1, min(smp.rows, got))
        dt, _ = smp.run(probe, smp.case.N)
        rows = int(max(probe, min(smp.rows, probe * seconds / max(dt, 1e-6))))
        dt, ops = smp.run(rows, smp.case.N)
    finally:
        oracle.set_threads(1)
    return rows, dt, ops, min(got, rows)


def cpu_baseline(case, seconds=10.0, gated=False):
    """The oracle on the GPU machine's host cores, over bounded samples of the same
    workload: one thread, then every core (OpenMP over rows)."""
    ncores = host_cores()
    # enough rows that the all-core leg keeps every thread busy for its share
    smp = OracleSample(case, "w4a8" in case.name, gated=gated,
                       max_rows=int(min(case.M, max(1024, 64 * ncores))))
    r1, t1, o1, _ = _oracle_leg(smp, seconds / 2, 1)
    rn, tn, on, used = _oracle_leg(smp, seconds / 2, ncores)
    what = (f"of {case.M} rows x all {case.N} output channels (quant + exact int accumulate "
            f"+ fp64 dequant)")
    return {"value": on / tn / 1e12, "unit": "TOPS", "cores": used, "kind": "oracle",
            "sample": f"{rn} {what}, {used} OpenMP threads over rows, {tn:.1f} s",
            "nproc": ncores, "cpu_model": cpu_model(),
            "one_thread": {"value": o1 / t1 / 1e12, "unit": "TOPS", "cores": 1,
                           "sample": f"{r1} {what}, single thread, {t1:.1f} s"}}


def run_reference(args, world, rank, local):
    if rank != 0:
        return  # rank 0 alone runs the oracle
    import oracle

    case = get_case(args.workload)
    threads = oracle.set_threads(host_cores())
    oracle.set_threads(1)
    rows = max(1, min(case.M, threads))  # one row per thread in every step
    smp = OracleSample(case, is_w4(args.workload), max_rows=rows, gated=is_gated(args.workload))
    # size each step so that warm-up + timed steps take about `budget` seconds
    budget = args.ref_seconds
    oracle.set_threads(threads)
    try:
        dt1, _ = smp.run(rows, 8)
        dtn, _ = smp.run(rows, min(case.N, 64))
        per_col = max((dtn - dt1) / max(1, min(case.N, 64) - 8), 1e-9)
        per_step = budget / max(1, args.steps + args.warmup)
        ncols = int(max(8, min(case.N, per_step / per_col))) // 8 * 8
        for _ in range(args.warmup):
            smp.run(rows, ncols)
        t_total, ops_total = 0.0, 0.0
        for _ in range(args.steps):
            dt, ops = smp.run(rows, ncols)
            t_total += dt
            ops_total += ops
    finally:
        oracle.set_threads(1)
    value = ops_total / t_total / 1e12
    threads = min(threads, rows)  # the row loops give each thread one row at most
    sample = (f"per step: {rows} of {case.M} rows x {ncols} of {case.N} output channels "
              f"(quant + exact int accumulate + fp64 dequant), {threads} OpenMP threads over rows")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": case.name + ("_gated_residual" if is_gated(args.workload) else "")
                               + ("_prepared_weight" if is_prepared(args.workload) else ""),
                   "M": case.M, "K": case.K, "N": case.N},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": threads, "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def attention_cpu_baseline(case, seconds=10.0, threads=None):
    """The oracle on the host cores: sampled query rows of head 0 against every key."""
    import oracle

    threads = host_cores() if threads is None else threads
    qb, kb, vb = case.draw(heads=1)
    q, k, v = qb[0, 0], kb[0, 0], vb[0, 0]
    used = oracle.set_threads(threads)
    try:
        probe = max(2, used)
        t0 = time.perf_counter()
        oracle.sage_attention_rows(q, k, v, case.D ** -0.5, np.arange(probe))
        dt = max(time.perf_counter() - t0, 1e-6)
        rows = int(max(probe, min(case.L, probe * seconds / dt)))
        t0 = time.perf_counter()
        oracle.sage_attention_rows(q, k, v, case.D ** -0.5, np.arange(rows))
        dt = time.perf_counter() - t0
    finally:
        oracle.set_threads(1)
    ops = 4.0 * rows * case.L * case.D
    return {"value": ops / dt / 1e12, "unit": "TFLOP/s", "cores": used, "kind": "oracle",
            "sample": f"{rows} query rows of head 0 x all {case.L} keys (quantization of the "
                      f"head's q and k included), {used} OpenMP threads over rows, {dt:.1f} s",
            "cpu_model": cpu_model()}


def run_attention_reference(args, world):
    """The oracle's INT8 attention on the host cores, a bounded sample per step."""
    case = get_case(args.workload)
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    cpu = attention_cpu_baseline(case, seconds=budget)
    line = {
        "impl": "reference", "metric": ATTN_METRIC, "value": cpu["value"], "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 scores, fp64 softmax and P V", "data": "synthetic",
        "config": {"workload": case.name, "B": case.B, "H": case.H, "L": case.L, "D": case.D},
        "cpu_baseline": cpu,
        "e2e": {"value": cpu["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="dit_mlp")
    ap.add_argument("--sets", type=int, default=0,
                    help="rotating input sets (default: enough to exceed twice the L2)")
    ap.add_argument("--graph", choices=["auto", "on", "off"], default="auto",
                    help="replay the timed steps from a CUDA graph (auto: small M)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-configuration record of the default run")
    ap.add_argument("--no-sustained", action="store_true",
                    help="skip the seconds-long sustained records")
    ap.add_argument("--no-peak-probe", action="store_true",
                    help="skip the INT8 tensor-pipe probe (then bf16 x 2 is the denominator)")
    ap.add_argument("--probe-only", action="store_true",
                    help="run only the INT8 tensor-pipe probe and print its record")
    ap.add_argument("--cpu-seconds", type=float, default=16.0)
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world, rank, local = dist_env()
    if world != args.gpus and world != 1:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)

    if args.impl == "reference":
        if is_attention(args.workload):
            if rank == 0:
                run_attention_reference(args, world)
            return
        run_reference(args, world, rank, local)
        return

    import datetime

    import torch
    import torch.distributed as dist

    if args.probe_only:
        torch.cuda.set_device(local)
        print(json.dumps({"int8_peak_probe": measure_int8_peak(
            local, sustained_s=0.0 if args.no_sustained else 2.0)}), flush=True)
        return
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        if is_attention(args.workload):
            run_attention(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
