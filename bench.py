#!/usr/bin/env python
"""Throughput of the conv2d forward hot path on B200 -- prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole forward path over one batch of the workload:
output-size computation, the layout-in copy (NCHW -> channels-last, channels padded),
the implicit-GEMM tensor-core kernel (patch gather, weight tiles, product, bias
epilogue) and the NCHW output store -- one call of the C ABI's conv2d_forward.
The default workload is the ResNet-style 3x3 layer, 64x256x56x56 -> 256 channels,
stride 1, pad 1, bf16, channels-last: the largest configuration that runs on one
GPU (236.8 GFLOP per pass) and the one the >= 60%-of-dense-bf16 target is set on.
Other workloads: --workload NAME (see cnn_convolution_conv2d_b200/workloads.py).

Timing: W untimed warm-up steps, then exactly K steps, captured as CUDA graphs
of G steps each and replayed, bracketed by a barrier and a device synchronise on
both sides and timed with CUDA events on the launching stream (max over ranks).
Consecutive steps rotate over several input/output sets whose total size is more
than twice the 126 MB L2, so no step finds its input in L2.  The tensor-core
kernel is timed separately by events recorded around each of its launches.
SM clocks and throttle reasons are sampled through NVML during the timed region.

Multi-GPU (torchrun): every rank runs its own batch (different seed), nothing is
exchanged on the data path; `value` is the work of all ranks over the slowest
rank's time (weak scaling).

--impl reference times the CPU oracle (fp64, OpenMP) on bounded samples of the
same workload, as the comparison arm; on torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "resnet3x3_bf16_nhwc"
L2_BYTES = 126 * 1000 * 1000
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Dense TF32 over dense bf16 tensor throughput on B200 (nominal 1.125 / 2.25 PFLOP/s): only
# bf16 is measured, so the fp32 path's TF32 peak is the measured bf16 figure times this.
TF32_PER_BF16 = 0.5
# Tensor-core products per multiply-add of the fp32 path (a_hi*b_hi + a_hi*b_lo + a_lo*b_hi).
TF32_PRODUCTS = 3
# sources each measured kernel is built from (a change voids its committed ncu counters);
# "file:Struct" stands for that struct's definition alone (the kernel's parameter block in
# the shared header, whose other structs belong to other kernels)
KERNEL_SOURCES = {
    "igemm_kernel": ["igemm.cu", "epilogue.cuh", "ptx.cuh", "common.cuh:IgemmParams"],
    "gather_kernel": ["gather.cu", "epilogue.cuh", "ptx.cuh", "common.cuh:GatherParams"],
    "gather_t_kernel": ["gather_t.cu", "ptx.cuh", "common.cuh:GatherParams"],
    "dw_kernel": ["depthwise.cu", "ptx.cuh", "common.cuh:DwParams"],
}


# ------------------------------------------------------------ arithmetic ---
def flops(cfg) -> float:
    """Algorithmic FLOPs of one forward pass: 2*N*C_out*Ho*Wo*(C_in/groups)*Kh*Kw
    ("PyTorch高维张量乘法与conv2d/conv3d维度语义解析" §3.3); padding taps included,
    channel padding and split-K partial sums not."""
    return 2.0 * cfg.N * cfg.C_out * cfg.Ho * cfg.Wo * (cfg.C_in // cfg.groups) * cfg.Kh * cfg.Kw


def elt_bytes(cfg) -> int:
    return 2 if cfg.dtype == "bf16" else 4


def step_bytes(cfg) -> float:
    """Minimum bytes a whole step must move: x, w, bias read once, y written once."""
    e = elt_bytes(cfg)
    return e * (cfg.N * cfg.C_in * cfg.H * cfg.W + cfg.C_out * (cfg.C_in // cfg.groups) * cfg.Kh * cfg.Kw
                + (cfg.C_out if cfg.bias else 0) + cfg.N * cfg.C_out * cfg.Ho * cfg.Wo)


def padded_channels(cfg) -> int:
    align = 16 // elt_bytes(cfg)
    cg = cfg.C_in // cfg.groups
    return (cg + align - 1) // align * align


def uses_gather(cfg) -> bool:
    """Mirrors the library's choice of the software-gather kernel: one group, fewer
    than 32 bytes of input channels per pixel, a reduction that fits its tables."""
    e = elt_bytes(cfg)
    per16 = 16 // e
    vec = cfg.layout == "nchw" and cfg.dilation == 1 and (cfg.W * e) % 16 == 0 and cfg.Kw <= per16
    kc = cfg.C_in * cfg.Kh * (per16 if vec else cfg.Kw)
    kpad = -(-kc // (32 // e)) * (32 // e)
    return cfg.groups == 1 and cfg.C_in * e < 32 and kpad <= 256 and cfg.C_out <= (256 if e == 2 else 128)


def uses_depthwise(cfg) -> bool:
    """Mirrors the library's choice of the depthwise stencil kernel: groups = C_in = C_out."""
    return cfg.groups == cfg.C_in == cfg.C_out


def main_kernel_bytes(cfg) -> float:
    """Minimum bytes the tensor-core kernel itself moves per launch: its input (x
    itself for the gather kernel, else the channels-last input or its channel-padded
    copy when the step makes one), the packed weights, the bias, and the output."""
    e = elt_bytes(cfg)
    if uses_depthwise(cfg):  # x (or its channel-padded channels-last copy), one weight per tap and channel
        cp = -(-cfg.C_in // (16 // e)) * (16 // e)
        c_in = cp if (cfg.layout == "nchw" or cp != cfg.C_in) else cfg.C_in
        return e * (cfg.N * cfg.H * cfg.W * c_in + cfg.C_out * cfg.Kh * cfg.Kw + (cfg.C_out if cfg.bias else 0)
                    + cfg.N * cfg.C_out * cfg.Ho * cfg.Wo)
    cpg = padded_channels(cfg)
    copy = (cfg.layout == "nchw" or cpg != cfg.C_in // cfg.groups) and not uses_gather(cfg)
    x_in = cfg.N * cfg.H * cfg.W * (cfg.groups * cpg if copy else cfg.C_in)
    w = cfg.C_out * cfg.Kh * cfg.Kw * cpg
    return e * (x_in + w + (cfg.C_out if cfg.bias else 0) + cfg.N * cfg.C_out * cfg.Ho * cfg.Wo)


def xcol_bytes(cfg) -> float:
    """Bytes of the explicit X_col matrix: M rows of groups * Kh*Kw*Cpg elements."""
    return elt_bytes(cfg) * cfg.N * cfg.Ho * cfg.Wo * cfg.groups * cfg.Kh * cfg.Kw * padded_channels(cfg)


def explicit_kernel_bytes(cfg) -> float:
    """Minimum bytes of the tensor-core GEMM of the explicit path: X_col, packed
    weights, bias, output."""
    e = elt_bytes(cfg)
    w = cfg.C_out * cfg.Kh * cfg.Kw * padded_channels(cfg)
    return xcol_bytes(cfg) + e * (w + (cfg.C_out if cfg.bias else 0) + cfg.N * cfg.C_out * cfg.Ho * cfg.Wo)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, ValueError, KeyError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for entry in KERNEL_SOURCES[kernel]:
        name, _, struct = entry.partition(":")
        with open(os.path.join(ROOT, "cnn_convolution_conv2d_b200", "csrc", name), "rb") as f:
            data = f.read()
        if struct:
            start = data.index(b"struct " + struct.encode() + b" {")
            data = data[start:data.index(b"\n};", start) + 3]
        h.update(data)
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """DRAM traffic per launch of the tensor-core kernel from the committed ncu summary:
    dram__bytes_read.sum plus the larger of dram__bytes_write.sum and the L2's write
    bytes (lts__t_sectors_op_write.sum x 32) -- one launch's DRAM write count misses the
    output still held in L2 when the kernel ends, the L2-side count does not.  None when
    there is no entry or the kernel source changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f).get(workload)
    except (OSError, ValueError):
        return None
    if not d or d.get("kernel") not in KERNEL_SOURCES or d.get("kernel_hash") != kernel_source_hash(d["kernel"]):
        return None
    if "l2_write_bytes" not in d:
        return None
    scale = float(d.get("scale_to_full_launch", 1.0))
    return scale * (float(d["dram_bytes_read"]) + max(float(d["dram_bytes_write"]), float(d["l2_write_bytes"])))


KERNEL_LABELS = {
    "igemm": "igemm_kernel (implicit GEMM: TMA im2col/tiled loads, tcgen05; CTA pairs on large bf16 problems)",
    "gather": "gather_kernel (software-gathered im2col rows in tensor memory, tcgen05)",
    "gather_t": "gather_t_kernel (transposed product: output channels on the lanes, one output row per tile)",
    "depthwise": "dw_kernel (depthwise stencil over TMA-staged channels-last tiles, CUDA cores)",
}


def roofline(cfg, kernel_ms: float, peaks, peak_kind: str, workload: str, explicit: bool = False,
             plan_kernel: str | None = None) -> dict:
    f = flops(cfg)
    b = explicit_kernel_bytes(cfg) if explicit else main_kernel_bytes(cfg)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if cfg.dtype == "bf16" and f / b >= ridge:
        achieved = f / (kernel_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        out = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
               "peak_source": f"{peak_kind} bf16 sustained (kernel timed inside a long run)"}
    elif cfg.dtype == "f32" and TF32_PRODUCTS * f / b >= ridge * TF32_PER_BF16:
        # fp32 runs as three TF32 products per multiply-add: the tensor pipe executes 3x the
        # algorithmic FLOPs, against a TF32 peak of half the measured bf16 figure.
        achieved = TF32_PRODUCTS * f / (kernel_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"] * TF32_PER_BF16
        out = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
               "peak_source": (f"{peak_kind} bf16 sustained x {TF32_PER_BF16} (nominal dense TF32/bf16 ratio); "
                               f"achieved counts the {TF32_PRODUCTS} TF32 products per multiply-add"),
               "algorithmic_tflops": f / (kernel_ms * 1e-3) / 1e12,
               "executed_tf32_tflops": achieved}
    else:
        achieved = b / (kernel_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        out = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
               "peak_source": f"{peak_kind} HBM copy bandwidth"}
    out["frac"] = achieved / peak
    if plan_kernel is None:
        plan_kernel = "depthwise" if uses_depthwise(cfg) else "gather" if uses_gather(cfg) else "igemm"
    out["kernel"] = KERNEL_LABELS.get(plan_kernel, plan_kernel)
    out["kernel_ms"] = kernel_ms
    out["algorithmic_bytes_per_launch"] = b
    out["algorithmic_flops_per_launch"] = f
    out["traffic"] = None if explicit else committed_traffic(workload)
    if explicit:
        out["kernel"] = "igemm_kernel over the explicit X_col (tiled TMA loads, tcgen05)"
    return out


def with_write_context(rl: dict, cfg, kernel_ms: float, fill_gbs: float) -> dict:
    """Adds, for an HBM-bound kernel, the output bytes over the measured plain-fill
    write rate: no kernel that writes y can be faster than that."""
    if rl["bound"] == "hbm":
        y_bytes = cfg.N * cfg.C_out * cfg.Ho * cfg.Wo * elt_bytes(cfg)
        write_ms = y_bytes / (fill_gbs * 1e9) * 1e3
        rl["write_context"] = {"output_bytes": y_bytes, "fill_gbs": fill_gbs,
                               "output_write_ms_at_fill_rate": write_ms,
                               "frac_of_write_bound": write_ms / kernel_ms}
    return rl


# ---------------------------------------------------------------- clocks ---
class ClockSampler:
    """Polls SM clock and throttle reasons through NVML (what nvidia-smi reads)."""

    REASONS = {  # NVML clocks-event reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, interval_s: float = 0.005):
        self.samples = []
        self.interval = interval_s
        self.error = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # no NVML: report why instead of numbers
            self.error = f"NVML unavailable: {exc}"
            self.handle = None
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((t, mhz, reasons))
            except Exception as exc:
                self.error = str(exc)
                return
            time.sleep(self.interval)

    def start(self):
        if self.handle is not None:
            self._thread.start()

    def stop(self):
        self._stop.set()
        if self._thread.is_alive():
            self._thread.join()

    def summary(self, t0: float, t1: float) -> dict:
        if self.handle is None:
            return {"error": self.error}
        window = [s for s in self.samples if t0 <= s[0] <= t1]
        if not window:  # region shorter than one polling interval: nearest sample
            window = sorted(self.samples, key=lambda s: abs(s[0] - (t0 + t1) / 2))[:1]
        if not window:
            return {"error": self.error or "no samples"}
        mask = 0
        for s in window:
            mask |= s[2]
        reasons = [name for bit, name in self.REASONS.items() if mask & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in window), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(window)}


# ----------------------------------------------------------- distributed ---
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(cfg, rank: int) -> int:
    """Seed of a rank's batch: each rank draws a different batch of the same workload."""
    return cfg.seed + 1000 * rank


def weak_scaling_value(world: int, flop_per_rank_step: float, steps: int, max_elapsed_ms: float) -> float:
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's timed region."""
    return world * flop_per_rank_step * steps / (max_elapsed_ms * 1e-3) / 1e12


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ CPU oracle ---
def oracle_rate_sample(cfg, inp, seconds: float, seed: int = 1234, max_points=None):
    """Times the fp64 oracle on random output points of the workload for about
    `seconds`; returns (flop_per_s, points, wall_s, threads)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    shape = (cfg.N, cfg.C_out, cfg.Ho, cfg.Wo)
    per_point = 2.0 * (cfg.C_in // cfg.groups) * cfg.Kh * cfg.Kw
    x64 = inp["x"].astype(np.float64)
    w64 = inp["w"].astype(np.float64)
    b64 = None if inp["b"] is None else inp["b"].astype(np.float64)

    def run(points):
        idx = np.stack([rng.integers(0, n, points) for n in shape], axis=1)
        t = time.perf_counter()
        oracle.conv2d_points(x64, w64, b64, idx, cfg.stride, cfg.pad, cfg.dilation, cfg.groups)
        return time.perf_counter() - t

    probe = 2000
    dt = max(run(probe), 1e-4)
    points = int(probe * seconds / dt)
    total = cfg.N * cfg.C_out * cfg.Ho * cfg.Wo
    points = max(1, min(points, total, max_points or total))
    wall = run(points)
    return points * per_point / wall, points, wall, oracle.num_threads()


def capture_steps(cb, G, step, kev=None):
    """A CUDA graph of G steps (step(i) for i < G) and the library launches it holds; with
    kev, the library records kev[i] around step i's main kernel."""
    import torch
    launches0 = cb.conv2d_kernel_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(G):
            if kev is not None:
                cb.conv2d_set_main_kernel_events(*kev[i])
            step(i)
    cb.conv2d_set_main_kernel_events(None, None)
    launches = cb.conv2d_kernel_launch_count() - launches0
    graph.replay()  # one untimed replay: graph upload
    torch.cuda.synchronize()
    return graph, launches


def kernel_time_ms(step_ms, launches_per_step, graph_k, kev):
    """The main kernel's average launch time.  A step that is one library launch is timed by
    the events around the whole timed region (step_ms); otherwise the events the library
    records around the main kernel, in a separate replay of a graph holding them (each event
    pair adds a few microseconds, so this errs long)."""
    import torch
    if launches_per_step == 1:
        return step_ms, "one launch per step: events over the timed region / steps"
    graph_k.replay()
    torch.cuda.synchronize()
    return (statistics.fmean(a.elapsed_time(c) for a, c in kev),
            "events around the main kernel in a separate graph replay (each pair adds a few us)")


def run_reference(args, cfg):
    """The comparison arm: the oracle as it stands on this machine's host cores."""
    import numpy as np
    from cnn_convolution_conv2d_b200 import workloads
    inp = workloads.make_inputs(cfg)
    per_point = 2.0 * (cfg.C_in // cfg.groups) * cfg.Kh * cfg.Kw
    budget = 90.0 / max(1, args.steps + args.warmup)  # whole run: about a minute and a half
    rate, _, _, threads = oracle_rate_sample(cfg, inp, min(budget, 2.0))
    points = max(64, int(budget * rate / per_point))
    import oracle
    rng = np.random.default_rng(7)
    shape = (cfg.N, cfg.C_out, cfg.Ho, cfg.Wo)
    x64, w64 = inp["x"].astype(np.float64), inp["w"].astype(np.float64)
    b64 = None if inp["b"] is None else inp["b"].astype(np.float64)
    idx = [np.stack([rng.integers(0, n, points) for n in shape], axis=1)
           for _ in range(args.steps + args.warmup)]
    for i in range(args.warmup):
        oracle.conv2d_points(x64, w64, b64, idx[i], cfg.stride, cfg.pad, cfg.dilation, cfg.groups)
    t = time.perf_counter()
    for i in range(args.warmup, args.warmup + args.steps):
        oracle.conv2d_points(x64, w64, b64, idx[i], cfg.stride, cfg.pad, cfg.dilation, cfg.groups)
    wall = time.perf_counter() - t
    value = args.steps * points * per_point / wall / 1e12
    sample = (f"{points} random output points per step of {cfg.name} (drawn with replacement; "
              f"{points / (cfg.N * cfg.C_out * cfg.Ho * cfg.Wo):.3g} forward passes' worth of outputs), "
              f"fp64 on the host cores, no GPU")
    line = {
        "impl": "reference", "metric": metric_name(cfg), "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": wall / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, args, world=1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- our path ---
def metric_name(cfg) -> str:
    return "conv2d fwd TFLOP/s on 1 B200 and % of dense tensor (or HBM) roofline"


def workload_config(cfg, args, world: int) -> dict:
    desc = (f"{cfg.name}: N={cfg.N} C_in={cfg.C_in} {cfg.H}x{cfg.W} -> C_out={cfg.C_out}, "
            f"{cfg.Kh}x{cfg.Kw} s{cfg.stride} p{cfg.pad} d{cfg.dilation} g{cfg.groups}, "
            f"{'bias' if cfg.bias else 'no bias'}, {cfg.dtype}, {cfg.layout.upper()} in/out")
    return {"workload": desc, "global_batch": cfg.N * world, "per_gpu_batch": cfg.N,
            "flop_per_step_per_gpu": flops(cfg),
            "parallelism": f"replicas x{world} (batch shards, no collective on the data path)"}


def run_ours(args, cfg):
    import numpy as np
    import torch

    import cnn_convolution_conv2d_b200 as cb
    from cnn_convolution_conv2d_b200 import build, workloads

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    if rank == 0:
        build.build()
    barrier(world)
    cb.load()

    inp = workloads.make_inputs(cfg, seed=rank_seed(cfg, rank))
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    x_host = torch.from_numpy(inp["x"]).to(dt)
    if cfg.layout == "nhwc":
        x_host = x_host.permute(0, 2, 3, 1).contiguous()
    w = torch.from_numpy(inp["w"]).to(dt).to(device)
    b = None if inp["b"] is None else torch.from_numpy(inp["b"]).to(dt).to(device)
    layer = cb.Conv2dB200(w, b, cfg.stride, cfg.pad, cfg.dilation, cfg.groups, cfg.layout)
    y_shape = layer.out_shape(cfg.N, cfg.H, cfg.W)
    set_bytes = (x_host.numel() + math.prod(y_shape)) * x_host.element_size()
    nsets = max(2, min(16, math.ceil(2 * L2_BYTES / set_bytes) + 1))
    xs = [x_host.to(device) for _ in range(nsets)]
    ys = [torch.empty(y_shape, dtype=dt, device=device) for _ in range(nsets)]
    ex = args.explicit_im2col
    layer.workspace(cfg.N, cfg.H, cfg.W, ex)
    stream = torch.cuda.current_stream()

    for i in range(max(args.warmup, 3)):
        layer(xs[i % nsets], ys[i % nsets], explicit_im2col=ex)
    cb.conv2d_sync_status()

    # Steps per captured graph: a divisor of K, at most 512.
    G = 1
    for g in range(min(args.steps, 512), 0, -1):
        if args.steps % g == 0:
            G = g
            break
    reps = args.steps // G
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(G)]
    for a, c in kev:  # create the underlying events before capture
        a.record()
        c.record()
    torch.cuda.synchronize()
    if args.graph:
        # the timed graph holds no timing events (a pair per step would add a few us to each)
        def fstep(i):
            layer(xs[i % nsets], ys[i % nsets], explicit_im2col=ex)
        graph, launches_per_rep = capture_steps(cb, G, fstep)
        graph_k, _ = capture_steps(cb, G, fstep, kev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.05)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    launches_before = cb.conv2d_kernel_launch_count()
    t0 = time.perf_counter()
    ev0.record(stream)
    if args.graph:
        for _ in range(reps):
            graph.replay()
    else:
        for r in range(reps):
            for i in range(G):
                cb.conv2d_set_main_kernel_events(*kev[i])
                layer(xs[i % nsets], ys[i % nsets], explicit_im2col=ex)
        cb.conv2d_set_main_kernel_events(None, None)
    ev1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier(world)
    clocks.stop()
    cb.conv2d_sync_status()
    launches = (launches_per_rep * reps if args.graph
                else cb.conv2d_kernel_launch_count() - launches_before)
    elapsed_ms = max_over_ranks(ev0.elapsed_time(ev1), world, device)
    if args.graph:
        kernel_ms, ktiming = kernel_time_ms(ev0.elapsed_time(ev1) / args.steps, launches_per_rep / G, graph_k, kev)
    else:
        kernel_ms = statistics.fmean(a.elapsed_time(c) for a, c in kev)
        ktiming = "events around the main kernel, eager launches"
    kernel_ms = max_over_ranks(kernel_ms, world, device)
    ms_per_step = elapsed_ms / args.steps
    value = weak_scaling_value(world, flops(cfg), args.steps, elapsed_ms)

    # End to end through the host-buffer entry point: H2D of x, forward, D2H of y.
    x_pin = x_host.pin_memory()
    y_pin = torch.empty(y_shape, dtype=dt).pin_memory()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(3):
        layer.forward_hostio(x_pin, y_pin, xs[0], ys[0])
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        layer.forward_hostio(x_pin, y_pin, xs[0], ys[0])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    cb.conv2d_sync_status()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device) / e2e_steps
    e2e_value = weak_scaling_value(world, flops(cfg), 1, e2e_ms)

    # Context for memory-bound layers: how fast this GPU writes the output's bytes
    # at all (a plain device fill of the same buffer), since their traffic is mostly
    # writes, which the copy bandwidth of the roofline peak does not isolate.
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        ys[0].fill_(0.5)
    f0.record(stream)
    for _ in range(20):
        ys[0].fill_(0.5)
    f1.record(stream)
    torch.cuda.synchronize()
    fill_gbs = ys[0].numel() * ys[0].element_size() / (f0.elapsed_time(f1) / 20 * 1e-3) / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, points, wall, threads = oracle_rate_sample(cfg, inp, args.cpu_seconds)
        cpu = {"value": rate / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{points} random output points of one {cfg.name} forward pass "
                         f"({wall:.1f} s of fp64 CPU work)"}

    if rank == 0:
        peaks, peak_kind = load_peaks()
        plan = cb.conv2d_describe_plan(cfg.N, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.Kh, cfg.Kw, cfg.stride, cfg.pad,
                                       cfg.dilation, cfg.groups, cb.CONV_BF16 if cfg.dtype == "bf16" else cb.CONV_F32,
                                       cfg.layout, explicit_im2col=ex)
        cfgd = workload_config(cfg, args, world)
        cfgd["plan"] = plan
        cfgd["l2"] = (f"not resident: steps rotate over {nsets} input/output sets "
                      f"({nsets * set_bytes / 1e6:.0f} MB > 2x the 126 MB L2)")
        cfgd["launch"] = f"CUDA graphs of {G} steps x {reps} replays" if args.graph else "eager"
        if ex:
            cfgd["path"] = (f"explicit im2col + GEMM (conv2d_forward_im2col_gemm): X_col of "
                            f"{xcol_bytes(cfg) / 1e6:.1f} MB written and read back every step")
        line = {
            "metric": metric_name(cfg), "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic (seeded; x ~ N(0,1), He-scaled weights)",
            "config": cfgd,
            "roofline": dict(with_write_context(roofline(cfg, kernel_ms, peaks, peak_kind, cfg.name, ex,
                                                    plan_kernel=plan["kernel"]), cfg, kernel_ms, fill_gbs), kernel_timing=ktiming),
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
                    "d2h_bytes_per_step": math.prod(y_shape) * x_host.element_size(),
                    "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "api": "conv2d_forward_hostio (pinned host x -> device, forward, device y -> pinned host)"},
            "gpu_launches": launches,
            "clocks": clocks.summary(t0, t1),
        }
        print(json.dumps(line), flush=True)
    if args.graph:
        del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_backward(args, cfg):
    """Throughput of one backward pass on one GPU: --backward data (dx: the transposed
    convolution on the forward kernels, zero-inserted dy for stride > 1) or weight (dW
    and db: the pixel-reduction tensor-core product, or the CUDA-core kernel for few
    channels per group).  Same timing as the forward line: W warm-up steps, K steps in
    CUDA graphs, inputs rotated over sets larger than 2x L2, CUDA events on the stream
    and around the main kernel.  FLOPs are the gradient's algorithmic count, equal to
    the forward pass's (pwwt §3.3's formula)."""
    import torch
    import cnn_convolution_conv2d_b200 as cb
    from cnn_convolution_conv2d_b200 import build, workloads

    build.build()
    cb.load()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    inp = workloads.make_inputs(cfg)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    x_host = torch.from_numpy(inp["x"]).to(dt)
    if cfg.layout == "nhwc":
        x_host = x_host.permute(0, 2, 3, 1).contiguous()
    w = torch.from_numpy(inp["w"]).to(dt).to(device)
    b = None if inp["b"] is None else torch.from_numpy(inp["b"]).to(dt).to(device)
    layer = cb.Conv2dB200(w, b, cfg.stride, cfg.pad, cfg.dilation, cfg.groups, cfg.layout)
    y_shape = layer.out_shape(cfg.N, cfg.H, cfg.W)
    g = torch.Generator().manual_seed(cfg.seed + 500)
    dy_host = torch.randn(y_shape, generator=g).to(dt)
    set_bytes = (x_host.numel() + dy_host.numel()) * x_host.element_size()
    nsets = max(2, min(16, math.ceil(2 * L2_BYTES / set_bytes) + 1))
    dys = [dy_host.to(device) for _ in range(nsets)]
    if args.backward == "data":
        outs = [torch.empty(x_host.shape, dtype=dt, device=device) for _ in range(nsets)]

        def step(i):
            layer.backward_data(dys[i % nsets], cfg.H, cfg.W, dx=outs[i % nsets])
    else:
        xs = [x_host.to(device) for _ in range(nsets)]
        dw = torch.empty(tuple(w.shape), dtype=dt, device=device)
        db = None if b is None else torch.empty(cfg.C_out, dtype=dt, device=device)

        def step(i):
            layer.backward_weight(xs[i % nsets], dys[i % nsets], dw=dw, db=db)
    for i in range(max(args.warmup, 3)):
        step(i)
    cb.conv2d_sync_status()
    G = 1
    for gsz in range(min(args.steps, 256), 0, -1):
        if args.steps % gsz == 0:
            G = gsz
            break
    reps = args.steps // G
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(G)]
    for a, c in kev:
        a.record()
        c.record()
    torch.cuda.synchronize()
    # the timed graph holds no timing events (a pair per step would add a few us to each)
    graph, launches_per_rep = capture_steps(cb, G, step)
    graph_k, _ = capture_steps(cb, G, step, kev)
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.05)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ev0.record(stream)
    for _ in range(reps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    clocks.stop()
    cb.conv2d_sync_status()
    elapsed = ev0.elapsed_time(ev1)
    kernel_ms, ktiming = kernel_time_ms(elapsed / args.steps, launches_per_rep / G, graph_k, kev)
    f = flops(cfg)
    peaks, peak_kind = load_peaks()
    plan = cb.conv2d_describe_plan(cfg.N, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.Kh, cfg.Kw, cfg.stride, cfg.pad,
                                   cfg.dilation, cfg.groups, cb.CONV_BF16 if cfg.dtype == "bf16" else cb.CONV_F32,
                                   cfg.layout)
    executed = f * (cfg.stride ** 2 if args.backward == "data" else 1)
    achieved = executed / (kernel_ms * 1e-3) / 1e12
    if cfg.dtype == "bf16":
        peak, ksrc = peaks["bf16_tflops_sustained"], f"{peak_kind} bf16 sustained"
    else:
        achieved *= TF32_PRODUCTS
        peak, ksrc = peaks["bf16_tflops_sustained"] * TF32_PER_BF16, f"{peak_kind} bf16 sustained x {TF32_PER_BF16}"
    line = {
        "metric": f"conv2d backward-{args.backward} TFLOP/s on 1 B200 and % of dense tensor roofline",
        "value": f * args.steps / (elapsed * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded; dy ~ N(0,1))",
        "config": {"workload": workload_config(cfg, args, 1)["workload"], "pass": args.backward,
                   "l2": f"not resident: steps rotate over {nsets} sets ({nsets * set_bytes / 1e6:.0f} MB)",
                   "launch": f"CUDA graphs of {G} steps x {reps} replays", "forward_plan": plan},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": ksrc, "kernel_ms": kernel_ms, "kernel_timing": ktiming,
                     "algorithmic_flops_per_launch": f,
                     "executed_flops_per_launch": executed, "traffic": None,
                     "kernel": ("igemm_kernel / dw_kernel on the transposed convolution" if args.backward == "data"
                                else "wgrad_kernel (pixel-reduction tcgen05 product, MN-major operands)"
                                if (cfg.C_in // cfg.groups) * elt_bytes(cfg) >= 32
                                else "wgrad_direct_kernel (CUDA cores)")},
        "gpu_launches": launches_per_rep * reps,
        "clocks": clocks.summary(t0, t1),
    }
    print(json.dumps(line), flush=True)
    del graph


def run_conv3d(args, cfg):
    """Throughput of the 3-D forward pass (conv3d_forward) on one GPU, with the forward
    line's timing: W warm-up steps, K steps in CUDA graphs, inputs rotated over sets
    larger than 2x L2, CUDA events on the stream and around the tensor-core kernel.
    FLOPs = 2*N*C_out*Do*Ho*Wo*(C_in/groups)*Kd*Kh*Kw (pwwt §3.3's count, one more
    spatial factor)."""
    import torch
    import cnn_convolution_conv2d_b200 as cb
    from cnn_convolution_conv2d_b200 import build, workloads

    build.build()
    cb.load()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    inp = workloads.make_inputs3d(cfg)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    x_host = torch.from_numpy(inp["x"]).to(dt)
    if cfg.layout == "nhwc":
        x_host = x_host.permute(0, 2, 3, 4, 1).contiguous()
    w = torch.from_numpy(inp["w"]).to(dt).to(device)
    b = None if inp["b"] is None else torch.from_numpy(inp["b"]).to(dt).to(device)
    layer = cb.Conv3dB200(w, b, cfg.stride, cfg.pad, cfg.dilation, cfg.groups, cfg.layout)
    y_shape = layer.out_shape(cfg.N, cfg.D, cfg.H, cfg.W)
    set_bytes = (x_host.numel() + math.prod(y_shape)) * x_host.element_size()
    nsets = max(2, min(16, math.ceil(2 * L2_BYTES / set_bytes) + 1))
    xs = [x_host.to(device) for _ in range(nsets)]
    ys = [torch.empty(y_shape, dtype=dt, device=device) for _ in range(nsets)]
    for i in range(max(args.warmup, 3)):
        layer(xs[i % nsets], ys[i % nsets])
    cb.conv2d_sync_status()
    G = 1
    for gsz in range(min(args.steps, 256), 0, -1):
        if args.steps % gsz == 0:
            G = gsz
            break
    reps = args.steps // G
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(G)]
    for a, c in kev:
        a.record()
        c.record()
    torch.cuda.synchronize()
    # the timed graph holds no timing events (a pair per step would add a few us to each)
    def lstep(i):
        layer(xs[i % nsets], ys[i % nsets])
    graph, launches_per_rep = capture_steps(cb, G, lstep)
    graph_k, _ = capture_steps(cb, G, lstep, kev)
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.05)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ev0.record(stream)
    for _ in range(reps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    clocks.stop()
    cb.conv2d_sync_status()
    elapsed = ev0.elapsed_time(ev1)
    kernel_ms, ktiming = kernel_time_ms(elapsed / args.steps, launches_per_rep / G, graph_k, kev)
    e = elt_bytes(cfg)
    f = 2.0 * cfg.N * cfg.C_out * cfg.Do * cfg.Ho * cfg.Wo * (cfg.C_in // cfg.groups) * cfg.Kd * cfg.Kh * cfg.Kw
    nbytes = e * (cfg.N * cfg.C_in * cfg.D * cfg.H * cfg.W + cfg.C_out * (cfg.C_in // cfg.groups) * cfg.Kd * cfg.Kh
                  * cfg.Kw + (cfg.C_out if cfg.bias else 0) + cfg.N * cfg.C_out * cfg.Do * cfg.Ho * cfg.Wo)
    peaks, peak_kind = load_peaks()
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    mult = 1 if cfg.dtype == "bf16" else TF32_PRODUCTS
    tpeak = peaks["bf16_tflops_sustained"] * (1 if cfg.dtype == "bf16" else TF32_PER_BF16)
    if mult * f / nbytes >= ridge * tpeak / peaks["bf16_tflops_sustained"]:
        achieved = mult * f / (kernel_ms * 1e-3) / 1e12
        rl = {"bound": "tensor", "achieved": achieved, "peak": tpeak, "unit": "TFLOP/s", "frac": achieved / tpeak,
              "peak_source": f"{peak_kind} bf16 sustained" + ("" if mult == 1 else f" x {TF32_PER_BF16}, x3 products")}
    else:
        achieved = nbytes / (kernel_ms * 1e-3) / 1e9
        rl = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
              "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peak_kind} HBM copy bandwidth"}
    plan = cb.conv3d_describe_plan(cfg.N, cfg.C_in, cfg.D, cfg.H, cfg.W, cfg.C_out, cfg.Kd, cfg.Kh, cfg.Kw,
                                   cfg.stride, cfg.pad, cfg.dilation, cfg.groups,
                                   cb.CONV_BF16 if cfg.dtype == "bf16" else cb.CONV_F32, cfg.layout)
    if plan["fold"]:
        kname = ("igemm_kernel on the (kd, kh)-folded input (2-D TMA im2col of 1 x Kw, tcgen05); the fold and "
                 "weight passes are outside kernel_ms, inside ms_per_step")
    elif plan["kernel"] == "vol_reuse":
        kname = "vol_reuse_kernel (5-D TMA im2col, each input slice loaded once for all depth taps, tcgen05)"
    else:
        kname = "igemm_kernel (5-D TMA im2col, tcgen05)"
    rl.update({"kernel": kname, "kernel_ms": kernel_ms, "kernel_timing": ktiming, "plan": plan,
               "algorithmic_flops_per_launch": f, "algorithmic_bytes_per_launch": nbytes, "traffic": None,
               "step_frac": (rl["achieved"] * kernel_ms / (elapsed / args.steps)) / rl["peak"]})
    desc = (f"{cfg.name}: N={cfg.N} C_in={cfg.C_in} {cfg.D}x{cfg.H}x{cfg.W} -> C_out={cfg.C_out}, "
            f"{cfg.Kd}x{cfg.Kh}x{cfg.Kw} s{cfg.stride} p{cfg.pad} d{cfg.dilation} g{cfg.groups}, {cfg.dtype}, "
            f"{'NDHWC' if cfg.layout == 'nhwc' else 'NCDHW'} in/out")
    line = {
        "metric": "conv3d fwd TFLOP/s on 1 B200 and % of dense tensor (or HBM) roofline",
        "value": f * args.steps / (elapsed * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded; x ~ N(0,1), He-scaled weights)",
        "config": {"workload": desc, "l2": f"not resident: steps rotate over {nsets} sets",
                   "launch": f"CUDA graphs of {G} steps x {reps} replays"},
        "roofline": rl, "gpu_launches": launches_per_rep * reps, "clocks": clocks.summary(t0, t1),
    }
    print(json.dumps(line), flush=True)
    del graph


def run_winograd(args, cfg):
    """Throughput of the Winograd forward pass F(m x m, 3 x 3) (conv2d_forward_winograd)
    on one GPU for a 3x3 stride-1 workload, with the forward line's timing.  `value` counts
    the convolution's algorithmic FLOPs (as every forward line); the roofline is the
    transformed-domain product (the (m+2)^2 channel GEMMs on the tensor cores) against the
    tensor peak, and the step's bytes (x, V and M written and read, y) against HBM."""
    import numpy as np
    import torch
    import cnn_convolution_conv2d_b200 as cb
    from cnn_convolution_conv2d_b200 import build, workloads
    import oracle

    m = args.winograd
    if (cfg.Kh, cfg.Kw, cfg.stride, cfg.dilation, cfg.groups) != (3, 3, 1, 1, 1):
        raise SystemExit("--winograd needs a 3x3, stride-1, unit-dilation, ungrouped workload")
    build.build()
    cb.load()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    inp = workloads.make_inputs(cfg)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    x_host = torch.from_numpy(inp["x"]).to(dt)
    if cfg.layout == "nhwc":
        x_host = x_host.permute(0, 2, 3, 1).contiguous()
    w = torch.from_numpy(inp["w"]).to(dt).to(device)
    b = None if inp["b"] is None else torch.from_numpy(inp["b"]).to(dt).to(device)
    layer = cb.WinogradConv2dB200(w, b, cfg.pad, m, cfg.layout)
    y_shape = (cfg.N, cfg.Ho, cfg.Wo, cfg.C_out) if cfg.layout == "nhwc" else (cfg.N, cfg.C_out, cfg.Ho, cfg.Wo)
    set_bytes = (x_host.numel() + math.prod(y_shape)) * x_host.element_size()
    nsets = max(2, min(16, math.ceil(2 * L2_BYTES / set_bytes) + 1))
    xs = [x_host.to(device) for _ in range(nsets)]
    ys = [torch.empty(y_shape, dtype=dt, device=device) for _ in range(nsets)]
    for i in range(max(args.warmup, 3)):
        layer(xs[i % nsets], ys[i % nsets])
    cb.conv2d_sync_status()
    # accuracy of this run against the oracle on sampled outputs (the transforms' rounding)
    idx = np.stack([np.random.default_rng(5).integers(0, n, 2048) for n in (cfg.N, cfg.C_out, cfg.Ho, cfg.Wo)], 1)
    yy = ys[0].float()
    got = (yy[tuple(torch.from_numpy(idx[:, i]).to(device) for i in (0, 2, 3, 1))] if cfg.layout == "nhwc"
           else yy[tuple(torch.from_numpy(idx[:, i]).to(device) for i in range(4))]).cpu().numpy()
    ref = oracle.conv2d_points(inp["x"], inp["w"], inp["b"], idx, 1, cfg.pad, 1, 1)
    err = {"max_abs_over_max_ref": float(np.abs(got - ref).max() / np.abs(ref).max()),
           "normwise_sampled": float(np.linalg.norm(got - ref) / np.linalg.norm(ref)), "points": 2048}
    G = 1
    for gsz in range(min(args.steps, 256), 0, -1):
        if args.steps % gsz == 0:
            G = gsz
            break
    reps = args.steps // G
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(G)]
    for a, c in kev:
        a.record()
        c.record()
    torch.cuda.synchronize()
    # the timed graph holds no timing events (a pair per step would add a few us to each)
    def lstep(i):
        layer(xs[i % nsets], ys[i % nsets])
    graph, launches_per_rep = capture_steps(cb, G, lstep)
    graph_k, _ = capture_steps(cb, G, lstep, kev)
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.05)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ev0.record(stream)
    for _ in range(reps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    clocks.stop()
    cb.conv2d_sync_status()
    elapsed = ev0.elapsed_time(ev1)
    kernel_ms, ktiming = kernel_time_ms(elapsed / args.steps, launches_per_rep / G, graph_k, kev)
    a2 = (m + 2) ** 2
    tiles = cfg.N * (-(-cfg.Ho // m)) * (-(-cfg.Wo // m))
    e = elt_bytes(cfg)
    cpg = -(-cfg.C_in // (16 // e)) * (16 // e)
    gemm_flops = 2.0 * a2 * tiles * cpg * cfg.C_out
    mult = 1 if cfg.dtype == "bf16" else TF32_PRODUCTS
    peaks, peak_kind = load_peaks()
    tpeak = peaks["bf16_tflops_sustained"] * (1 if cfg.dtype == "bf16" else TF32_PER_BF16)
    v_bytes = tiles * a2 * cpg * e
    m_bytes = tiles * a2 * cfg.C_out * 4
    step_b = step_bytes(cfg) + 2 * v_bytes + 2 * m_bytes
    # the product reads V and the transformed filters once and writes M once: bound by
    # whichever of its FLOPs and bytes takes longer at the measured peaks
    prod_bytes = v_bytes + m_bytes + a2 * cfg.C_out * cpg * e
    prod_plan = cb.conv2d_winograd_describe_plan(cfg.N, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.pad, m,
                                                 cb.CONV_BF16 if cfg.dtype == "bf16" else cb.CONV_F32, cfg.layout)
    hbm_bound = prod_bytes / (peaks["hbm_gbs"] * 1e9) > mult * gemm_flops / (tpeak * 1e12)
    if hbm_bound:
        ach, pk, unit = prod_bytes / (kernel_ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
        psrc = f"{peak_kind} HBM copy bandwidth"
    else:
        ach, pk, unit = mult * gemm_flops / (kernel_ms * 1e-3) / 1e12, tpeak, "TFLOP/s"
        psrc = f"{peak_kind} bf16 sustained" + ("" if mult == 1 else " x 0.5")
    line = {
        "metric": "conv2d fwd TFLOP/s on 1 B200 and % of dense tensor (or HBM) roofline",
        "value": flops(cfg) * args.steps / (elapsed * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded)",
        "config": {"workload": workload_config(cfg, args, 1)["workload"], "path": f"Winograd F({m}x{m},3x3)",
                   "l2": f"not resident: steps rotate over {nsets} sets",
                   "launch": f"CUDA graphs of {G} steps x {reps} replays"},
        "roofline": {"bound": "hbm" if hbm_bound else "tensor", "achieved": ach, "peak": pk, "unit": unit,
                     "frac": ach / pk, "peak_source": psrc,
                     "kernel": ("pw_kernel" if prod_plan["kernel"] == "pointwise" else "igemm_kernel")
                     + " on the transformed tiles ((m+2)^2 groups of 1x1)",
                     "kernel_ms": kernel_ms, "kernel_timing": ktiming, "gemm_flops_per_launch": gemm_flops,
                     "product_bytes_per_launch": prod_bytes,
                     "tensor_frac": mult * gemm_flops / (kernel_ms * 1e-3) / 1e12 / tpeak, "traffic": None,
                     "multiplies_vs_direct": a2 / (m * m * 9.0),
                     "step_bytes": step_b, "step_hbm_frac": step_b / (elapsed / args.steps * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "accuracy_vs_oracle": err,
        "gpu_launches": launches_per_rep * reps, "clocks": clocks.summary(t0, t1),
    }
    print(json.dumps(line), flush=True)
    del graph


def run_transpose(args, cfg):
    """Bandwidth of the standalone layout kernels on this workload's tensors: x NCHW ->
    channels-last (channel-padded per group), and y channels-last -> NCHW.  One GPU;
    buffers rotate over sets larger than 2x L2; CUDA events; bytes = read + write once."""
    import torch
    import cnn_convolution_conv2d_b200 as cb
    from cnn_convolution_conv2d_b200 import build

    build.build()
    cb.load()
    device = torch.device("cuda", 0)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    dcode = cb.CONV_BF16 if cfg.dtype == "bf16" else cb.CONV_F32
    e = elt_bytes(cfg)
    cpg = padded_channels(cfg)
    peaks, peak_kind = load_peaks()
    lines = {}
    cases = [("nchw_to_nhwc", cfg.N * cfg.C_in * cfg.H * cfg.W, cfg.N * cfg.H * cfg.W * cfg.groups * cpg,
              lambda s_, d_: cb.conv2d_nchw_to_nhwc(s_, d_, cfg.N, cfg.C_in, cfg.H, cfg.W, cfg.groups, cpg, dcode)),
             ("nhwc_to_nchw", cfg.N * cfg.C_out * cfg.Ho * cfg.Wo, cfg.N * cfg.C_out * cfg.Ho * cfg.Wo,
              lambda s_, d_: cb.conv2d_nhwc_to_nchw(s_, d_, cfg.N, cfg.C_out, cfg.Ho, cfg.Wo, dcode))]
    for name, n_in, n_out, fn in cases:
        nsets = max(2, min(16, math.ceil(2 * L2_BYTES / ((n_in + n_out) * e)) + 1))
        srcs = [torch.randn(n_in, device=device).to(dt) for _ in range(nsets)]
        dsts = [torch.empty(n_out, dtype=dt, device=device) for _ in range(nsets)]
        for i in range(max(args.warmup, 3)):
            fn(srcs[i % nsets], dsts[i % nsets])
        cb.conv2d_sync_status()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        steps = max(1, min(args.steps, 2000))
        a.record()
        for i in range(steps):
            fn(srcs[i % nsets], dsts[i % nsets])
        b.record()
        torch.cuda.synchronize()
        cb.conv2d_sync_status()
        ms = a.elapsed_time(b) / steps
        gbs = (n_in + n_out) * e / (ms * 1e-3) / 1e9
        lines[name] = {"us_per_launch": ms * 1e3, "bytes_per_launch": (n_in + n_out) * e, "achieved_gbs": gbs,
                       "frac_of_hbm_peak": gbs / peaks["hbm_gbs"], "sets": nsets, "launches": steps}
    print(json.dumps({"metric": "layout transpose GB/s on 1 B200 and % of HBM copy bandwidth",
                      "workload": cfg.name, "peak_gbs": peaks["hbm_gbs"], "peak_source": f"{peak_kind} HBM copy bandwidth",
                      **lines}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-graph", dest="graph", action="store_false")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--explicit-im2col", action="store_true",
                    help="time the pages' formulation: explicit X_col in HBM, then the GEMM")
    ap.add_argument("--transpose", action="store_true",
                    help="time the standalone NCHW<->NHWC kernels on the workload's x and y instead")
    ap.add_argument("--backward", choices=["data", "weight"],
                    help="time one backward pass (input or weight gradient) of the workload instead")
    ap.add_argument("--winograd", type=int, choices=[2, 4],
                    help="time the Winograd F(m x m, 3 x 3) forward pass of a 3x3 stride-1 workload instead")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from cnn_convolution_conv2d_b200 import workloads
    if args.workload in workloads.CONFIGS3D:
        if args.impl != "ours" or args.gpus != 1:
            ap.error("3-D workloads run on one GPU through this library")
        run_conv3d(args, workloads.CONFIGS3D[args.workload])
        return
    cfg = workloads.CONFIGS[args.workload]
    rank, world, _ = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, cfg)
        return
    if args.transpose:
        if world != 1:
            ap.error("--transpose runs on one GPU")
        run_transpose(args, cfg)
        return
    if args.backward:
        if world != 1:
            ap.error("--backward runs on one GPU")
        run_backward(args, cfg)
        return
    if args.winograd:
        if world != 1:
            ap.error("--winograd runs on one GPU")
        run_winograd(args, cfg)
        return
    run_ours(args, cfg)


if __name__ == "__main__":
    main()
