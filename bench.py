#!/usr/bin/env python3
"""Benchmark: implicit-GEMM convolution forward on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one convolution forward pass (the whole hot path: one kernel
launch) over one batch of the workload, inputs already resident in HBM.
Between timed steps the inputs rotate over enough independent buffer sets to
exceed twice the L2 cache, so every step reads x and w from DRAM.

Metric: conv fwd TFLOP/s, FLOPs = 2 * N * Do * Ho * Wo * O * kD * kH * kW * C/groups
(the "Convolutions" tutorial's count, section 4, extended to batch, depth and
groups); also the fraction of the B200's dense fp16/bf16 tensor peak.

With N > 1 GPUs (torchrun, one process per GPU) every rank runs the same
workload on its own device (independent batches: weak scaling, no data-path
collective); the time is the maximum over ranks and the value counts the
FLOPs of all ranks.

--impl reference times the CPU oracle (fp64 direct loop, the test-suite's
checker) on the host cores over a bounded sample of the workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as WL  # noqa: E402

METRIC = "conv fwd TFLOP/s (fp16/bf16) and % of B200 dense tensor peak, 1 GPU"
SPEC_DENSE_TFLOPS = 2250.0          # B200 dense fp16/bf16, datasheet
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_DIR = os.path.join(ROOT, "profiles")


# ---------------------------------------------------------------- counting

def out_dims(wl, pad_hi=None, via_oracle=False):
    """Output extents from the library, or from the oracle on the CPU arms
    (which must not load the library)."""
    if via_oracle:
        import oracle as C
        if wl.transpose:
            return C.convT_out_dims(wl.D, wl.H, wl.W, *wl.k, wl.stride, wl.pad, wl.out_pad, wl.dil)
        return C.out_dims(wl.D, wl.H, wl.W, *wl.k, wl.stride, wl.pad, wl.dil, pad_hi)
    import implicit_gemm_convolution_conv2d_b200 as C
    if wl.transpose:
        return C.transpose_out_dims(wl.D, wl.H, wl.W, *wl.k, wl.stride, wl.pad, wl.out_pad, wl.dil)
    return C.out_dims(wl.D, wl.H, wl.W, *wl.k, wl.stride, wl.pad, wl.dil, pad_hi)


def conv_flops(wl, dims=None, via_oracle=False):
    """Algorithmic FLOPs: 2 * N * Do*Ho*Wo * O * kD*kH*kW * C/groups (padding taps counted).
    A transposed convolution counts those of the forward pass it is the adjoint
    of: 2 * N * D*H*W (its input pixels) * C * kD*kH*kW * O/groups."""
    if wl.transpose:
        return 2 * wl.N * wl.D * wl.H * wl.W * wl.C * wl.k[0] * wl.k[1] * wl.k[2] * (wl.O // wl.groups)
    Do, Ho, Wo = dims if dims is not None else out_dims(wl, via_oracle=via_oracle)
    return 2 * wl.N * Do * Ho * Wo * wl.O * wl.k[0] * wl.k[1] * wl.k[2] * (wl.C // wl.groups)


def conv_bytes(wl, dims=None):
    """Algorithmic bytes: x, w and y each moved once (the tutorial's intensity convention)."""
    Do, Ho, Wo = dims if dims is not None else out_dims(wl)
    e = WL.ELEM_BYTES[wl.dtype]
    nx = wl.N * wl.D * wl.H * wl.W * wl.C
    nw = wl.O * wl.k[0] * wl.k[1] * wl.k[2] * (wl.C // wl.groups)
    ny = wl.N * Do * Ho * Wo * wl.O
    return e * nx, e * nw, e * ny


# ---------------------------------------------------------------- peaks / profiles

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Device and host source files each kernel variant's behaviour depends on: a
# traffic record taken with ncu stays valid while these files are unchanged. Each
# set holds every local header its headers include.
_COMMON_SRC = ["conv_fwd.cu", "ptx.cuh", "conv_tc.cuh", "launch.cuh"]
KERNEL_SOURCES = {
    "tcgen05_tma_im2col": _COMMON_SRC,
    "tcgen05_tma_im2col_pair": _COMMON_SRC,
    "tcgen05_gather": _COMMON_SRC,
    "tcgen05_tma_im2col_t": _COMMON_SRC + ["conv_tct.cuh"],
    "tcgen05_tma_halo": _COMMON_SRC + ["conv_halo.cuh"],
    "tcgen05_tma_halo_pair": _COMMON_SRC + ["conv_halo.cuh"],
    "tcgen05_tma_halo_t": _COMMON_SRC + ["conv_halo.cuh", "conv_tct.cuh", "conv_halo_t.cuh"],
    "tcgen05_tma_halo_t_pair": _COMMON_SRC + ["conv_halo.cuh", "conv_tct.cuh", "conv_halo_t.cuh"],
    "tcgen05_tma_phase": _COMMON_SRC + ["conv_tct.cuh", "conv_phase.cuh"],
    "simt_ffma": ["conv_fwd.cu", "conv_simt.cuh", "ptx.cuh", "launch.cuh"],
    "depthwise_tma": _COMMON_SRC + ["conv_simt.cuh", "conv_dw.cuh"],
    "depthwise_direct": ["conv_fwd.cu", "conv_simt.cuh", "conv_dw.cuh", "conv_tc.cuh", "ptx.cuh", "launch.cuh"],
    "simt_wgrad": ["conv_wgrad.cu", "conv_wgrad.cuh", "conv_simt.cuh", "ptx.cuh", "launch.cuh"],
    "tcgen05_tma_phases_pair": _COMMON_SRC + ["conv_tconv.cuh"],
    "tcgen05_staged_t": _COMMON_SRC + ["conv_tct.cuh", "conv_staged.cuh"],
    "tcgen05_wgrad_pair": ["conv_fwd.cu", "conv_wgrad.cu", "conv_wgrad.cuh", "conv_wgrad_tc.cuh", "conv_simt.cuh",
                           "conv_tc.cuh", "ptx.cuh", "launch.cuh"],
}


def kernel_source_hash(kernel=None):
    """Short hash of the sources a kernel variant depends on (all CUDA sources
    when `kernel` is None or unknown)."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "implicit_gemm_convolution_conv2d_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) if kernel else None
    if names is None:
        names = [n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh"))]
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:12]


def simt_tile(wl, dims, bn, ctas):
    """[pixels, channels] of the SIMT kernel's tile: BN from the plan, BM (64 or
    128) from the number of CTAs it launches."""
    M = wl.N * dims[0] * dims[1] * dims[2]
    og = wl.O // wl.groups
    n_tiles = -(-og // bn) * wl.groups
    m_tiles = ctas // max(n_tiles, 1)
    return [128 if m_tiles == -(-M // 128) else 64, bn]


def profiled_traffic(workload, variant_name):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    if not os.path.isdir(PROFILE_DIR):
        return None
    src = kernel_source_hash(variant_name)
    for name in sorted(os.listdir(PROFILE_DIR)):
        if not name.endswith((".txt", ".md")):
            continue
        with open(os.path.join(PROFILE_DIR, name)) as f:
            text = f.read()
        m = re.search(r"^traffic_record:\s*(\{.*\})\s*$", text, re.M)
        if not m:
            continue
        try:
            rec = json.loads(m.group(1))
        except ValueError:
            continue
        if rec.get("workload") == workload and rec.get("kernel") == variant_name and rec.get("source") == src:
            return rec.get("dram_bytes_per_launch_full")
    return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled DURING the timed region.

    Uses NVML (the library nvidia-smi reads) every ~5 ms from a thread, so that
    a timed region of a few milliseconds still gets samples; falls back to
    `nvidia-smi -lms 200` where NVML cannot be loaded."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index):
        self.index = index
        self.samples = []      # (sm_mhz, max_mhz, reasons bitmask)
        self._stop = threading.Event()
        self._t = None
        self._nvml = None
        self._smi = None
        self._lines = []

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self._nvml = (pynvml, h)
            self._t = threading.Thread(target=self._poll_nvml, daemon=True)
        except Exception:
            self._nvml = None
            try:
                fields = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                          "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                          "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
                self._smi = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.index}", f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                     "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self._t = threading.Thread(target=self._read_smi, daemon=True)
            except (OSError, ValueError):
                return
        self._t.start()

    def sample_now(self):
        """One NVML sample from the calling thread (used while the timed
        launches run, so that a region of a few milliseconds has samples)."""
        if self._nvml is None:
            return
        pynvml, h = self._nvml
        try:
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.samples.append((float(sm), float(mx), int(rs), time.perf_counter()))
        except Exception:
            pass

    def _poll_nvml(self):
        pynvml, h = self._nvml
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), int(rs), t))
            except Exception:
                break
            time.sleep(0.005)

    def _read_smi(self):
        for line in self._smi.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                bits = 0
                for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                   parts[5:9]):
                    if v.lower().startswith("active"):
                        bits |= self.REASONS[name]
                self.samples.append((float(parts[1]), float(parts[2]), bits, time.perf_counter()))
            except ValueError:
                continue

    def stop(self, t0=None, t1=None):
        """Stop sampling; summarise the samples taken inside [t0, t1] (the timed
        region's wall clock) when there are any, else all of them."""
        self._stop.set()
        if self._smi is not None:
            self._smi.terminate()
            try:
                self._smi.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._smi.kill()
        if self._t is not None:
            self._t.join(timeout=5)
        if t0 is not None:
            inside = [x for x in self.samples if t0 <= x[3] <= t1]
            if inside:
                self.samples = inside
        if not self.samples:
            return None
        reasons = sorted(n for n, b in self.REASONS.items() if any(s[2] & b for s in self.samples))
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": max(s[1] for s in self.samples),
                "sm_min_mhz": min(s[0] for s in self.samples), "reasons": reasons, "samples": len(self.samples),
                "source": "nvml" if self._nvml else "nvidia-smi"}


# ---------------------------------------------------------------- distributed

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(ws, backend):
    import datetime
    import torch.distributed as dist
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if ws > 1 else None


def aggregate(dist, local_ms, device=None):
    """(max time over ranks, number of ranks) -- the job's time is the slowest rank's."""
    if dist is None:
        return local_ms, 1
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item()), dist.get_world_size()


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- our arm

def bench_ours(args):
    import implicit_gemm_convolution_conv2d_b200 as C

    ws, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the CUDA path has no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(ws, "nccl")

    wl = WL.WORKLOADS[args.workload]
    # --pad-hi / --flip: the general form of the operation (per-side padding, true convolution)
    pad_hi = tuple(int(v) for v in args.pad_hi.split(",")) if args.pad_hi else None
    flip = 1 if args.flip else 0
    dims = out_dims(wl, pad_hi)
    flops = conv_flops(wl, dims)
    xb, wb, yb = conv_bytes(wl, dims)
    if wl.wgrad:
        # the weight gradient: inputs x and dy, output dw; the path (tensor cores or FP32) from its planner
        e = WL.ELEM_BYTES[wl.dtype]
        wb = e * wl.N * dims[0] * dims[1] * dims[2] * wl.O        # dy
        yb = e * wl.O * wl.k[0] * wl.k[1] * wl.k[2] * (wl.C // wl.groups)  # dw
        wpath, wsplit = C.wgrad_plan(wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, wl.k, wl.stride, wl.pad, wl.dil,
                                     wl.groups, wl.dtype)
        variant, bn, stages, ctas = None, (256 if wpath == C.WGRAD_TENSOR_CORES else 64), 1, 0
        vname = C.WGRAD_PATH_NAMES[wpath]
    elif wl.transpose:
        variant, bn, stages, ctas = C.transpose_plan(wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, wl.k, wl.stride, wl.pad,
                                                     wl.out_pad, wl.dil, wl.groups, wl.dtype,
                                                     getattr(C, "VARIANT_" + args.variant))
    else:
        variant, bn, stages, ctas = C.plan(wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, wl.k, wl.stride, wl.pad, wl.dil,
                                           wl.groups, wl.dtype, getattr(C, "VARIANT_" + args.variant),
                                           pad_hi=pad_hi, flip=flip)
    if not wl.wgrad:
        vname = C.VARIANT_NAMES[variant]

    # inputs: seeded on the host (rank-dependent seed), copied once
    if wl.wgrad:
        x_h, w_h = WL.make_wgrad_inputs(wl, (wl.N, *dims, wl.O), seed=wl.seed + 1000 * rank)  # w_h: dy
    else:
        x_h, w_h = WL.make_inputs(wl, seed=wl.seed + 1000 * rank)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_set = xb + wb + yb
    nsets = max(2, min(64, math.ceil(2 * l2 / per_set) + 1))
    xs = [x_h.to(dev) for _ in range(nsets)]
    wts = [w_h.to(dev) for _ in range(nsets)]
    Do, Ho, Wo = dims
    if wl.wgrad:
        ys = [torch.empty(wl.w_shape, dtype=x_h.dtype, device=dev) for _ in range(nsets)]  # dw
        ws_bytes = C.wgrad_workspace_size(wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, wl.k, wl.stride, wl.pad, wl.dil,
                                          wl.groups, wl.dtype)
        wsbuf = torch.empty(max(1, ws_bytes // 4), dtype=torch.float32, device=dev)
    else:
        ys = [torch.empty((wl.N, Do, Ho, Wo, wl.O), dtype=x_h.dtype, device=dev) for _ in range(nsets)]
    stream = torch.cuda.current_stream(dev)
    geo = lambda i: (wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, *wl.k, wl.stride, wl.pad, wl.dil, wl.groups)
    dcode = {"f32": 0, "f16": 1, "bf16": 2}[wl.dtype]
    launches = 0

    def step(i):
        nonlocal launches
        s = i % nsets
        # the launch goes to the current stream (the capture stream while a graph is recorded)
        if wl.wgrad:
            rc = C.conv_wgrad_raw(xs[s].data_ptr(), wts[s].data_ptr(), ys[s].data_ptr(),
                                  (wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, *wl.k, wl.stride, wl.pad, wl.pad, wl.dil,
                                   wl.groups), dcode, wsbuf.data_ptr() if ws_bytes else None, ws_bytes,
                                  torch.cuda.current_stream(dev).cuda_stream)
        elif wl.transpose:
            rc = C.conv_transpose_raw(xs[s].data_ptr(), wts[s].data_ptr(), ys[s].data_ptr(),
                                      (wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, *wl.k, wl.stride, wl.pad, wl.out_pad,
                                       wl.dil, wl.groups), dcode, variant, torch.cuda.current_stream(dev).cuda_stream)
        else:
            rc = C.conv_fwd_raw(xs[s].data_ptr(), wts[s].data_ptr(), ys[s].data_ptr(), geo(s), dcode,
                                variant, torch.cuda.current_stream(dev).cuda_stream, pad_hi=pad_hi, flip=flip)
        if rc:
            raise C.ConvError(rc, "conv_fwd")
        launches += 1

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if C.last_status() != 0:
        raise SystemExit("bench.py: device status word set during warm-up")

    # eager launches (host overhead included) -- reported beside the graph time
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n_eager = min(args.steps, 20)
    e0.record(stream)
    for i in range(n_eager):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    eager_ms = e0.elapsed_time(e1) / n_eager

    # the K timed launches, recorded once through the same C-ABI calls into a
    # CUDA graph, so that the timed region measures the kernels rather than
    # the Python/ctypes call overhead of each launch
    graph = None
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(args.steps):
                step(args.warmup + i)
        graph.replay()  # untimed: one more warm-up pass over every buffer set
        torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.01)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    launches = 0
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.perf_counter()
    ev0.record(stream)
    if graph is not None:
        graph.replay()
        launches = args.steps
    else:
        for i in range(args.steps):
            step(args.warmup + i)
    ev1.record(stream)
    while not ev1.query():      # the launches run: sample the clocks meanwhile
        clocks.sample_now()
        time.sleep(0.0002)
    torch.cuda.synchronize(dev)
    t_wall1 = time.perf_counter()
    barrier(dist, dev)
    clk = clocks.stop(t_wall0, t_wall1)
    local_ms = ev0.elapsed_time(ev1)
    timed_launches = launches
    status = C.last_status()
    if status != 0:
        raise SystemExit("bench.py: device status word set during the timed region")
    ms, nranks = aggregate(dist, local_ms, dev)
    ms_per_step = ms / args.steps
    value = nranks * flops * args.steps / (ms * 1e-3) / 1e12

    # ---- per-launch distribution (each launch between its own events, after
    # the timed region): cold L2 (rotating buffer sets) and warm L2 (one set)
    n_dist = max(5, min(args.steps, 50))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_dist + 1)]
    evs[0].record(stream)
    for i in range(n_dist):
        step(i)
        evs[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    cold = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(n_dist))
    evs[0].record(stream)
    for i in range(n_dist):
        step(0)
        evs[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    warm = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(n_dist))
    launch_dist = {"n": n_dist, "median_ms": round(cold[n_dist // 2], 5), "min_ms": round(cold[0], 5),
                   "warm_l2_median_ms": round(warm[n_dist // 2], 5), "warm_l2_min_ms": round(warm[0], 5),
                   "how": "eager launches, one event pair each, after the timed region"}

    # ---- end to end through the host-buffer C entry point (pinned host memory)
    e2e = None
    if pad_hi is not None or flip:
        e2e = {"skipped": "the host-buffer entry point takes symmetric padding and no flip"}
    elif wl.transpose or wl.wgrad:
        e2e = {"skipped": "the host-buffer entry point is the forward convolution's"}
    elif not args.no_e2e:
        xp = x_h.pin_memory()
        wp = w_h.pin_memory()
        yp = torch.empty(ys[0].shape, dtype=x_h.dtype).pin_memory()
        e_steps = max(3, min(args.steps, 20))
        for _ in range(2):
            C.conv_fwd_host(xp, wp, yp, xs[0], wts[0], ys[0], stride=wl.stride, padding=wl.pad,
                            dilation=wl.dil, groups=wl.groups, stream=stream)
        barrier(dist, dev)
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            C.conv_fwd_host(xp, wp, yp, xs[0], wts[0], ys[0], stride=wl.stride, padding=wl.pad,
                            dilation=wl.dil, groups=wl.groups, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems, _ = aggregate(dist, e0.elapsed_time(e1), dev)
        e2e = {"value": round(nranks * flops * e_steps / (ems * 1e-3) / 1e12, 4), "unit": "TFLOP/s",
               "h2d_bytes_per_step": xb + wb, "d2h_bytes_per_step": yb, "steps": e_steps,
               "ms_per_step": round(ems / e_steps, 5), "path": "conv_fwd_host (C ABI, pinned host buffers)"}

    # ---- roofline of the (single) kernel
    peaks, peak_src = measured_peaks()
    kern_ms = local_ms / timed_launches
    achieved_tflops = flops / (kern_ms * 1e-3) / 1e12
    # The bound is the roof whose time is longer: FLOPs at the kernel's own
    # arithmetic peak (FP32 FMA lanes for the SIMT and depthwise kernels, the
    # tensor cores for the rest) against the algorithmic bytes at HBM speed.
    sm_mhz = (clk or {}).get("sm_max_mhz") or 1965.0
    alu_peak = torch.cuda.get_device_properties(dev).multi_processor_count * 128 * 2 * sm_mhz * 1e6 / 1e12
    fma_kernel = (wl.wgrad and vname == "simt_wgrad") or variant in (C.VARIANT_SIMT, C.VARIANT_DEPTHWISE,
                                                                      C.VARIANT_DEPTHWISE_DIRECT)
    compute_peak = alu_peak if fma_kernel else float(peaks["bf16_tflops"])
    hbm_bound = (xb + wb + yb) / (float(peaks["hbm_gbs"]) * 1e9) > flops / (compute_peak * 1e12)
    tensor_bound = not fma_kernel and not hbm_bound
    if fma_kernel and not hbm_bound:
        peak = alu_peak
        roof = {"bound": "alu", "achieved": round(achieved_tflops, 3), "peak": round(peak, 2),
                "unit": "TFLOP/s", "frac": round(achieved_tflops / peak, 4),
                "peak_source": "148 SMs x 128 FP32 lanes x 2 FLOP x max SM clock"}
    elif tensor_bound:
        peak = float(peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": round(achieved_tflops, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved_tflops / peak, 4),
                "peak_source": f"{peak_src} cuBLAS bf16 burst (MEASURED_PEAKS.json bf16_tflops)"}
    else:
        gbs = (xb + wb + yb) / (kern_ms * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                "frac": round(gbs / peak, 4), "peak_source": f"{peak_src} copy bandwidth (hbm_gbs)"}
    roof["traffic"] = profiled_traffic(args.workload, vname)
    roof["launch_distribution"] = launch_dist
    roof["kernel"] = vname
    roof["ms_per_launch"] = round(kern_ms, 5)

    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": nranks, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "frac_of_dense_peak": round(value / nranks / SPEC_DENSE_TFLOPS, 4),
        "config": {"workload": wl.name, "N": wl.N, "DHW": [wl.D, wl.H, wl.W], "C": wl.C, "O": wl.O,
                   "kernel": list(wl.k), "stride": list(wl.stride), "pad": list(wl.pad), "dil": list(wl.dil),
                   "groups": wl.groups, "out_DHW": list(dims),
                   **({"transpose": True, "out_pad": list(wl.out_pad)} if wl.transpose else {}),
                   **({"pass": "weight gradient (x, dy -> dw)"} if wl.wgrad else {}), "gflop_per_step": round(flops / 1e9, 4),
                   "global_batch": wl.N * nranks, "parallelism": f"independent batches x{nranks}",
                   "variant": vname,
                   "tile": ([bn, bn] if wl.wgrad  # output channels x weight columns per block (or CTA pair)
                            else simt_tile(wl, dims, bn, ctas) if variant == C.VARIANT_SIMT else
                            [4, bn] if variant in (C.VARIANT_DEPTHWISE, C.VARIANT_DEPTHWISE_DIRECT)  # pixels x channels per thread
                            else [bn, 128] if variant == C.VARIANT_TC_TMA_T
                            else [bn, 128 if (wl.O // wl.groups) % 128 == 0 else 64] if variant == C.VARIANT_TC_HALO_T
                            else [bn, 256] if variant == C.VARIANT_TC_HALO_T_PAIR
                            else [256 if "pair" in vname else 128, bn]),
                   "stages": stages, "ctas": ctas,
                   "l2": f"inputs rotate over {nsets} buffer sets ({nsets * per_set / 2**20:.0f} MiB > 2x L2)"},
        "roofline": roof,
        "launch": "cuda_graph_of_steps" if graph is not None else "eager",
        "eager_ms_per_step": round(eager_ms, 5),
        "e2e": e2e,
        # the weight gradient queues two kernels per call (the split-K partial sums, their ordered sum)
        "gpu_launches": timed_launches * (2 if wl.wgrad else 1),
        "clocks": clk,
    }
    if pad_hi is not None or flip:
        out["config"]["pad_hi"] = list(pad_hi) if pad_hi is not None else list(wl.pad)
        out["config"]["flip"] = flip
        if rank == 0 and not args.no_cpu_baseline:
            out["cpu_baseline"] = {"skipped": "the CPU baseline is timed on the workload's own padding, no flip"}
    elif rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_seconds)
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# ---------------------------------------------------------------- CPU oracle

def _sample_inputs(wl):
    """The workload's host inputs: (x, w), or (x, dy) for a weight gradient."""
    if wl.wgrad:
        return WL.make_wgrad_inputs(wl, (wl.N, *out_dims(wl, via_oracle=True), wl.O))
    return WL.make_inputs(wl)


def host_cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _oracle_sample_step(wl, x, w, n_img):
    import oracle
    xs = x[:n_img].contiguous()
    if wl.wgrad:  # w is dy here
        y, _ = oracle.conv_wgrad(xs, w[:n_img].contiguous(), wl.k, wl.stride, wl.pad, wl.dil, wl.groups)
    elif wl.transpose:
        y, _ = oracle.conv_transpose(xs, w, wl.stride, wl.pad, wl.out_pad, wl.dil, wl.groups)
    else:
        y, _ = oracle.conv_fwd(xs, w, wl.stride, wl.pad, wl.dil, wl.groups)
    return y


def cpu_baseline(wl, budget_s=15.0):
    """The oracle as it stands, on the host cores, over the first images of the
    workload (as many as fit the time budget)."""
    import oracle
    x, w = _sample_inputs(wl)
    one = wl.with_(N=1)
    f1 = conv_flops(one, via_oracle=True)
    t0 = time.perf_counter()
    _oracle_sample_step(wl, x, w, 1)
    t1 = time.perf_counter() - t0
    n_img = 1
    total_t, total_f = t1, f1
    while total_t < budget_s and n_img < wl.N:
        k = min(wl.N - n_img, max(1, int((budget_s - total_t) / max(t1, 1e-3))))
        t0 = time.perf_counter()
        _oracle_sample_step(wl, x[n_img:], w, k)
        total_t += time.perf_counter() - t0
        total_f += f1 * k
        n_img += k
    out = {"value": round(total_f / total_t / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
           "cpu_model": host_cpu_model(),
           "kind": "oracle", "sample": f"first {n_img} of {wl.N} images of {wl.name} ({total_t:.1f} s)"}
    out["single_thread"] = _oracle_single_thread(wl, x, w)
    return out


def _oracle_single_thread(wl, x, w, max_flops=3e9):
    """The oracle on one host thread: the full direct loop over the first image,
    its depth halved (3-D) until the work is about `max_flops` or the depth is
    down to 4 (FLOPs count every tap, as everywhere in this file, so a thinner
    slab would count mostly padding taps)."""
    import oracle
    sub = wl.with_(N=1)
    while conv_flops(sub, via_oracle=True) > max_flops and sub.D > 4:
        sub = sub.with_(D=(sub.D + 1) // 2)
    xs = x[:1, :sub.D].contiguous()
    full = oracle.max_threads()
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        _oracle_sample_step(sub, xs, w, 1)
        dt = time.perf_counter() - t0
    finally:
        oracle.set_threads(full)
    return {"value": round(conv_flops(sub, via_oracle=True) / dt / 1e12, 6), "unit": "TFLOP/s", "cores": 1,
            "sample": f"image 0 of {wl.name}, depth {sub.D} of {wl.D} ({dt:.1f} s)"}


def bench_reference(args):
    """The reference arm for this build is the CPU oracle (fp64 direct loop)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    wl = WL.WORKLOADS[args.workload]
    x, w = _sample_inputs(wl)
    one = wl.with_(N=1)
    f1 = conv_flops(one, via_oracle=True)
    # one step = the oracle on one image of the workload (a bounded sample)
    for i in range(args.warmup):
        _oracle_sample_step(wl, x[i % wl.N:], w, 1)
    t0 = time.perf_counter()
    for i in range(args.steps):
        _oracle_sample_step(wl, x[i % wl.N:], w, 1)
    dt = time.perf_counter() - t0
    value = f1 * args.steps / dt / 1e12
    out = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 0, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": wl.name, "global_batch": wl.N,
                      "sample": f"one image of the {wl.N}-image batch per step (a bounded sample of the same "
                                f"workload; the metric is per FLOP, so the value compares with the full batch)"},
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
                            "cpu_model": host_cpu_model(),
                            "kind": "oracle", "sample": f"one image of {wl.name} per step, {args.steps} steps"},
           "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=WL.HEADLINE, choices=sorted(WL.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of a CUDA graph")
    ap.add_argument("--variant", default="AUTO",
                    choices=["AUTO", "SIMT", "TC_TMA", "TC_GATHER", "TC_TMA_PAIR", "TC_HALO", "TC_HALO_PAIR", "TC_TMA_T", "TC_HALO_T",
                             "TC_HALO_T_PAIR", "TC_PHASE", "DEPTHWISE", "DEPTHWISE_DIRECT", "TC_TMA_PHASES",
                             "TC_STAGED"],
                    help="kernel variant (default: the library's own choice)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--pad-hi", default=None,
                    help="padding above each dimension, 'd,h,w' (the workload's pad stays the padding below)")
    ap.add_argument("--flip", action="store_true", help="read the filter reversed (a true convolution)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)   # at least three untimed warm-up steps
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_ours(args)


if __name__ == "__main__":
    main()
