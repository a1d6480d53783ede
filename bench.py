"""Benchmark: grouped-conv TFLOP/s and depthwise GB/s on B200, as fractions of the tensor / HBM
roofline, with the fp64 CPU oracle timed beside it.

One step = one forward of the wide-group layer x[1, 512, 256, 256] * w[512, 128, 3, 3],
groups = 4, pad 1 (the layer timed in "F.conv2d runs x15 slower in mixed-precision/
half-precision mode"), bf16 in / fp32 accumulate / bf16 out, NHWC by default, through the
library's C ABI. `value` is whole-job TFLOP/s (77.31 GFLOP per step per GPU) over the K timed
steps. Inputs are synthetic (seeded, x ~ N(0,1), w ~ N(0, 1/1152)); the timed steps rotate
over enough x/y buffer sets that every step's working set is evicted from L2 by the next.

The same JSON line carries the depthwise measurements (GB/s against the HBM roofline):
the depthwise conv2d x[32, 56, 56, 1024] 3x3 at stride 1 and 2, and the Conformer depthwise
conv1d x[8, 2048, 512], K = 31 (fwd, dgrad, wgrad), each kernel timed with CUDA events on its
own stream with an L2 flush before every launch (outside the event bracket).

Multi-GPU: the path does not shard (one conv runs on one GPU); with N ranks each GPU runs an
independent replica on its own inputs, no data-path collective, and the timing is the max
over ranks ("scaling": "weak").

`--impl reference` times the fp64 CPU oracle (the only reference that exists for this path)
on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from depthwise_convolution_gconv2d_b200 import workloads as wl  # noqa: E402

METRIC = "grouped-conv TFLOP/s and depthwise GB/s on 1 B200; % of tensor / HBM roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "of measured"
    except (OSError, ValueError):
        return dict(FALLBACK), "of fallback"


def kernel_source_hash(name: str) -> str:
    path = os.path.join(ROOT, "depthwise_convolution_gconv2d_b200", "csrc", name)
    try:
        return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    except OSError:
        return ""


def traffic_for(kernel: str, source: str):
    """DRAM read and write bytes per launch from a committed ncu capture, if the kernel's
    source is unchanged since (None otherwise)."""
    try:
        d = json.load(open(TRAFFIC_FILE)).get(kernel)
    except (OSError, ValueError):
        return None
    if not d or d.get("source_sha") != kernel_source_hash(source):
        return None
    return d


# Timed regions shorter than this run at burst clocks (the power cap needs seconds of
# sustained load to pull the SM clock down), so their roofline uses the burst GEMM peak.
SUSTAINED_MIN_S = 2.0


def tensor_peak_for(pk, timed_s: float, clocks):
    """(peak TFLOP/s, which) for a kernel timed over `timed_s` seconds: the sustained bf16
    figure only when the region lasted seconds AND the sampled clocks show the power cap (or
    a median SM clock under 90 % of max); the burst figure otherwise."""
    sustained = pk.get("bf16_tflops_sustained")
    if sustained and timed_s >= SUSTAINED_MIN_S and clocks:
        capped = "sw_power_cap" in clocks.get("reasons", [])
        slow = (clocks.get("sm_max_mhz") or 0) > 0 and \
            clocks["sm_mhz"] < 0.9 * clocks["sm_max_mhz"]
        if capped or slow:
            return sustained, "bf16_tflops_sustained"
    return pk["bf16_tflops"], "bf16_tflops"


def compact_rooflines(dwm, more, bwd, extra=None):
    """One flat map of roofline fractions, named workload_bound, for every secondary
    workload (the headline has its own roofline object)."""
    out = {}
    names = {"depthwise56_s1": "dw56_s1", "depthwise56_s2": "dw56_s2"}
    for k, v in (dwm or {}).items():
        if k.startswith("dw1d_") and k.endswith("_cudacore"):
            continue
        out[f"{names.get(k, k)}_hbm"] = v["frac"]
        if "frac_b2b" in v:
            out[f"{names.get(k, k)}_b2b_hbm"] = v["frac_b2b"]
    for k, v in (more or {}).items():
        if "_direct" in k and v.get("us", 0) > 5000:
            continue
        out[f"{k}_{v['bound']}"] = v["frac"]
        if "frac_b2b" in v:
            out[f"{k}_b2b_{v['bound']}"] = v["frac_b2b"]
        if "ffma_frac" in v:
            out[f"{k}_ffma"] = v["ffma_frac"]
        if "tensor_frac" in v:
            out[f"{k}_tensor"] = v["tensor_frac"]
    for k, v in (bwd or {}).items():
        out[f"bwd_{k}_{v['bound']}"] = v["frac"]
        if "frac_b2b" in v:
            out[f"bwd_{k}_b2b_{v['bound']}"] = v["frac_b2b"]
    for k, v in (extra or {}).items():
        out[f"{k}_{v['bound']}"] = v["frac"]
    return out


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if not self.out:
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- device helpers

def dev_tensor(torch, storage, dtype, device):
    a = np.ascontiguousarray(storage)
    if dtype == wl.F32:
        return torch.from_numpy(a.astype(np.float32)).to(device)
    t = torch.from_numpy(a.view(np.int16)).to(device)
    return t.view(torch.bfloat16 if dtype == wl.BF16 else torch.float16)


def torch_dtype(torch, dtype):
    return {wl.F32: torch.float32, wl.F16: torch.float16, wl.BF16: torch.bfloat16}[dtype]


def l2_flusher(torch, device):
    """L2 flush before a timed launch: write a buffer of 2x L2, then read another of 2x L2.
    The write evicts the launch's own data; the read then evicts the write's dirty lines, so
    the timed kernel starts with a cold L2 holding only clean lines, as under ncu's cache
    control. (With the write alone, ~126 MB of the flush's dirty lines were written back to
    DRAM inside the timed kernel: 79 us cold under ncu against 90 us in the bench for the
    depthwise 3x3 layer.)"""
    wbuf = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=device)
    rbuf = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device=device)
    sink = torch.empty((), dtype=torch.int32, device=device)

    def flush(stream):
        with torch.cuda.stream(stream):
            wbuf.fill_(1)
            torch.amax(rbuf, dim=0, out=sink)
    return flush


def gpu_spin(torch, stream, us=200):
    """Keep the stream busy for ~`us` microseconds so that the host has enqueued what follows
    before the GPU reaches it (host launch latency stays outside event brackets)."""
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(us * 2000))


def max_over_ranks(torch, dist, value: float, device) -> float:
    """The maximum of `value` over all ranks of the default process group (the job's time is
    its slowest rank's); `value` itself when no group is initialised."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_launches(torch, fn, stream, reps, flush=None):
    """Median and mean CUDA-event time (ms) of `fn(i)` over `reps` launches on `stream`,
    flushing L2 before each launch outside the event bracket."""
    times = []
    for i in range(reps):
        if flush is not None:
            flush(stream)
        gpu_spin(torch, stream)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn(i)
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times), sum(times) / len(times)


def sets_for(set_bytes: int) -> int:
    """Buffer sets for a back-to-back figure: at least 2, and together more than 2x L2."""
    return max(2, -(-2 * L2_BYTES // max(1, set_bytes)) + 1)


def time_graph_b2b(torch, fn, stream, n_sets, launches=32, reps=5):
    """Per-launch CUDA-event time (ms) of `launches` back-to-back launches of `fn(i)`, i cycling
    over `n_sets` buffer sets whose combined size exceeds 2x L2 (a launch reads inputs that 7
    others have evicted since it last touched them), captured in one CUDA graph and replayed
    after a spin; median over `reps` replays. A single launch after a spin also pays the idle
    stream's launch latency (~6 us for an empty kernel on B200, against ~1 us per launch inside
    a graph), which dominates kernels whose HBM floor is a few microseconds."""
    with torch.cuda.stream(stream):
        for i in range(n_sets):
            fn(i)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(launches):
            fn(i % n_sets)
    times = []
    for _ in range(reps):
        gpu_spin(torch, stream, 400)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g.replay()
            b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b) / launches)
    del g
    return statistics.median(times)


# ---------------------------------------------------------------------------- workloads

def conv2d_problem(layout: str):
    return wl.wide_group(wl.NHWC if layout == "nhwc" else wl.NCHW)


def kernel_name(code: int) -> str:
    return {1: "direct_generic", 2: "depthwise_nhwc", 3: "igemm_tc", 4: "igemm_tc_nchw",
            8: "grouped_nhwc"}.get(code, str(code))


LAUNCHES_PER_CALL = {1: 1, 2: 1, 3: 1, 4: 3, 8: 1}
CUDA_CORE_KERNELS = (1, 2, 8)
SM_MAX_MHZ = 1965.0     # B200 clocks.max.sm


def ffma_peak_tflops(sms: int = 148, mhz: float = SM_MAX_MHZ) -> float:
    """FP32 FMA roofline of the CUDA cores: 128 FMA lanes per SM, 2 FLOP per FMA."""
    return sms * 128 * 2 * mhz * 1e6 / 1e12
# source file of the kernel that runs the headline layer for each kernel code (the wide-group
# layer takes the transposed row-strip kernel, igemm_rowt.cu)
KERNEL_SOURCE = {1: "direct_generic.cu", 2: "depthwise_nhwc.cu", 3: "igemm_rowt.cu",
                 4: "igemm_rowt.cu", 8: "grouped_nhwc.cu"}


def conv2d_measurement(torch, gb, device, stream, pk, p, workload, path, reps, flush):
    inp = wl.make_conv2d_inputs(p, workload)
    w = dev_tensor(torch, inp.w, p.dtype, device)
    n_sets = sets_for(p.bytes())
    xs = [dev_tensor(torch, inp.x, p.dtype, device) for _ in range(n_sets)]
    ys = [torch.empty(p.y_shape, dtype=torch.bfloat16, device=device) for _ in range(n_sets)]
    need = gb.gconv2d_fwd_workspace_size(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride,
                                         p.pad, p.dilation, p.groups, p.layout, p.dtype, path)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    kcode = gb.gconv2d_select_path(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad,
                                   p.dilation, p.groups, p.layout, p.dtype, path)
    fn = lambda i: gb.gconv2d_fwd(xs[i], w, None, p.stride, p.pad, p.dilation, p.groups,
                                  p.layout, out=ys[i], workspace=ws, path=path, stream=stream)
    for _ in range(2):
        fn(0)
    med, mean = time_launches(torch, lambda i: fn(0), stream, reps, flush)
    # back to back in a graph, except for the slow generic fallbacks (milliseconds a launch)
    b2b = time_graph_b2b(torch, fn, stream, n_sets) if med < 5.0 else None
    tf = p.flops() / (med * 1e-3) / 1e12
    gbs = p.bytes() / (med * 1e-3) / 1e9
    t_hbm = p.bytes() / (pk["hbm_gbs"] * 1e9)
    rec = {"kernel": kernel_name(kcode), "us": round(med * 1e3, 2), "TFLOP/s": round(tf, 1),
           "GB/s": round(gbs, 1)}
    if kcode in CUDA_CORE_KERNELS:
        # fp32 FMAs on the CUDA cores: the arithmetic roofline is the FFMA rate
        t_alu = p.flops() / (ffma_peak_tflops() * 1e12)
        rec["ffma_frac"] = round(tf / ffma_peak_tflops(), 3)
        bound, t_roof = ("alu", t_alu) if t_alu >= t_hbm else ("hbm", t_hbm)
    else:
        t_tensor = p.flops() / (pk["bf16_tflops"] * 1e12)
        bound, t_roof = ("tensor", t_tensor) if t_tensor >= t_hbm else ("hbm", t_hbm)
    rec.update({"bound": bound, "frac": round(t_roof / (med * 1e-3), 3),
                "alg_flops": p.flops(), "alg_bytes": p.bytes()})
    if b2b is not None:
        rec.update({"us_b2b": round(b2b * 1e3, 2), "frac_b2b": round(t_roof / (b2b * 1e-3), 3)})
    del xs, ys, ws
    return rec


def variant_measurement(torch, gb, device, stream, pk, p, workload, mode, reps, flush):
    """The wide-group layer with its output in another channel order or merged across groups
    (gconv2d_fwd_out): same FLOPs as the layer; bytes x + w + y, y with C_out / groups channels
    for the merges."""
    inp = wl.make_conv2d_inputs(p, workload)
    w = dev_tensor(torch, inp.w, p.dtype, device)
    x0 = dev_tensor(torch, inp.x, p.dtype, device)
    y0 = gb.gconv2d_fwd_out(x0, w, None, p.stride, p.pad, p.dilation, p.groups, p.layout, mode)
    nbytes = (x0.numel() + w.numel() + y0.numel()) * 2
    n_sets = sets_for(nbytes)
    xs = [x0] + [dev_tensor(torch, inp.x, p.dtype, device) for _ in range(n_sets - 1)]
    ys = [y0] + [torch.empty_like(y0) for _ in range(n_sets - 1)]
    kcode = gb.gconv2d_fwd_out_select_path(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride,
                                           p.pad, p.dilation, p.groups, p.layout, p.dtype, mode)
    fn = lambda i: gb.gconv2d_fwd_out(xs[i], w, None, p.stride, p.pad, p.dilation, p.groups,
                                      p.layout, mode, out=ys[i], stream=stream)
    for _ in range(2):
        fn(0)
    med, mean = time_launches(torch, lambda i: fn(0), stream, reps, flush)
    b2b = time_graph_b2b(torch, fn, stream, n_sets)
    t_tensor = p.flops() / (pk["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    bound, t_roof = ("tensor", t_tensor) if t_tensor >= t_hbm else ("hbm", t_hbm)
    rec = {"kernel": kernel_name(kcode), "us": round(med * 1e3, 2),
           "TFLOP/s": round(p.flops() / (med * 1e-3) / 1e12, 1),
           "GB/s": round(nbytes / (med * 1e-3) / 1e9, 1), "bound": bound,
           "frac": round(t_roof / (med * 1e-3), 3), "us_b2b": round(b2b * 1e3, 2),
           "frac_b2b": round(t_roof / (b2b * 1e-3), 3), "alg_flops": p.flops(),
           "alg_bytes": nbytes}
    del xs, ys
    return rec


def more_conv2d_measurements(torch, gb, device, stream, pk, reps):
    """The other conv2d workloads: ensemble-as-groups layer and the groups sweep at C = 1024."""
    flush = l2_flusher(torch, device)
    out = {}
    out["ensemble_g64_nhwc"] = conv2d_measurement(torch, gb, device, stream, pk,
                                                  wl.ensemble_groups(), 4, gb.PATH_AUTO, reps,
                                                  flush)
    out["wide_group_nchw"] = conv2d_measurement(torch, gb, device, stream, pk,
                                                wl.wide_group(wl.NCHW), 2, gb.PATH_AUTO, reps,
                                                flush)
    # grouped linear x[16384, 4096] -> [16384, 4096] in 4 groups (1x1 conv of 1x1 images)
    out["grouped_linear"] = conv2d_measurement(torch, gb, device, stream, pk,
                                               wl.grouped_linear(), 6, gb.PATH_AUTO, reps, flush)
    for mode in ("interleaved", "avg", "max"):
        out[f"wide_group_{mode}"] = variant_measurement(torch, gb, device, stream, pk,
                                                        wl.wide_group(wl.NHWC), 2, mode, reps,
                                                        flush)
    for g in (1024, 256, 64, 16):
        p = wl.depthwise_56(1, g)
        for name, path in (("auto", gb.PATH_AUTO), ("direct", gb.PATH_DIRECT),
                           ("igemm", gb.PATH_IGEMM)):
            if path == gb.PATH_IGEMM and gb.gconv2d_select_path(
                    p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad, p.dilation,
                    p.groups, p.layout, p.dtype, path) < 0:
                continue
            r = 3 if (path == gb.PATH_DIRECT and g <= 64) else reps
            out[f"sweep56_g{g}_{name}"] = conv2d_measurement(torch, gb, device, stream, pk, p, 5,
                                                             path, r, flush)
    return out


def depthwise_measurements(torch, gb, device, stream, pk, reps):
    """GB/s of the depthwise kernels (config shapes), L2 flushed before each launch."""
    flush = l2_flusher(torch, device)
    out = {}
    hbm = pk["hbm_gbs"]
    for stride in (1, 2):
        p = wl.depthwise_56(stride)
        inp = wl.make_conv2d_inputs(p, 5)
        w = dev_tensor(torch, inp.w, p.dtype, device)
        n_sets = sets_for(p.bytes())
        xs = [dev_tensor(torch, inp.x, p.dtype, device) for _ in range(n_sets)]
        ys = [torch.empty(p.y_shape, dtype=torch.bfloat16, device=device) for _ in range(n_sets)]
        fn = lambda i: gb.gconv2d_fwd(xs[i], w, None, p.stride, p.pad, p.dilation, p.groups,
                                      p.layout, out=ys[i], stream=stream)
        for _ in range(3):
            fn(0)
        med, mean = time_launches(torch, lambda i: fn(0), stream, reps, flush)
        b2b = time_graph_b2b(torch, fn, stream, n_sets)
        gbs = p.bytes() / (med * 1e-3) / 1e9
        gbs_b2b = p.bytes() / (b2b * 1e-3) / 1e9
        out[f"depthwise56_s{stride}"] = {"us": round(med * 1e3, 2), "GB/s": round(gbs, 1),
                                         "frac": round(gbs / hbm, 3),
                                         "us_b2b": round(b2b * 1e3, 2),
                                         "frac_b2b": round(gbs_b2b / hbm, 3),
                                         "alg_bytes": p.bytes()}
        del xs, w, ys
    for causal in (False, True):
        p = wl.conformer_dw1d(causal)
        inp = wl.make_dwconv1d_inputs(p, 3)
        # 8 buffer sets (x, dy, y, dx: 537 MB > 2x L2) for the back-to-back figure; the
        # single-launch figure uses set 0
        n_sets = 8
        w = dev_tensor(torch, inp.w, p.dtype, device)
        xs = [dev_tensor(torch, inp.x, p.dtype, device) for _ in range(n_sets)]
        dys = [dev_tensor(torch, inp.dy, p.dtype, device) for _ in range(n_sets)]
        ys = [torch.empty((p.B, p.T_out, p.C), dtype=torch.bfloat16, device=device)
              for _ in range(n_sets)]
        dxs = [torch.empty((p.B, p.T, p.C), dtype=torch.bfloat16, device=device)
               for _ in range(n_sets)]
        dw = torch.empty((p.C, p.K), dtype=torch.bfloat16, device=device)
        need = gb.dwconv1d_bwd_weight_workspace_size(p.B, p.T, p.C, p.K, p.pad_left, p.pad_right,
                                                     p.dtype)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
        sel = lambda path: gb.KERNEL_NAMES.get(gb.dwconv1d_select_path(
            p.B, p.T, p.C, p.K, p.pad_left, p.pad_right, p.dtype, path), "?")
        ops = {
            "fwd": (lambda i: gb.dwconv1d_fwd(xs[i], w, p.pad_left, p.pad_right, out=ys[i],
                                              stream=stream), sel(gb.PATH_AUTO)),
            "dgrad": (lambda i: gb.dwconv1d_bwd_data(dys[i], w, p.T, p.pad_left, p.pad_right,
                                                     out=dxs[i], stream=stream),
                      sel(gb.PATH_AUTO)),
            "wgrad": (lambda i: gb.dwconv1d_bwd_weight(xs[i], dys[i], p.K, p.pad_left,
                                                       p.pad_right, out=dw, workspace=ws,
                                                       stream=stream),
                      "conv1d_wgrad"),
            # the CUDA-core kernel of the DIRECT family on the same problem, for comparison
            "fwd_cudacore": (lambda i: gb.dwconv1d_fwd(xs[i], w, p.pad_left, p.pad_right,
                                                       out=ys[i], stream=stream,
                                                       path=gb.PATH_DIRECT),
                             sel(gb.PATH_DIRECT)),
        }
        tag = "causal" if causal else "same"
        for op, (fn, kname) in ops.items():
            for _ in range(3):
                fn(0)
            med, mean = time_launches(torch, lambda i: fn(0), stream, reps, flush)
            b2b = time_graph_b2b(torch, fn, stream, n_sets)
            ab = p.bytes(op.split("_")[0])
            gbs = ab / (med * 1e-3) / 1e9
            gbs_b2b = ab / (b2b * 1e-3) / 1e9
            out[f"dw1d_{tag}_{op}"] = {"kernel": kname, "us": round(med * 1e3, 2),
                                       "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 3),
                                       "us_b2b": round(b2b * 1e3, 2),
                                       "frac_b2b": round(gbs_b2b / hbm, 3), "alg_bytes": ab}
        del xs, dys, ys, dxs
    return out


def dwsep_measurements(torch, gb, device, stream, pk, reps):
    """The depthwise-separable block of the Conformer convolution module: x[8, 2048, 512],
    depthwise K = 31 'same', then pointwise 512 -> 512 (+ bias), fused in one kernel, and the
    same block as two launches (depthwise into a workspace, then the pointwise GEMM) for
    comparison. Algorithmic bytes x + w_dw + w_pw + bias + z; FLOPs 2*B*T*C*(K + C_out);
    L2 flushed before each launch."""
    flush = l2_flusher(torch, device)
    p = wl.conformer_dw1d(False)
    C_out = 512
    inp = wl.make_dwsep1d_inputs(p, C_out, 7)
    wdw, wpw, b = (dev_tensor(torch, a, p.dtype, device) for a in (inp.w_dw, inp.w_pw, inp.bias))
    nbytes = (inp.x.size + wdw.numel() + wpw.numel() + b.numel() + p.B * p.T_out * C_out) * 2
    n_sets = sets_for(nbytes)
    xs = [dev_tensor(torch, inp.x, p.dtype, device) for _ in range(n_sets)]
    zs = [torch.empty((p.B, p.T_out, C_out), dtype=torch.bfloat16, device=device)
          for _ in range(n_sets)]
    flops = 2 * p.B * p.T_out * p.C * (p.K + C_out)
    out = {}
    for name, path in (("dwsep1d_fused", gb.PATH_AUTO), ("dwsep1d_two_launches", gb.PATH_DIRECT)):
        need = gb.load_library().dwsep1d_fwd_workspace_size(p.B, p.T, p.C, p.K, p.pad_left,
                                                            p.pad_right, C_out, p.dtype, path)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
        kname = gb.KERNEL_NAMES.get(gb.dwsep1d_select_path(p.B, p.T, p.C, p.K, p.pad_left,
                                                           p.pad_right, C_out, p.dtype, path))
        fn = lambda i: gb.dwsep1d_fwd(xs[i], wdw, wpw, b, p.pad_left, p.pad_right, out=zs[i],
                                      workspace=ws, path=path, stream=stream)
        for _ in range(3):
            fn(0)
        med, mean = time_launches(torch, lambda i: fn(0), stream, reps, flush)
        b2b = time_graph_b2b(torch, fn, stream, n_sets)
        t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
        out[name] = {"kernel": kname, "us": round(med * 1e3, 2),
                     "TFLOP/s": round(flops / (med * 1e-3) / 1e12, 1),
                     "GB/s": round(nbytes / (med * 1e-3) / 1e9, 1), "bound": "hbm",
                     "frac": round(t_hbm / (med * 1e-3), 3),
                     "us_b2b": round(b2b * 1e3, 2), "frac_b2b": round(t_hbm / (b2b * 1e-3), 3),
                     "tensor_frac": round(2 * p.B * p.T_out * p.C * C_out / (med * 1e-3) /
                                          (pk["bf16_tflops"] * 1e12), 3),
                     "alg_bytes": nbytes, "alg_flops": flops}
        del ws
    # strided 2-D blocks: a Fast Conformer downsampler layer, x[8, 512, 40, 256] NHWC (frames x
    # frequency bins; 20 output columns, narrower than the fused kernel's 32-column tiles, so
    # AUTO runs the two launches there), and the same layer on 128 bins (64 output columns)
    del xs, zs
    for tag, W in (("", 40), ("_w128", 128)):
        out.update(dwsep2d_measurement(torch, gb, device, stream, pk, reps, flush, W, tag))
    return out


def dwsep2d_measurement(torch, gb, device, stream, pk, reps, flush, W, tag):
    out = {}
    N, H, C, k, st, pad, Co = 8, 512, 256, 3, 2, 1, 256
    p2 = wl.Dwconv1dProblem(N, H * W, C, k * k, 0, 0, wl.BF16)
    inp2 = wl.make_dwsep1d_inputs(p2, Co, 8)
    wdw2 = dev_tensor(torch, inp2.w_dw.reshape(C, k, k, 1), wl.BF16, device)
    wpw2, b2 = (dev_tensor(torch, a, wl.BF16, device) for a in (inp2.w_pw, inp2.bias))
    Ho, Wo = gb.out_shape(N, C, H, W, C, k, k, st, pad, 1, C, "NHWC", wl.BF16)
    nbytes2 = (N * H * W * C + wdw2.numel() + wpw2.numel() + b2.numel() + N * Ho * Wo * Co) * 2
    n_sets = sets_for(nbytes2)
    x2s = [dev_tensor(torch, inp2.x.reshape(N, H, W, C), wl.BF16, device) for _ in range(n_sets)]
    z2s = [torch.empty((N, Ho, Wo, Co), dtype=torch.bfloat16, device=device)
           for _ in range(n_sets)]
    flops2 = 2 * N * Ho * Wo * C * (k * k + Co)
    for name, path in ((f"dwsep2d{tag}_auto", gb.PATH_AUTO),
                       (f"dwsep2d{tag}_two_launches", gb.PATH_DIRECT)):
        kname = gb.KERNEL_NAMES.get(gb.dwsep2d_select_path(N, C, H, W, k, k, st, pad, 1, Co,
                                                           "NHWC", wl.BF16, path))
        need = gb.load_library().dwsep2d_fwd_workspace_size(N, C, H, W, k, k, st, pad, 1, Co,
                                                            wl.NHWC, wl.BF16, path)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
        fn = lambda i: gb.dwsep2d_fwd(x2s[i], wdw2, wpw2, b2, st, pad, 1, "NHWC", out=z2s[i],
                                      workspace=ws, path=path, stream=stream)
        for _ in range(3):
            fn(0)
        med, mean = time_launches(torch, lambda i: fn(0), stream, reps, flush)
        b2b = time_graph_b2b(torch, fn, stream, n_sets)
        t_hbm = nbytes2 / (pk["hbm_gbs"] * 1e9)
        out[name] = {"kernel": kname, "us": round(med * 1e3, 2),
                     "TFLOP/s": round(flops2 / (med * 1e-3) / 1e12, 1),
                     "GB/s": round(nbytes2 / (med * 1e-3) / 1e9, 1), "bound": "hbm",
                     "frac": round(t_hbm / (med * 1e-3), 3),
                     "us_b2b": round(b2b * 1e3, 2), "frac_b2b": round(t_hbm / (b2b * 1e-3), 3),
                     "alg_bytes": nbytes2, "alg_flops": flops2}
        del ws
    del x2s, z2s
    return out


def backward_measurements(torch, gb, device, stream, pk, reps):
    """The grouped conv2d's data and weight gradients on the depthwise 56x56x1024 layer
    (strides 1 and 2) and the wide-group layer, L2 flushed before each launch. Algorithmic
    bytes: dgrad dy + w + dx, wgrad x + dy + dw (the workspace partials are reported apart);
    FLOPs as the forward."""
    flush = l2_flusher(torch, device)
    out = {}
    cases = [("depthwise56_s1", wl.depthwise_56(1), reps), ("depthwise56_s2", wl.depthwise_56(2), reps),
             ("wide_group_nhwc", wl.wide_group(wl.NHWC), reps),
             ("wide_group_nchw", wl.wide_group(wl.NCHW), reps)]
    for tag, p, r in cases:
        inp = wl.make_conv2d_inputs(p, 5)
        w = dev_tensor(torch, inp.w, p.dtype, device)
        dy_host = wl.make_conv2d_dy(p, 5)
        n_sets = sets_for(p.bytes())
        xs = [dev_tensor(torch, inp.x, p.dtype, device) for _ in range(n_sets)]
        dys = [dev_tensor(torch, dy_host, p.dtype, device) for _ in range(n_sets)]
        dxs = [torch.empty(p.x_shape, dtype=torch.bfloat16, device=device) for _ in range(n_sets)]
        dw = torch.empty(p.w_shape, dtype=torch.bfloat16, device=device)
        dims = (p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad, p.dilation,
                p.groups, p.layout, p.dtype, gb.PATH_AUTO)
        wsd = torch.empty(max(gb.gconv2d_bwd_data_workspace_size(*dims), 16), dtype=torch.uint8,
                          device=device)
        wsw_n = gb.gconv2d_bwd_weight_workspace_size(*dims)
        wsw = torch.empty(max(wsw_n, 16), dtype=torch.uint8, device=device)
        ops = {
            "dgrad": (lambda i: gb.gconv2d_bwd_data(dys[i], w, (p.H, p.W), p.stride, p.pad,
                                                    p.dilation, p.groups, p.layout, out=dxs[i],
                                                    workspace=wsd, stream=stream),
                      gb.KERNEL_NAMES.get(gb.gconv2d_bwd_data_select_path(*dims))),
            "wgrad": (lambda i: gb.gconv2d_bwd_weight(xs[i], dys[i], (p.kH, p.kW), p.stride,
                                                      p.pad, p.dilation, p.groups, p.layout,
                                                      out=dw, workspace=wsw, stream=stream),
                      gb.KERNEL_NAMES.get(gb.gconv2d_bwd_weight_select_path(*dims))),
        }
        for op, (fn, kname) in ops.items():
            fn(0)
            torch.cuda.synchronize()
            n = r if not (tag.startswith("wide") and op == "wgrad") else 3
            med, mean = time_launches(torch, lambda i: fn(0), stream, n, flush)
            b2b = time_graph_b2b(torch, fn, stream, n_sets)
            t_tensor = p.flops() / (pk["bf16_tflops"] * 1e12)
            t_hbm = p.bytes() / (pk["hbm_gbs"] * 1e9)
            bound = "tensor" if t_tensor >= t_hbm else "hbm"
            rec = {"kernel": kname, "us": round(med * 1e3, 2),
                   "TFLOP/s": round(p.flops() / (med * 1e-3) / 1e12, 1),
                   "GB/s": round(p.bytes() / (med * 1e-3) / 1e9, 1), "bound": bound,
                   "frac": round(max(t_tensor, t_hbm) / (med * 1e-3), 3),
                   "us_b2b": round(b2b * 1e3, 2),
                   "frac_b2b": round(max(t_tensor, t_hbm) / (b2b * 1e-3), 3),
                   "alg_bytes": p.bytes(), "alg_flops": p.flops()}
            if op == "wgrad":
                rec["workspace_bytes"] = wsw_n
            out[f"{tag}_{op}"] = rec
        del xs, w, dys, dxs, dw, wsd, wsw
    return out


# ---------------------------------------------------------------------------- CPU oracle

def oracle_sample(p, inp_x64, inp_w64, target_s: float):
    """Time the fp64 oracle on the first rows of the workload, growing the sample until it
    takes about `target_s` seconds. Returns (TFLOP/s, seconds, rows, threads)."""
    import oracle
    rows = 2
    while True:
        if p.layout == wl.NCHW:
            xs = np.ascontiguousarray(inp_x64[:, :, :rows, :])
        else:
            xs = np.ascontiguousarray(inp_x64[:, :rows, :, :])
        t0 = time.perf_counter()
        y = oracle.conv2d(xs, inp_w64, None, p.stride, p.pad, p.dilation, p.groups, p.layout)
        dt = time.perf_counter() - t0
        Ho, Wo = (y.shape[2], y.shape[3]) if p.layout == wl.NCHW else (y.shape[1], y.shape[2])
        flops = 2 * p.N * Ho * Wo * p.C_out * p.cpg_in * p.kH * p.kW
        if dt >= target_s * 0.5 or rows >= p.H:
            return flops / dt / 1e12, dt, rows, oracle.num_threads()
        rows = min(p.H, max(rows + 1, int(rows * target_s / max(dt, 1e-3) * 0.8)))


def run_reference(args):
    """--impl reference: the fp64 oracle on host cores, same metric and unit."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    p = conv2d_problem(args.layout)
    inp = wl.make_conv2d_inputs(p, 2)
    x64, w64 = inp.x64(), inp.w64()
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    for i in range(args.warmup + args.steps):
        v, dt, rows, thr = oracle_sample(p, x64, w64, per_step)
        if i >= args.warmup:
            vals.append((v, dt, rows, thr))
    value = statistics.median(v for v, *_ in vals)
    rows, thr = vals[-1][2], vals[-1][3]
    sample = (f"first {rows} of {p.H} input rows of the workload (all channels, groups, taps), "
              f"fp64 nested loops, {thr} OpenMP threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(statistics.median(dt for _, dt, *_ in vals) * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(p, args),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": thr,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_dict(p, args):
    return {"workload": f"wide-group conv2d x[1,512,256,256] w[512,128,3,3] groups=4 pad=1 "
                        f"bf16/fp32-acc {args.layout.upper()}",
            "N": p.N, "C_in": p.C_in, "H": p.H, "W": p.W, "C_out": p.C_out, "kH": p.kH,
            "kW": p.kW, "groups": p.groups, "stride": p.stride, "pad": p.pad,
            "layout": args.layout.upper(), "global_batch": p.N * max(1, args.gpus),
            "l2": "rotating buffer sets larger than 2x L2 between timed steps",
            "l2_secondary": "before each timed launch of the other workloads: 252 MB written, "
                            "then 252 MB read (cold L2 holding clean lines)",
            "parallelism": f"replicas x{max(1, args.gpus)}"}


# ---------------------------------------------------------------------------- main

PROFILE_WORKLOADS = ("wide_group_nhwc", "wide_group_nchw", "ensemble_g64", "depthwise56_s1",
                     "depthwise56_s2", "dw1d_same", "dw1d_same_direct", "sweep56_g64", "sweep56_g16",
                     "depthwise56_bwd", "depthwise56_s2_bwd", "wide_group_dgrad",
                     "wide_group_wgrad", "dwsep1d", "grouped_linear", "wide_group_avg")


def run_profile(name: str, reps: int, batch: int = 0) -> int:
    """--profile: run one workload's launches `reps` times (no timing), for profiler captures;
    `batch` > 0 replaces the conv2d workload's batch size (a smaller capture)."""
    import torch

    from depthwise_convolution_gconv2d_b200 import binding as gb
    device = torch.device("cuda", 0)
    if name == "dw1d_same_direct":
        # the forward on the CUDA-core 128-byte-row kernel (the DIRECT family)
        p = wl.conformer_dw1d(False)
        inp = wl.make_dwconv1d_inputs(p, 3)
        x, w = (dev_tensor(torch, a, p.dtype, device) for a in (inp.x, inp.w))
        for _ in range(reps):
            gb.dwconv1d_fwd(x, w, p.pad_left, p.pad_right, path=gb.PATH_DIRECT)
    elif name == "dw1d_same":
        p = wl.conformer_dw1d(False)
        inp = wl.make_dwconv1d_inputs(p, 3)
        x, w, dy = (dev_tensor(torch, a, p.dtype, device) for a in (inp.x, inp.w, inp.dy))
        for _ in range(reps):
            gb.dwconv1d_fwd(x, w, p.pad_left, p.pad_right)
            gb.dwconv1d_bwd_data(dy, w, p.T, p.pad_left, p.pad_right)
            gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right)
    elif name == "dwsep1d":
        p = wl.conformer_dw1d(False)
        inp = wl.make_dwsep1d_inputs(p, 512, 7)
        x, wdw, wpw, b = (dev_tensor(torch, a, p.dtype, device)
                          for a in (inp.x, inp.w_dw, inp.w_pw, inp.bias))
        for _ in range(reps):
            gb.dwsep1d_fwd(x, wdw, wpw, b, p.pad_left, p.pad_right)
    elif name == "wide_group_wgrad":
        p = wl.wide_group(wl.NHWC)
        if batch > 0:
            p = dataclasses.replace(p, N=batch)
        inp = wl.make_conv2d_inputs(p, 5)
        x = dev_tensor(torch, inp.x, p.dtype, device)
        dy = dev_tensor(torch, wl.make_conv2d_dy(p, 5), p.dtype, device)
        for _ in range(reps):
            gb.gconv2d_bwd_weight(x, dy, (p.kH, p.kW), p.stride, p.pad, p.dilation, p.groups,
                                  p.layout)
    elif name == "wide_group_avg":
        p = wl.wide_group(wl.NHWC)
        inp = wl.make_conv2d_inputs(p, 2)
        x, w = dev_tensor(torch, inp.x, p.dtype, device), dev_tensor(torch, inp.w, p.dtype, device)
        for _ in range(reps):
            gb.gconv2d_fwd_out(x, w, None, p.stride, p.pad, p.dilation, p.groups, p.layout, "avg")
    elif name in ("depthwise56_bwd", "depthwise56_s2_bwd", "wide_group_dgrad"):
        p = {"depthwise56_bwd": lambda: wl.depthwise_56(1),
             "depthwise56_s2_bwd": lambda: wl.depthwise_56(2),
             "wide_group_dgrad": lambda: wl.wide_group(wl.NHWC)}[name]()
        if batch > 0:
            p = dataclasses.replace(p, N=batch)
        inp = wl.make_conv2d_inputs(p, 5)
        x, w = dev_tensor(torch, inp.x, p.dtype, device), dev_tensor(torch, inp.w, p.dtype, device)
        dy = dev_tensor(torch, wl.make_conv2d_dy(p, 5), p.dtype, device)
        for _ in range(reps):
            gb.gconv2d_bwd_data(dy, w, (p.H, p.W), p.stride, p.pad, p.dilation, p.groups,
                                p.layout)
            if name != "wide_group_dgrad":
                gb.gconv2d_bwd_weight(x, dy, (p.kH, p.kW), p.stride, p.pad, p.dilation,
                                      p.groups, p.layout)
    else:
        p = {"wide_group_nhwc": lambda: wl.wide_group(wl.NHWC),
             "wide_group_nchw": lambda: wl.wide_group(wl.NCHW),
             "ensemble_g64": wl.ensemble_groups,
             "depthwise56_s1": lambda: wl.depthwise_56(1),
             "depthwise56_s2": lambda: wl.depthwise_56(2),
             "sweep56_g64": lambda: wl.depthwise_56(1, 64),
             "sweep56_g16": lambda: wl.depthwise_56(1, 16),
             "grouped_linear": wl.grouped_linear}[name]()
        if batch > 0:
            p = dataclasses.replace(p, N=batch)
        inp = wl.make_conv2d_inputs(p, 2)
        x, w = dev_tensor(torch, inp.x, p.dtype, device), dev_tensor(torch, inp.w, p.dtype, device)
        # every launch writes its own y: the outputs are kept, so a capture of launch k > 1
        # with --cache-control none sees launch k-1's dirty y lines written back to DRAM
        ys = []
        for _ in range(reps):
            ys.append(gb.gconv2d_fwd(x, w, None, p.stride, p.pad, p.dilation, p.groups,
                                     p.layout))
    torch.cuda.synchronize()
    code = gb.device_error()
    print(json.dumps({"profile": name, "reps": reps, "device_error": code}))
    return 0 if code == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layout", default="nhwc", choices=["nhwc", "nchw"])
    ap.add_argument("--path", default="auto", choices=["auto", "direct", "igemm", "generic"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-depthwise", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--profile", choices=PROFILE_WORKLOADS,
                    help="run this workload's launches --profile-reps times for a profiler "
                         "capture, untimed, and exit")
    ap.add_argument("--profile-reps", type=int, default=2)
    ap.add_argument("--profile-batch", type=int, default=0,
                    help="batch size of the --profile conv2d workload (0: the workload's own)")
    args = ap.parse_args()
    if args.profile:
        return run_profile(args.profile, args.profile_reps, args.profile_batch)
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from depthwise_convolution_gconv2d_b200 import binding as gb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    pk, peak_src = peaks()

    p = conv2d_problem(args.layout)
    path = {"auto": gb.PATH_AUTO, "direct": gb.PATH_DIRECT, "igemm": gb.PATH_IGEMM,
            "generic": gb.PATH_GENERIC}[args.path]
    kcode = gb.gconv2d_select_path(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad,
                                   p.dilation, p.groups, p.layout, p.dtype, path)
    inp = wl.make_conv2d_inputs(p, 2 + 100 * rank)
    x_host = torch.from_numpy(np.ascontiguousarray(inp.x).view(np.int16)).view(torch.bfloat16)
    w_host = torch.from_numpy(np.ascontiguousarray(inp.w).view(np.int16)).view(torch.bfloat16)
    step_bytes = (x_host.numel() + p.N * p.C_out * p.Ho * p.Wo) * 2
    nsets = max(2, -(-4 * L2_BYTES // step_bytes))       # >= 2x L2 between reuses
    xs = [x_host.to(device) for _ in range(nsets)]
    w = w_host.to(device)
    ys = [torch.empty(p.y_shape, dtype=torch.bfloat16, device=device) for _ in range(nsets)]
    ws_need = gb.gconv2d_fwd_workspace_size(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride,
                                            p.pad, p.dilation, p.groups, p.layout, p.dtype, path)
    ws = torch.empty(max(ws_need, 16), dtype=torch.uint8, device=device)

    # the C ABI call with its arguments marshalled once (device pointers rotate per step)
    import ctypes
    lib = gb.load_library()
    fixed = (p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad, p.dilation, p.groups,
             p.layout, p.dtype, path)
    tail = (ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(ws.numel()),
            ctypes.c_void_p(stream.cuda_stream))
    wptr = ctypes.c_void_p(w.data_ptr())
    xptrs = [ctypes.c_void_p(t.data_ptr()) for t in xs]
    yptrs = [ctypes.c_void_p(t.data_ptr()) for t in ys]

    def step(i):
        st = lib.gconv2d_fwd_path(xptrs[i % nsets], wptr, None, yptrs[i % nsets], *fixed, *tail)
        if st != 0:
            raise gb.GconvError(st, "gconv2d_fwd_path")

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    # one launch per step and no events between the steps (an event recorded between two
    # launches kept the next one from starting until the first had fully drained: ~5 us a
    # launch, measured), so the kernel's average launch duration is the region's time / K
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.25)
        gpu_spin(torch, stream, 500)
        t_start.record(stream)
        for i in range(args.steps):
            step(i)
        t_end.record(stream)
        torch.cuda.synchronize()
        time.sleep(0.25)
    total_ms = t_start.elapsed_time(t_end)
    local_ms = total_ms
    if world > 1:
        total_ms = max_over_ranks(torch, dist, total_ms, device)
        dist.barrier()

    flops = p.flops()
    value = flops * world * args.steps / (total_ms * 1e-3) / 1e12
    avg_launch_ms = local_ms / args.steps
    achieved = flops / (avg_launch_ms * 1e-3) / 1e12
    clocks = clk.summary()
    tensor_peak, which = tensor_peak_for(pk, total_ms * 1e-3, clocks)
    tr = traffic_for(kernel_name(kcode), KERNEL_SOURCE.get(kcode, ""))
    roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": tensor_peak,
            "unit": "TFLOP/s", "frac": round(achieved / tensor_peak, 4),
            "traffic": tr.get("dram_bytes_per_launch") if tr else None,
            "kernel": kernel_name(kcode),
            "peak_source": f"{which} {peak_src} (timed region {total_ms:.2f} ms)",
            "frac_of_burst_peak": round(achieved / pk["bf16_tflops"], 4)}
    if pk.get("bf16_tflops_sustained"):
        roof["frac_of_sustained_peak"] = round(achieved / pk["bf16_tflops_sustained"], 4)
    if tr:
        # reads compare with x + w, writes with y: one launch of a back-to-back sequence, each
        # launch with its own y, so the previous launch's y is written back inside it
        roof["traffic_read"] = tr.get("dram_read_bytes")
        roof["traffic_write"] = tr.get("dram_write_bytes")
        roof["alg_read"] = p.bytes() - p.N * p.C_out * p.Ho * p.Wo * 2
        roof["alg_write"] = p.N * p.C_out * p.Ho * p.Wo * 2
        roof["traffic_scope"] = tr.get("note", "")
    if kcode in (1, 2):   # CUDA-core kernels on this workload are not tensor-bound
        roof["note"] = "CUDA-core path selected; tensor peak used as the headline denominator"

    # e2e: host (pinned) -> device copy of x and w, the call, device -> host copy of y
    e2e = None
    if True:
        x_pin = x_host.pin_memory()
        w_pin = w_host.pin_memory()
        y_pin = torch.empty(p.y_shape, dtype=torch.bfloat16).pin_memory()
        xd, wd, yd = xs[0], w, ys[0]
        def e2e_step():
            with torch.cuda.stream(stream):
                xd.copy_(x_pin, non_blocking=True)
                wd.copy_(w_pin, non_blocking=True)
            gb.gconv2d_fwd(xd, wd, None, p.stride, p.pad, p.dilation, p.groups, p.layout,
                           out=yd, workspace=ws, path=path, stream=stream)
            with torch.cuda.stream(stream):
                y_pin.copy_(yd, non_blocking=True)
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 10))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        gpu_spin(torch, stream)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b)
        if world > 1:
            e_ms = max_over_ranks(torch, dist, e_ms, device)
        e2e = {"value": round(flops * world * n_e2e / (e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": (x_host.numel() + w_host.numel()) * 2,
               "d2h_bytes_per_step": y_pin.numel() * 2, "steps": n_e2e}

    dwm = None
    more = None
    bwd = None
    if not args.no_depthwise and rank == 0:
        dwm = depthwise_measurements(torch, gb, device, stream, pk, 20)
        more = more_conv2d_measurements(torch, gb, device, stream, pk, 10)
        bwd = backward_measurements(torch, gb, device, stream, pk, 10)
        more.update(dwsep_measurements(torch, gb, device, stream, pk, 20))
    dev_err = gb.device_error(stream)

    cpu = None
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        v, dt, rows, thr = oracle_sample(p, inp.x64(), inp.w64(), args.cpu_seconds)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
               "sample": f"first {rows} of {p.H} input rows of the workload, fp64 nested loops, "
                         f"{dt:.1f} s"}

    rooflines = compact_rooflines(dwm, more, bwd)
    if rooflines:
        # the secondary workloads' fractions travel inside the headline roofline object too
        roof["others"] = rooflines
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(p, argparse.Namespace(layout=args.layout, gpus=world)),
            "kernel": kernel_name(kcode), "roofline": roof, "e2e": e2e,
            "gpu_launches": LAUNCHES_PER_CALL.get(kcode, 1) * args.steps,
            "clocks": clocks, "cpu_baseline": cpu, "rooflines": rooflines, "depthwise": dwm,
            "other_workloads": more, "backward": bwd,
            "device_error": dev_err,
            "peaks": {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                      "source": peak_src},
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
