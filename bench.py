"""Benchmark of the exact tiled attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload dense_causal|packed_causal|long_outlier|mxfp8_packed|
                     mxfp8_incoherent|nvfp4_packed]
                    [--pass fwd|bwd]

One step = one ``attn_fwd`` call through the C ABI (the schedule-build
kernel, the MXFP8 pre-pass for the MXFP8 workload, and the attention
kernel) over the workload's whole batch, inputs resident in HBM.  Prints one
JSON line (rank 0).  Throughput is TFLOP/s with the causal FLOP convention
4 L^2 d / 2 per head and document.  Under torchrun each rank runs the same
workload on its own GPU (independent replicas, weak scaling: the path has no
cross-GPU exchange); the time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload and prints the same metric (rank 0 only).

``--pass bwd`` times the backward instead (bf16 workloads): one step = one
``attn_bwd`` call (schedule, D pre-pass, backward kernel, dQ conversion)
with the forward's out and lse resident; FLOPs = 2.5 x the forward's (five
products against two); the fp64 gradient oracle is the CPU baseline, and
``--impl reference --pass bwd`` times that oracle the same way.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_tiled_attention_39_b200 import workloads  # noqa: E402

METRIC = "attention fwd TFLOP/s (causal, bf16 & MXFP8) and % of B200 dense tensor peak"
METRIC_BWD = ("attention bwd TFLOP/s (causal, bf16 & MXFP8; 2.5 x forward FLOPs) and % of B200 "
              "dense tensor peak")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# attn_api.cu holds, after the forward's host code, one section per later
# part, each opening with one of these marker lines.
BWD_SECTION_MARK = b"\n// " + b"=" * 75 + b"\n// Backward (bf16)"
INCOHERENT_SECTION_MARK = b"\n// " + b"=" * 75 + b"\n// Incoherent processing"

# The CUDA sources each measured kernel is built and launched from, and the
# marker where that part's share of attn_api.cu ends.
FWD_SOURCES = ["attn_api.cu", "attn_fwd_pair_sm100.cuh", "attn_fwd_sm100.cuh", "common.cuh",
               "incoherent.cuh", "ptx.cuh", "quant_mxfp8.cuh", "quant_nvfp4.cuh", "schedule.cuh",
               "tmem_ops.cuh"]
PART_SOURCES = {
    "fwd": (FWD_SOURCES, BWD_SECTION_MARK),
    "bwd": (FWD_SOURCES + ["attn_bwd_sm100.cuh"], INCOHERENT_SECTION_MARK),
}


def kernel_sources_sha256(part: str = "fwd") -> str:
    """Hash of the CUDA sources (names and bytes, sorted by name) a measured
    kernel is built and launched from: "fwd" the forward kernels, "bwd" the
    backward (the forward's files, the backward kernel's, and attn_api.cu up
    to the next part's section)."""
    import hashlib
    d = os.path.join(ROOT, "exact_tiled_attention_39_b200", "csrc")
    files, end_mark = PART_SOURCES[part]
    h = hashlib.sha256()
    for n in sorted(files):
        h.update(n.encode())
        with open(os.path.join(d, n), "rb") as f:
            data = f.read()
        if n == "attn_api.cu":
            cut = data.find(end_mark)
            if cut >= 0:
                data = data[:cut]
        h.update(data)
    return h.hexdigest()


def recorded_traffic(workload: str, kernel: str, part: str = "fwd"):
    """DRAM bytes (read + write) per attention-kernel launch from the committed
    ncu summary of this kernel and workload, or None when there is none or it
    was taken on other kernel sources."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            line = line.strip().strip("`")
            for key in ("kernel_sources_sha256", "dram_bytes_per_launch"):
                if line.startswith(key + ":"):
                    vals[key] = line.split(":", 1)[1].strip()
    if vals.get("kernel_sources_sha256") != kernel_sources_sha256(part):
        return None
    try:
        return int(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def init_group(backend: str, device=None):
    """Process group over the launcher's ranks (torchrun env, 127.0.0.1
    rendezvous), or None for one process.  A short timeout makes ranks that
    wait for a missing peer fail instead of hanging."""
    world, _, _ = dist_env()
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    kw = {"device_id": device} if backend == "nccl" else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def max_over_ranks(pg, value: float, device) -> float:
    """The largest of every rank's value (every rank gets it)."""
    if pg is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job throughput: every rank runs the same workload (independent
    replicas), the job takes the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """SM clock and throttle-reason samples while the timed kernels run.

    NVML is polled from a background thread about every millisecond (the
    timed regions last milliseconds, far shorter than nvidia-smi's sampling
    period); without NVML, nvidia-smi is sampled every 100 ms instead."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device):
        self.device = device
        self.proc = None
        self.thread = None
        self.samples = []       # (sm_mhz, max_mhz, set of reasons)
        self.source = "none"

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            props = torch.cuda.get_device_properties(self.device)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId_v2(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            masks = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
            self._stop = threading.Event()

            def poll():
                while not self._stop.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    except Exception:
                        break
                    self.samples.append((float(sm), float(mx),
                                         {n for n, m in masks if rs & m}))
                    time.sleep(0.001)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = "nvml, ~1 ms"
        except Exception:
            self.thread = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.device.index or 0),
                     f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms",
                     "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi, 100 ms"
                time.sleep(0.25)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = [n for n, _ in self.REASONS]
            for line in out.splitlines():
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, mx = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                self.samples.append((sm, mx, {n for n, v in zip(names, parts[5:9])
                                              if v.lower() == "active"}))
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [x[0] for x in self.samples]
        loaded = [x for x in sm if x >= 0.5 * max(sm)] or sm
        reasons = set()
        for x in self.samples:
            reasons |= x[2]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": self.samples[-1][1],
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source,
                "window": "timed steps and the per-kernel timing launches"}


KERNEL_TIMING_LAUNCHES = 50       # per-kernel time: median of at least this many launches
KERNEL_TIMING_MIN_S = 0.05        # ... and of at least this much device time
EXTRA_WORKLOADS = ("packed_causal", "long_outlier", "mxfp8_packed", "mxfp8_incoherent",
                   "nvfp4_packed")


def kernel_name_for(dtype_name: str) -> str:
    """Every forward form (bf16, MXFP8, NVFP4) runs the two-query-tile
    kernel."""
    return "attn_fwd_pair_kernel"


def measure_workload(A, name, steps, warmup, dev, stream, pg, clk):
    """Time one workload: after `warmup` untimed calls, the attention kernel
    alone (CUDA events the library records on the launching stream around
    that kernel; median over at least KERNEL_TIMING_LAUNCHES launches and
    KERNEL_TIMING_MIN_S of device time), then `steps` back-to-back attn_fwd
    calls (device events, barrier + synchronize on both sides, max over
    ranks).  Returns the figures and the device tensors for the end-to-end
    leg."""
    w = workloads.get(name)
    inp = workloads.make_inputs(w)
    T, H, d = inp["q"].shape
    causal = True
    dtype = {"mxfp8": A.ATTN_MXFP8, "nvfp4": A.ATTN_NVFP4}.get(w.dtype, A.ATTN_BF16)
    lengths = inp["lengths"]
    max_seqlen = max(lengths)
    flops = workloads.flops(lengths, H, d, causal)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    cu = inp["cu_seqlens"].to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    ws = A.make_workspace(A.Shape(T, len(lengths), H, d, max_seqlen), dtype, dev)
    if w.incoherent:
        signs = inp["signs"].to(dev)

        def step():
            A.attn_fwd_incoherent(q, k, v, cu, out, lse, causal, inp["scale"], signs,
                                  stream=stream, workspace=ws, max_seqlen=max_seqlen)
    else:
        def step():
            A.attn_fwd(q, k, v, cu, out, lse, causal, inp["scale"], dtype=dtype, stream=stream,
                       workspace=ws, max_seqlen=max_seqlen)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    assert A.attn_get_device_error(ws) == 0, f"device error during warm-up ({name})"

    with clk:
        # The attention kernel alone, before the timed steps: it also brings
        # the GPU from idle (input generation) to its steady clocks, so the
        # timed steps below measure steady-state throughput.
        A.attn_timing_enable(True)
        per, pre = [], []
        while len(per) < KERNEL_TIMING_LAUNCHES or sum(per) < 1e3 * KERNEL_TIMING_MIN_S:
            step()
            a_ms, p_ms = A.attn_timing_read()
            per.append(a_ms)
            pre.append(p_ms)
            if len(per) >= 20000:
                break
        A.attn_timing_enable(False)
        # ---- device-timed region: `steps` back-to-back steps, barrier +
        # synchronize on both sides
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    ms_total = max_over_ranks(pg, t0.elapsed_time(t1), dev)
    ms_step = ms_total / steps
    err = A.attn_get_device_error(ws)
    return {
        "w": w, "inp": inp, "dtype": dtype, "flops": flops, "ms_total": ms_total,
        "ms_step": ms_step, "kernel_ms": statistics.median(per),
        "prepass_ms": statistics.median(pre), "launches_timed": len(per), "err": err,
        "tensors": (q, k, v, cu, out, lse), "step": step,
        "launches_per_step": 2 if dtype == A.ATTN_BF16 else 3,
    }


# Nominal dense tensor rate of each operand type relative to bf16.
LOWP_RATIO = {"mxfp8": 2.0, "nvfp4": 4.0}


def roofline_for(m, peaks, peak_src):
    """Roofline of the attention kernel: algorithmic FLOPs / its median
    launch time against the measured dense bf16 peak.  The block-scaled
    kernels run Q K^T on low-precision operands (2 x bf16 for E4M3, 4 x for
    E2M1, the nominal ratios) and P V in bf16, half of the FLOPs each, so
    their peak is the time-weighted mix 2 / (1 / r + 1); the fraction of the
    plain low-precision peak (r x bf16) is given as well."""
    peak_key = "bf16_tflops_sustained" if m["ms_total"] * 1e-3 > 1.0 else "bf16_tflops"
    bf16 = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    r = LOWP_RATIO.get(m["w"].dtype)
    peak = bf16 if r is None else bf16 * 2.0 / (1.0 / r + 1.0)
    achieved = m["flops"] / (m["kernel_ms"] * 1e-3) / 1e12
    kernel = kernel_name_for(m["w"].dtype)
    src = peak_source_name(peak_key, 0)
    if r is not None:
        src += (f"; Q K^T at {r:g} x bf16 ({m['w'].dtype} operands), P V at bf16, half the "
                f"FLOPs each: {2.0 / (1.0 / r + 1.0):.3f} x bf16")
    out = {
        "bound": "tensor",
        "achieved": round(achieved, 2),
        "peak": round(peak, 1),
        "unit": "TFLOP/s",
        "frac": round(achieved / peak, 4),
        "peak_source": f"{src} ({peak_src})",
        "timed_unit": (f"attention kernel alone (CUDA events around its launch), median of "
                       f"{m['launches_timed']} launches"),
        "kernel_ms": round(m["kernel_ms"], 4),
        "prepass_ms": round(m["prepass_ms"], 4),
        "kernel": kernel,
        "traffic": recorded_traffic(m["w"].name, kernel),
        "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
    }
    if r is not None:
        out[f"frac_of_{m['w'].dtype}_peak"] = round(achieved / (bf16 * r), 4)
    return out


def bench_ours(args):
    from exact_tiled_attention_39_b200 import attn as A

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = init_group("nccl", dev)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()

    clk = ClockSampler(dev)
    m = measure_workload(A, args.workload, args.steps, args.warmup, dev, stream, pg, clk)
    w, inp, dtype, flops = m["w"], m["inp"], m["dtype"], m["flops"]
    q, k, v, cu, out, lse = m["tensors"]
    step = m["step"]
    T, H, d = inp["q"].shape
    lengths = inp["lengths"]
    value = aggregate_tflops(world, flops, m["ms_step"])

    # ---- end to end through the public API: pinned host in, host out
    hq, hk, hv = (inp[n].pin_memory() for n in ("q", "k", "v"))
    hcu = inp["cu_seqlens"].pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        cu.copy_(hcu, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
        hlse.copy_(lse, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    e2e_step()
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    s1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(pg, s0.elapsed_time(s1) / e2e_steps, dev)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcu))
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
    roof = roofline_for(m, peaks, peak_src)
    ms_step, err = m["ms_step"], m["err"]
    del m, q, k, v, cu, out, lse, step, e2e_step, hq, hk, hv, hout, hlse
    torch.cuda.empty_cache()

    # ---- the other workloads of the metric (packed, long context, MXFP8):
    # same protocol, reported beside the headline
    extra = {}
    if not args.no_extra_workloads and args.workload == "dense_causal":
        for name in EXTRA_WORKLOADS:
            xclk = ClockSampler(dev)
            mx = measure_workload(A, name, args.steps, args.warmup, dev, stream, pg, xclk)
            extra[name] = {
                "workload": f"{name}: {mx['w'].description}",
                "dtype": mx["w"].dtype,
                "tokens": mx["inp"]["tokens"], "heads": mx["inp"]["q"].shape[1],
                "docs": len(mx["inp"]["lengths"]), "flops_per_step": mx["flops"],
                "ms_per_step": round(mx["ms_step"], 4),
                "value": round(aggregate_tflops(world, mx["flops"], mx["ms_step"]), 2),
                "unit": "TFLOP/s",
                "roofline": roofline_for(mx, peaks, peak_src),
                "clocks": xclk.summary(),
                "device_error": mx["err"],
                "gpu_launches": args.steps * mx["launches_per_step"],
            }
            del mx
            torch.cuda.empty_cache()

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return None

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) bf16, see workloads.py)",
        "config": workload_config(w, inp, world),
        "roofline": roof,
        "e2e": {
            "value": round(aggregate_tflops(world, flops, e2e_ms), 2),
            "unit": "TFLOP/s",
            "ms_per_step": round(e2e_ms, 3),
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
        },
        "gpu_launches": args.steps * (2 if dtype == A.ATTN_BF16 else 3),
        "clocks": clk.summary(),
        "device_error": err,
    }
    if extra:
        line["workloads"] = extra
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w, inp, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {key: cb[key] for key in ("value", "unit", "cores", "kind",
                                                         "sample")}
    return line


def workload_config(w, inp, world: int) -> dict:
    """The `config` object of a workload's line (the same keys in both arms)."""
    T, H, d = inp["q"].shape
    return {
        "workload": f"{w.name}: {w.description}",
        "tokens": T, "heads": H, "head_dim": d, "docs": len(inp["lengths"]),
        "causal": True, "flops_per_step": workloads.flops(inp["lengths"], H, d, True),
        "l2": f"inputs {3 * T * H * d * 2 / 1e6:.0f} MB > 126 MB L2; no flush",
        "parallelism": f"replicas x{world}",
    }


def peak_source_name(key, dtype):
    base = {"bf16_tflops": "bf16 burst", "bf16_tflops_sustained": "bf16 sustained"}[key]
    return base + (" x2 for fp8" if dtype == 1 else "")


def cpu_baseline(w, inp, budget_s=15.0):
    """Time the fp64 oracle on the host cores on a bounded sample of the
    workload: whole (document, head) problems, as many as fit the budget."""
    from oracle.attention import ref_attention
    from oracle.incoherent import incoherent_operands
    from oracle.mxfp8 import quantize_mxfp8_ref, dequantize_mxfp8_ref
    from oracle.nvfp4 import dequantize_nvfp4_ref, quantize_nvfp4_ref

    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    lengths = inp["lengths"]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    H, d = inp["q"].shape[1], inp["q"].shape[2]
    # order: documents first, heads second, largest documents first
    problems = [(i, h) for i in np.argsort(lengths)[::-1] for h in range(H)]
    done_flops, done = 0.0, 0
    t_start = time.perf_counter()
    for i, h in problems:
        a, b = int(starts[i]), int(starts[i + 1])
        q = inp["q"][a:b, h:h + 1].double().numpy()
        k = inp["k"][a:b, h:h + 1].double().numpy()
        v = inp["v"][a:b, h:h + 1].double().numpy()
        scale = inp["scale"]
        if w.dtype == "nvfp4":
            q, k = (dequantize_nvfp4_ref(*quantize_nvfp4_ref(x)) for x in (q, k))
            v = dequantize_mxfp8_ref(*quantize_mxfp8_ref(v))
        elif w.incoherent:
            q, k, v, scale = incoherent_operands(q, k, v, scale, inp["signs"].numpy())
        elif w.dtype == "mxfp8":
            q, k, v = (dequantize_mxfp8_ref(*quantize_mxfp8_ref(x)) for x in (q, k, v))
        ref_attention(q, k, v, [0, b - a], True, scale)
        done_flops += workloads.flops([b - a], 1, d, True)
        done += 1
        if time.perf_counter() - t_start > budget_s:
            break
    el = time.perf_counter() - t_start
    return {"value": round(done_flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{done} of {len(problems)} (document, head) problems, fp64, "
                      f"{el:.1f} s", "seconds": el, "problems": done}


def cpu_baseline_bwd(inp, dout, budget_s=15.0, mxfp8=False):
    """The fp64 gradient oracle on the host cores on whole (document, head)
    problems of the workload, largest documents first, within the budget
    (the MXFP8 gradient oracle for an MXFP8 workload)."""
    from oracle.attention_bwd import ref_attention_bwd, ref_attention_bwd_mxfp8

    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    lengths = inp["lengths"]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    H, d = inp["q"].shape[1], inp["q"].shape[2]
    problems = [(i, h) for i in np.argsort(lengths)[::-1] for h in range(H)]
    done_flops, done = 0.0, 0
    t_start = time.perf_counter()
    for i, h in problems:
        a, b = int(starts[i]), int(starts[i + 1])
        x = [t[a:b, h:h + 1].double().numpy() for t in (inp["q"], inp["k"], inp["v"], dout)]
        (ref_attention_bwd_mxfp8 if mxfp8 else ref_attention_bwd)(*x, [0, b - a], True,
                                                                  inp["scale"])
        done_flops += 2.5 * workloads.flops([b - a], 1, d, True)
        done += 1
        if time.perf_counter() - t_start > budget_s:
            break
    el = time.perf_counter() - t_start
    return {"value": round(done_flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{done} of {len(problems)} (document, head) problems, fp64 gradients, "
                      f"{el:.1f} s", "seconds": el, "problems": done}


def bench_ours_bwd(args):
    from exact_tiled_attention_39_b200 import attn as A

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = init_group("nccl", dev)

    w = workloads.get(args.workload)
    if w.incoherent or w.dtype == "nvfp4":
        raise SystemExit("--pass bwd: the backward covers the bf16 and MXFP8 paths")
    dtype = A.ATTN_MXFP8 if w.dtype == "mxfp8" else A.ATTN_BF16
    inp = workloads.make_inputs(w)
    T, H, d = inp["q"].shape
    causal = True
    lengths = inp["lengths"]
    max_seqlen = max(lengths)
    flops = 2.5 * workloads.flops(lengths, H, d, causal)
    g = torch.Generator().manual_seed(1000 + w.seed)
    hdo = torch.randn((T, H, d), generator=g).to(torch.bfloat16)

    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    do = hdo.to(dev)
    cu = inp["cu_seqlens"].to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    shape = A.Shape(T, len(lengths), H, d, max_seqlen)
    A.attn_fwd(q, k, v, cu, out, lse, causal, inp["scale"], dtype=dtype, max_seqlen=max_seqlen)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = A.make_bwd_workspace(shape, dev, dtype)
    stream = torch.cuda.current_stream(dev)

    def step():
        A.attn_bwd(q, k, v, out, do, lse, cu, dq, dk, dv, causal, inp["scale"], stream=stream,
                   workspace=ws, max_seqlen=max_seqlen, dtype=dtype)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert A.attn_get_device_error(ws) == 0, "device error during warm-up"

    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    ms_total = max_over_ranks(pg, t0.elapsed_time(t1), dev)
    ms_step = ms_total / args.steps
    err = A.attn_get_device_error(ws)
    value = aggregate_tflops(world, flops, ms_step)

    # end to end: q, k, v, out, dout, lse, cu_seqlens in from pinned host
    # memory, dq, dk, dv back
    host_in = [inp["q"].pin_memory(), inp["k"].pin_memory(), inp["v"].pin_memory(),
               out.cpu().pin_memory(), hdo.pin_memory(), lse.cpu().pin_memory(),
               inp["cu_seqlens"].pin_memory()]
    dev_in = [q, k, v, out, do, lse, cu]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]

    def e2e_step():
        for dst, src in zip(dev_in, host_in):
            dst.copy_(src, non_blocking=True)
        step()
        for dst, src in zip(host_out, (dq, dk, dv)):
            dst.copy_(src, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    e2e_step()
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    s1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(pg, s0.elapsed_time(s1) / e2e_steps, dev)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    peak_key = "bf16_tflops_sustained" if ms_total * 1e-3 > 1.0 else "bf16_tflops"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    achieved = flops / (ms_step * 1e-3) / 1e12
    line = {
        "metric": METRIC_BWD,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "mxfp8" if dtype == A.ATTN_MXFP8 else "bf16",
        "data": "synthetic (seeded N(0,1) bf16, see workloads.py; dout seeded N(0,1))",
        "config": dict(workload_config(w, inp, world),
                       workload=f"{w.name} backward: {w.description}", flops_per_step=flops,
                       l2=f"inputs {6 * q.numel() * 2 / 1e6:.0f} MB > 126 MB L2; no flush"),
        "roofline": {
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_source": f"{peak_source_name(peak_key, 0)} ({peak_src})",
            "timed_unit": (f"whole attn_bwd call ({5 if dtype == A.ATTN_MXFP8 else 4} kernels), "
                           "device events over the timed steps"),
            "kernel": "attn_bwd_kernel",
            "traffic": recorded_traffic(w.name, "attn_bwd_kernel", "bwd"),
            "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
        },
        "e2e": {
            "value": round(aggregate_tflops(world, flops, e2e_ms), 2),
            "unit": "TFLOP/s",
            "ms_per_step": round(e2e_ms, 3),
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
        },
        "gpu_launches": args.steps * (5 if dtype == A.ATTN_MXFP8 else 4),
        "clocks": clk.summary(),
        "device_error": err,
    }
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline_bwd(inp, hdo, budget_s=args.cpu_budget, mxfp8=dtype == A.ATTN_MXFP8)
        line["cpu_baseline"] = {key: cb[key] for key in ("value", "unit", "cores", "kind",
                                                         "sample")}
    return line


def bench_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    w = workloads.get(args.workload)
    inp = workloads.make_inputs(w)
    T, H, d = inp["q"].shape
    bwd = getattr(args, "which", "fwd") == "bwd"
    if bwd:
        # the same seeded upstream gradient as the GPU arm
        dout = torch.randn((T, H, d), generator=torch.Generator().manual_seed(1000 + w.seed))
        dout = dout.to(torch.bfloat16)

        def sample(budget_s):
            return cpu_baseline_bwd(inp, dout, budget_s=budget_s, mxfp8=w.dtype == "mxfp8")
    else:
        def sample(budget_s):
            return cpu_baseline(w, inp, budget_s=budget_s)
    budget = max(2.0, args.cpu_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        sample(budget)
    vals = [sample(budget) for _ in range(args.steps)]
    v = round(statistics.median(x["value"] for x in vals), 6)
    step_s = [x["seconds"] for x in vals]
    n_prob = [x["problems"] for x in vals]
    flops = (2.5 if bwd else 1.0) * workloads.flops(inp["lengths"], H, d, True)
    cfg = workload_config(w, inp, world)
    if bwd:
        cfg["workload"] = f"{w.name} backward: {w.description}"
        cfg["flops_per_step"] = flops
        cfg["l2"] = f"inputs {6 * T * H * d * 2 / 1e6:.0f} MB > 126 MB L2; no flush"
    n_all = len(inp["lengths"]) * H
    sample_desc = (f"each step: whole (document, head) problems, largest documents first, "
                   f"until {budget:.1f} s of fp64 {'gradient ' if bwd else ''}oracle work "
                   f"({min(n_prob)}-{max(n_prob)} of {n_all} problems); value = FLOPs done / "
                   f"time, median over steps")
    return {
        "impl": "reference",
        "metric": METRIC_BWD if bwd else METRIC,
        "value": v,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * statistics.mean(step_s), 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16, see workloads.py)",
        "config": cfg,
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": vals[0]["cores"],
                         "kind": "oracle", "sample": sample_desc},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "note": "ms_per_step is the host time of one timed sample step, not of the whole "
                "workload",
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="dense_causal", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="time only --workload (default: dense_causal plus the packed, "
                         "long-context and MXFP8 workloads as a `workloads` sub-object)")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd"])
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        line = bench_reference(args)
    else:
        from exact_tiled_attention_39_b200 import build
        if dist_env()[1] == 0 or not os.path.exists(build.LIB):
            build.build()
        line = bench_ours_bwd(args) if args.which == "bwd" else bench_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
