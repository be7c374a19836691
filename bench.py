#!/usr/bin/env python
"""Benchmark: exact attention forward+backward TFLOP/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-cpu-baseline] [--sweep]

One step is one pass of the whole hot path over one batch: the forward
(fa_forward: O and LSE) followed by the backward (fa_backward: the dQ
kernel, which also forms the row statistics D and LSE2, then the dK/dV
kernel) of the workload, inputs resident in HBM.  Throughput counts the algorithmic FLOPs of both passes
(forward 4 B H N^2 d, halved when causal; backward 2.5x the forward).

Default workload: causal_d128 (B4 H16 N4096 d128, bf16, causal fwd+bwd),
the configuration the metric's target is stated at (N >= 4096, d = 128).
Its working set (~0.5 GB) is larger than the 126 MB L2, so no flush is needed
between steps.  Under torchrun each rank runs the same per-GPU workload on its
own GPU (independent heads, no collective on the data path: weak scaling);
the time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle (the only reference this
project has) on a bounded sample of the same workload, on the host cores.
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
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402
from exact_io_aware_99_b200 import perf  # noqa: E402

METRIC = "attention fwd/bwd TFLOPs/s (bf16, 1 B200) and % of dense tensor peak vs N"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, ws: int, device) -> float:
    """The largest x over all ranks (for a time: the slowest rank's), x itself
    on one rank.  Every rank must call it at the same point."""
    if ws <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(ws: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job TFLOP/s: every rank does flops_per_rank in ms (the
    max over ranks), so the job does ws times that."""
    return ws * flops_per_rank / (ms * 1e-3) / 1e12


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and throttle-reason samples taken while a timed region runs.

    Read in-process through NVML (read-only queries) every ``period_s`` by a
    background thread, so even a timed region of a few tens of milliseconds
    gets a few dozen samples; falls back to ``nvidia-smi -lms 100`` when the
    NVML bindings are missing.  Samples taken while the GPU reported itself
    busy (NVML utilisation > 0) count as under load."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clocks-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown"}

    def __init__(self, gpu_index: int, period_s: float = 0.001):
        self.gpu = gpu_index
        self.period = period_s
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []
        self.stop_evt = threading.Event()
        self.nvml = None

    def _sample_nvml(self, nv, h):
        while not self.stop_evt.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                util = nv.nvmlDeviceGetUtilizationRates(h).gpu
                self.rows.append((time.perf_counter(), float(sm), int(rs), int(util)))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.nvml = nv
            self.thread = threading.Thread(target=self._sample_nvml, args=(nv, h), daemon=True)
            self.thread.start()
            return
        except Exception:
            self.nvml = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)  # let the sampler start
        except Exception:
            self.proc = None

    def window(self, t0: float, t1: float):
        """Median and lowest SM clock and the throttle reasons seen between
        two ``time.perf_counter()`` readings (NVML samples only)."""
        rows = [r for r in self.rows if t0 <= r[0] <= t1]
        if not rows:
            return None
        reasons = sorted({name for r in rows for bit, name in self.REASONS.items() if r[2] & bit})
        return {"sm_mhz": statistics.median(r[1] for r in rows),
                "sm_mhz_min": min(r[1] for r in rows), "reasons": reasons, "samples": len(rows)}

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.nvml is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            rows = list(self.rows)
            if not rows:
                return out
            load = [r for r in rows if r[3] > 0] or rows
            reasons = set()
            for r in load:
                for bit, name in self.REASONS.items():
                    if r[2] & bit:
                        reasons.add(name)
            out.update(sm_mhz=statistics.median(r[1] for r in load), sm_max_mhz=self.max_mhz,
                       reasons=sorted(reasons), samples=len(rows),
                       samples_under_load=len([r for r in rows if r[3] > 0]),
                       sm_mhz_min=min(r[1] for r in load), source="nvml",
                       period_ms=self.period * 1e3)
            return out
        if self.proc is None:
            return out
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.unlink(self.path)
        except Exception:
            return out
        if not rows:
            return out
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        out.update(sm_mhz=statistics.median(sm) if sm else None,
                   sm_max_mhz=max(mx) if mx else None, reasons=sorted(reasons),
                   samples=len(rows), source="nvidia-smi")
        return out


# --------------------------------------------------------------- ncu traffic

KERNEL_SOURCES = {
    "bwd": ["exact_io_aware_99_b200/csrc/fa_bwd_sm100.cu", "exact_io_aware_99_b200/csrc/fa_simt.cu",
            "exact_io_aware_99_b200/csrc/sm100.cuh", "exact_io_aware_99_b200/csrc/fa_internal.h"],
    "fwd": ["exact_io_aware_99_b200/csrc/fa_fwd_sm100.cu", "exact_io_aware_99_b200/csrc/sm100.cuh",
            "exact_io_aware_99_b200/csrc/fa_internal.h"],
    "fwd8": ["exact_io_aware_99_b200/csrc/fa_fwd_fp8_sm100.cu",
             "exact_io_aware_99_b200/csrc/fa_fp8.h", "exact_io_aware_99_b200/csrc/sm100.cuh",
             "exact_io_aware_99_b200/csrc/fa_internal.h"],
}


def _code_only(text: str) -> str:
    """Source text without C/C++ comments and blank lines, so that an edit of
    a comment does not mark a profile of the unchanged kernel as stale."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_hash(kernel: str) -> str:
    """Hash of the code (comments excluded) of the sources a kernel is built from."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_ncu.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)\s+source_sha256:\s*([0-9a-f]+)", text)
    if not m or m.group(2) != source_hash(kernel):
        return None
    return float(m.group(1))


# --------------------------------------------------------------- our impl

def run_ours(args, peaks, peak_kind):
    import exact_io_aware_99_b200 as fa

    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = workloads.WORKLOADS[args.workload]
    B, H, N, d = w.B, w.H, w.N, w.d
    x = workloads.make_inputs(w, with_grad_out=True)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wbytes = fa.fa_backward_workspace_size(B, H, N, d)
    wsbuf = torch.empty(wbytes, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    scale, causal = w.scale, w.causal
    mask_np = workloads.block_mask(w)
    if mask_np is not None:
        mask = torch.from_numpy(mask_np.astype("uint8")).to(dev).contiguous()
        mh = int(mask.shape[0])

        def fwd():
            fa.fa_forward_blocksparse(q, k, v, o, lse, B, H, N, d, scale, causal, mask, mh, sp)

        def bwd():
            fa.fa_backward_blocksparse(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, scale,
                                       causal, mask, mh, wsbuf, wbytes, sp)
    else:
        def fwd():
            fa.fa_forward(q, k, v, o, lse, B, H, N, d, scale, causal, sp)

        def bwd():
            fa.fa_backward(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, scale, causal, wsbuf,
                           wbytes, sp)

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    st, site = fa.fa_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"device wait timed out in warm-up (site {site:#x})")

    # Device-timed region: K steps, events on the launching stream around
    # each pass so the per-pass (kernel) durations are measured live.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        fwd()
        ev[i][1].record(stream)
        bwd()
        ev[i][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier()
    total_ms = t_start.elapsed_time(t_end)
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    bwd_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    st, site = fa.fa_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"device wait timed out (site {site:#x})")
    total_ms = max_over_ranks(total_ms, ws, dev)
    ms_step = total_ms / args.steps

    flops_f, flops_b = step_flop_counts(w)
    step_flops = flops_f + flops_b
    value = whole_job_tflops(ws, step_flops, ms_step)

    # End to end through the public API with host buffers: pinned host inputs
    # copied in, both passes, outputs copied back, every step.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (x[n].pin_memory() for n in ("q", "k", "v", "do"))
        ho, hdq, hdk, hdv = (torch.empty_like(hq).pin_memory() for _ in range(4))
        hlse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
        bi = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
        bo = sum(t.numel() * t.element_size() for t in (ho, hlse, hdq, hdk, hdv))

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            do.copy_(hdo, non_blocking=True)
            fwd()
            bwd()
            ho.copy_(o, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)
            hdq.copy_(dq, non_blocking=True)
            hdk.copy_(dk, non_blocking=True)
            hdv.copy_(dv, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ne = max(3, min(args.steps, 10))
        a.record(stream)
        for _ in range(ne):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(a.elapsed_time(b) / ne, ws, dev)
        e2e = {"value": round(whole_job_tflops(ws, step_flops, e_ms), 3), "unit": UNIT,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": round(e_ms, 4)}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)

    extras = {}
    if ws == 1 and not args.no_extras and args.workload == "causal_d128":
        extras = run_extras(fa, dev, stream, peaks, local)

    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None

    peak = float(peaks["bf16_tflops"])
    peak_s = float(peaks.get("bf16_tflops_sustained", peak))
    bwd_tf = flops_b / (bwd_ms * 1e-3) / 1e12
    fwd_tf = flops_f / (fwd_ms * 1e-3) / 1e12
    traffic = recorded_traffic("bwd", args.workload)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded iid N(0,1), rounded to bf16)",
        "config": {"workload": w.describe(), "B": B, "H": H, "N": N, "d": d,
                   "causal": causal, "passes": "fwd+bwd",
                   "l2": "working set ~%.2f GB > 126 MB L2 (no flush needed)"
                         % ((7 * B * H * N * d * 2 + wbytes) / 1e9),
                   "parallelism": f"{ws} independent replicas" if ws > 1 else "single GPU",
                   **({"block_mask": w.mask,
                       "visible_fraction": round(float(mask_np.mean()), 4)}
                      if mask_np is not None else {})},
        "fwd_tflops": round(fwd_tf, 3), "bwd_tflops": round(bwd_tf, 3),
        "fwd_frac_of_peak": round(fwd_tf / peak, 4), "bwd_frac_of_peak": round(bwd_tf / peak, 4),
        "frac_of_peak": round(value / ws / peak, 4),
        "frac_of_sustained_peak": round(value / ws / peak_s, 4),
        "peak_source": f"{peak_kind} (MEASURED_PEAKS.json bf16_tflops burst {peak}, "
                       f"sustained {peak_s})",
        "roofline": {"kernel": "fa_backward (row statistics + dQ kernel + dK/dV kernel)",
                     "bound": "tensor", "achieved": round(bwd_tf, 3), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(bwd_tf / peak, 4),
                     "traffic": traffic,
                     "algorithmic_bytes": perf.bwd_bytes(B, H, N, d)},
        "gpu_launches": 4 * args.steps,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                   "reasons": clk["reasons"], "samples": clk["samples"]},
        "e2e": e2e,
        "cpu_baseline": cpu,
        **extras,
    }
    return line


# ------------------------------------------------------------------ extras
# The other configurations, the TFLOP/s-vs-N curve and the FP8 and decode
# paths, each timed in the same process with CUDA events on the launching
# stream (3 warm-up steps, then every timed pass bracketed by its own events),
# so one benchmark line carries all of them.  Forward-only working sets that
# fit in L2 get a 256 MB write before every timed pass.

EXTRA_ITERS = 10
EXTRA_GAP_S = 0.5  # idle before each extra entry (lets the power draw settle)


def _timed_passes(passes, stream, iters, flush=None):
    """Mean device time (ms) of each callable in ``passes`` over ``iters``
    rounds; every pass gets its own event pair (and an L2 flush first when
    ``flush`` is given)."""
    for _ in range(3):
        for f in passes:
            f()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in passes] for _ in range(iters)]
    for i in range(iters):
        for f, (a, b) in zip(passes, ev[i]):
            if flush is not None:
                flush.zero_()
            a.record(stream)
            f()
            b.record(stream)
    torch.cuda.synchronize()
    return [statistics.mean(ev[i][p][0].elapsed_time(ev[i][p][1]) for i in range(iters))
            for p in range(len(passes))]


def _dense_entry(fa, dev, stream, B, H, N, d, causal, backward, inputs, peak, flush=None):
    """Forward (and backward) TFLOP/s of one dense bf16 problem."""
    q, k, v = (inputs[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    sp = stream.cuda_stream
    sc = 1.0 / math.sqrt(d)

    def f():
        fa.fa_forward(q, k, v, o, lse, B, H, N, d, sc, causal, sp)
    passes = [f]
    if backward:
        do = inputs["do"].to(dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        wb = fa.fa_backward_workspace_size(B, H, N, d)
        wsb = torch.empty(wb, device=dev, dtype=torch.uint8)

        def g():
            fa.fa_backward(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, sc, causal, wsb, wb, sp)
        passes.append(g)
    ms = _timed_passes(passes, stream, EXTRA_ITERS, flush)
    ff = perf.fwd_flops(B, H, N, d, causal)
    out = {"B": B, "H": H, "N": N, "d": d, "causal": causal,
           "fwd_ms": round(ms[0], 4), "fwd_tflops": round(ff / (ms[0] * 1e-3) / 1e12, 2)}
    out["fwd_frac_of_peak"] = round(out["fwd_tflops"] / peak, 4)
    if backward:
        fb = perf.bwd_flops(B, H, N, d, causal)
        out.update(bwd_ms=round(ms[1], 4), bwd_tflops=round(fb / (ms[1] * 1e-3) / 1e12, 2))
        out["bwd_frac_of_peak"] = round(out["bwd_tflops"] / peak, 4)
        out["step_tflops"] = round((ff + fb) / ((ms[0] + ms[1]) * 1e-3) / 1e12, 2)
    if flush is not None:
        out["l2"] = "flushed before every timed pass (256 MB write)"
    return out


def _device_randn(shape, seed, dev):
    g = torch.Generator(device=dev).manual_seed(seed)
    return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)


def _projected_inputs(w, dev):
    """The GPT-3-shaped workload's Q, K, V (X W projections) and dO, drawn
    from the workload's seed on the CPU with the projections multiplied on
    the GPU in fp32 (timing input only; the parity tests use the CPU
    product)."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    x = torch.randn(w.B, w.N, w.hidden, generator=g, dtype=torch.float32).to(dev)
    out = {}
    for name in ("q", "k", "v"):
        wm = (torch.randn(w.hidden, w.H * w.d, generator=g, dtype=torch.float32) * 0.02).to(dev)
        pr = torch.matmul(x, wm).view(w.B, w.N, w.H, w.d).permute(0, 2, 1, 3).contiguous()
        out[name] = pr.to(torch.bfloat16)
    out["do"] = torch.randn(w.B, w.H, w.N, w.d, generator=g, dtype=torch.float32).to(
        torch.bfloat16).to(dev)
    return out


def run_extras(fa, dev, stream, peaks, gpu_index):
    peak = float(peaks["bf16_tflops"])
    hbm = float(peaks.get("hbm_gbs", 6534.8))
    flush = torch.empty(256 << 20, device=dev, dtype=torch.uint8)
    clocks = ClockSampler(gpu_index, period_s=0.005)
    clocks.start()
    windows = []  # (entry dict, t0, t1): the clock samples of each entry's timed passes

    def entry(fn):
        # A short idle gap first, so that one entry's power draw does not cap
        # the clock of the next; each entry then carries its own clocks.
        torch.cuda.synchronize()
        time.sleep(EXTRA_GAP_S)
        t0 = time.perf_counter()
        out = fn()
        windows.append((out, t0, time.perf_counter()))
        return out

    configs = {}
    w = workloads.WORKLOADS["fwd_d64"]
    x = workloads.make_inputs(w)
    configs["fwd_d64"] = entry(lambda: _dense_entry(fa, dev, stream, w.B, w.H, w.N, w.d,
                                                    w.causal, False, x, peak, flush))
    for name in ("long_d128", "gpt3_d80"):
        w = workloads.WORKLOADS[name]
        x = _projected_inputs(w, dev) if w.projected else workloads.make_inputs(w)
        configs[name] = entry(lambda: _dense_entry(fa, dev, stream, w.B, w.H, w.N, w.d,
                                                   w.causal, True, x, peak))
        del x
    vs_n = []
    for causal in (True, False):
        for N in (512, 1024, 2048, 4096, 8192, 16384):
            H, d = 16, 128
            B = max(1, 262144 // (H * N))
            x = {n: _device_randn((B, H, N, d), 5000 + 10 * N + i + 7 * causal, dev)
                 for i, n in enumerate(("q", "k", "v", "do"))}
            vs_n.append(entry(lambda: _dense_entry(fa, dev, stream, B, H, N, d, causal, True, x,
                                                   peak)))
            del x
    # FP8 forward at the target shape (E4M3 codes from the library's own
    # per-tensor quantiser), L2 flushed before every pass
    w = workloads.WORKLOADS["fp8_causal_d128"]
    q8, qd = fa.quantize_fp8(_device_randn((w.B, w.H, w.N, w.d), 7001, dev))
    k8, kd = fa.quantize_fp8(_device_randn((w.B, w.H, w.N, w.d), 7002, dev))
    v8, vd = fa.quantize_fp8(_device_randn((w.B, w.H, w.N, w.d), 7003, dev))
    o8 = torch.empty((w.B, w.H, w.N, w.d), device=dev, dtype=torch.bfloat16)
    l8 = torch.empty((w.B, w.H, w.N), device=dev, dtype=torch.float32)

    def f8():
        fa.fa_forward_fp8(q8, k8, v8, qd, kd, vd, o8, l8, w.B, w.H, w.N, w.d, w.scale, w.causal,
                          stream.cuda_stream)
    ms8 = entry(lambda: {"ms": _timed_passes([f8], stream, EXTRA_ITERS, flush)[0]})["ms"]
    tf8 = perf.fwd_flops(w.B, w.H, w.N, w.d, w.causal) / (ms8 * 1e-3) / 1e12
    fp8 = {"workload": w.describe(), "fwd_ms": round(ms8, 4), "fwd_tflops": round(tf8, 2),
           "frac_of_fp8_peak": round(tf8 / (2 * peak), 4),
           "fp8_peak": round(2 * peak, 1), "fp8_peak_source": "2 x measured bf16 (nominal ratio)",
           "l2": "flushed before every timed pass (256 MB write)"}
    del q8, k8, v8, o8
    # split-KV decode (bound by reading K and V)
    w = workloads.WORKLOADS["decode_d128"]
    qd_ = _device_randn((w.B, w.H, w.N, w.d), 7101, dev)
    kd_ = _device_randn((w.B, w.H, w.nk, w.d), 7102, dev)
    vd_ = _device_randn((w.B, w.H, w.nk, w.d), 7103, dev)
    od_ = torch.empty_like(qd_)
    ld_ = torch.empty((w.B, w.H, w.N), device=dev, dtype=torch.float32)
    splits = fa.fa_splitkv_default_splits(w.B, w.H, w.N, w.nk)
    wb = fa.fa_splitkv_workspace_size(w.B, w.H, w.N, w.nk, w.d, splits)
    wsb = torch.empty(wb, device=dev, dtype=torch.uint8)

    def fdec():
        fa.fa_forward_splitkv(qd_, kd_, vd_, od_, ld_, w.B, w.H, w.N, w.nk, w.d, w.scale,
                              w.causal, splits, wsb, wb, stream.cuda_stream)
    msd = entry(lambda: {"ms": _timed_passes([fdec], stream, EXTRA_ITERS)[0]})["ms"]
    nbytes = perf.decode_bytes(w.B, w.H, w.N, w.nk, w.d)
    gbs = nbytes / (msd * 1e-3) / 1e9
    decode = {"workload": w.describe(), "num_splits": splits, "fwd_ms": round(msd, 4),
              "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / hbm, 4),
              "tflops": round(perf.decode_flops(w.B, w.H, w.N, w.nk, w.d, w.causal)
                              / (msd * 1e-3) / 1e12, 2),
              "algorithmic_bytes": nbytes,
              "l2": "K/V %.2f GB > 126 MB L2" % (2 * w.B * w.H * w.nk * w.d * 2 / 1e9)}
    clk = clocks.stop()
    win = [clocks.window(t0, t1) for _, t0, t1 in windows]
    for (out, _, _), c in zip(windows, win):
        if c is not None:
            out["clocks"] = c
    # the FP8 and decode timings went through scratch dicts (the last two)
    if win[-2] is not None:
        fp8["clocks"] = win[-2]
    if win[-1] is not None:
        decode["clocks"] = win[-1]
    st, site = fa.fa_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"device wait timed out in the extra measurements (site {site:#x})")
    return {"configs": configs, "vs_n": vs_n, "fp8_fwd": fp8, "decode": decode,
            "extras_clocks": clk,
            "extras_note": "each entry CUDA-event timed in this process after 3 warm-up "
                           f"steps, mean of {EXTRA_ITERS} timed passes, after {EXTRA_GAP_S} s "
                           "idle; its 'clocks' are the NVML samples of its own timed passes; "
                           "fractions of the measured bf16 peak (burst)"}


# ------------------------------------------------------------- CPU oracle

def run_decode(args, peaks, peak_kind):
    """Split-KV decode workload: forward only, N_q queries against N_k keys.
    Bound by HBM (K and V are read once per query tile pair), so the roofline
    is GB/s of algorithmic bytes against the measured copy bandwidth."""
    import exact_io_aware_99_b200 as fa

    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = workloads.WORKLOADS[args.workload]
    B, H, Nq, Nk, d = w.B, w.H, w.N, w.nk, w.d
    x = workloads.make_decode_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), device=dev, dtype=torch.float32)
    splits = args.splits if args.splits else fa.fa_splitkv_default_splits(B, H, Nq, Nk)
    wbytes = fa.fa_splitkv_workspace_size(B, H, Nq, Nk, d, splits)
    wsbuf = torch.empty(wbytes, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def fwd():
        fa.fa_forward_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, w.scale, w.causal, splits, wsbuf,
                              wbytes, sp)

    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        fwd()
    b.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    st, site = fa.fa_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"device wait timed out (site {site:#x})")
    ms = a.elapsed_time(b) / args.steps
    ms = max_over_ranks(ms, ws, dev)
    flops = perf.decode_flops(B, H, Nq, Nk, d, w.causal)
    nbytes = perf.decode_bytes(B, H, Nq, Nk, d)
    value = whole_job_tflops(ws, flops, ms)
    gbs = nbytes / (ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
        ho = torch.empty_like(hq).pin_memory()
        hlse = torch.empty((B, H, Nq), dtype=torch.float32).pin_memory()
        bi = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        bo = sum(t.numel() * t.element_size() for t in (ho, hlse))

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            fwd()
            ho.copy_(o, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ne = max(3, min(args.steps, 10))
        ea.record(stream)
        for _ in range(ne):
            e2e_step()
        eb.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(ea.elapsed_time(eb) / ne, ws, dev)
        e2e = {"value": round(whole_job_tflops(ws, flops, e_ms), 3), "unit": UNIT,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": round(e_ms, 4)}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        from oracle.decode import rect_forward
        cores = os.cpu_count() or 1
        x1 = workloads.make_decode_inputs(w, B=1)
        n, t0 = 0, time.perf_counter()
        while True:
            h = n % H
            rect_forward(x1["q"][0, h], x1["k"][0, h], x1["v"][0, h], w.scale, w.causal)
            n += 1
            if time.perf_counter() - t0 >= args.cpu_seconds:
                break
        el = time.perf_counter() - t0
        cpu = {"value": round(n * perf.decode_flops(1, 1, Nq, Nk, d, w.causal) / el / 1e12, 6),
               "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n} head(s) of {w.name}, forward, fp64 numpy on the host ({el:.1f} s)"}
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None
    hbm = float(peaks.get("hbm_gbs", 6534.8))
    peak = float(peaks["bf16_tflops"])
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded iid N(0,1), rounded to bf16)",
        "config": {"workload": w.describe(), "B": B, "H": H, "N_q": Nq, "N_k": Nk, "d": d,
                   "causal": w.causal, "passes": "fwd (split-KV decode)", "num_splits": splits,
                   "l2": "K/V ~%.2f GB > 126 MB L2 (no flush needed)"
                         % (2 * B * H * Nk * d * 2 / 1e9),
                   "parallelism": f"{ws} independent replicas" if ws > 1 else "single GPU"},
        "fwd_tflops": round(value / ws, 3), "fwd_frac_of_peak": round(value / ws / peak, 4),
        "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs {hbm}, bf16_tflops {peak})",
        "roofline": {"kernel": "fa_forward_splitkv (split forward + combine)", "bound": "hbm",
                     "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(gbs / hbm, 4), "traffic": None,
                     "algorithmic_bytes": nbytes},
        "gpu_launches": 2 * args.steps,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                   "reasons": clk["reasons"], "samples": clk["samples"]},
        "e2e": e2e,
        "cpu_baseline": cpu,
    }


def run_fp8(args, peaks, peak_kind):
    """FP8 (E4M3) forward workload.  Its three E4M3 inputs (1 byte per
    element) fit in L2, so L2 is flushed (a 256 MB write) before every timed
    step and each step is timed by its own pair of events; the roofline is
    the tensor pipe at the FP8 rate, twice the measured bf16 GEMM peak (the
    nominal 4.5 / 2.25 PFLOP/s ratio)."""
    import exact_io_aware_99_b200 as fa

    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = workloads.WORKLOADS[args.workload]
    B, H, N, d = w.B, w.H, w.N, w.d
    x = workloads.make_fp8_inputs(w)
    q8, k8, v8 = (x[n].to(dev) for n in ("q8", "k8", "v8"))
    ds = {n: torch.tensor([x[n + "_descale"]], device=dev, dtype=torch.float32)
          for n in ("q", "k", "v")}
    o = torch.empty((B, H, N, d), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    flush = torch.empty(256 << 20, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def fwd():
        fa.fa_forward_fp8(q8, k8, v8, ds["q"], ds["k"], ds["v"], o, lse, B, H, N, d, w.scale,
                          w.causal, sp)

    for _ in range(args.warmup):
        flush.zero_()
        fwd()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        fwd()
        b.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    st, site = fa.fa_device_status(reset=True)
    if st != 0:
        raise RuntimeError(f"device wait timed out (site {site:#x})")
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    ms = max_over_ranks(ms, ws, dev)
    flops = perf.fwd_flops(B, H, N, d, w.causal)
    value = whole_job_tflops(ws, flops, ms)

    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x[n].pin_memory() for n in ("q8", "k8", "v8"))
        ho = torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
        hlse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
        bi = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        bo = sum(t.numel() * t.element_size() for t in (ho, hlse))

        def e2e_step():
            q8.copy_(hq, non_blocking=True)
            k8.copy_(hk, non_blocking=True)
            v8.copy_(hv, non_blocking=True)
            fwd()
            ho.copy_(o, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ne = max(3, min(args.steps, 10))
        ea.record(stream)
        for _ in range(ne):
            e2e_step()
        eb.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(ea.elapsed_time(eb) / ne, ws, dev)
        e2e = {"value": round(whole_job_tflops(ws, flops, e_ms), 3), "unit": UNIT,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": round(e_ms, 4)}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None
    bf16_peak = float(peaks["bf16_tflops"])
    peak = 2.0 * bf16_peak
    achieved = value / ws
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic (seeded iid N(0,1) fp32, quantised per tensor to E4M3)",
        "config": {"workload": w.describe(), "B": B, "H": H, "N": N, "d": d,
                   "causal": w.causal, "passes": "fwd (FP8)",
                   "l2": "flushed before every timed step (256 MB write; inputs %.0f MB < L2)"
                         % (3 * B * H * N * d / 1e6),
                   "parallelism": f"{ws} independent replicas" if ws > 1 else "single GPU"},
        "fwd_tflops": round(achieved, 3),
        "fwd_frac_of_bf16_peak": round(achieved / bf16_peak, 4),
        "peak_source": (f"{peak_kind}: bf16_tflops {bf16_peak} x 2 (nominal FP8 / bf16 dense "
                        f"ratio 4.5 / 2.25 PFLOP/s)"),
        "roofline": {"kernel": "fwd_fp8_kernel", "bound": "tensor", "achieved": round(achieved, 1),
                     "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic("fwd8", args.workload),
                     "algorithmic_flops": flops},
        "gpu_launches": args.steps,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                   "reasons": clk["reasons"], "samples": clk["samples"]},
        "e2e": e2e,
        "cpu_baseline": cpu,
    }


def step_flop_counts(w, B=None, H=None):
    """Algorithmic forward and backward FLOPs of one step of workload w
    (visible pairs only for a block-sparse workload)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    if w.nk:
        return perf.decode_flops(B, H, w.N, w.nk, w.d, w.causal), 0.0
    if w.dtype == "e4m3":
        return perf.fwd_flops(B, H, w.N, w.d, w.causal), 0.0
    m = workloads.block_mask(w)
    if m is not None:
        return (perf.fwd_flops_masked(B, H, w.N, w.d, w.causal, m),
                perf.bwd_flops_masked(B, H, w.N, w.d, w.causal, m))
    return perf.fwd_flops(B, H, w.N, w.d, w.causal), perf.bwd_flops(B, H, w.N, w.d, w.causal)


def oracle_head_step(w, x, h):
    """Forward and backward of head h of x on the fp64 oracle (the
    block-sparse oracle for a block-sparse workload)."""
    import oracle
    if w.nk:
        from oracle.decode import rect_forward
        rect_forward(x["q"][0, h], x["k"][0, h], x["v"][0, h], w.scale, w.causal)
        return
    if w.dtype == "e4m3":
        from oracle.fp8 import forward
        forward(x["q8"][0, h], x["k8"][0, h], x["v8"][0, h], x["q_descale"], x["k_descale"],
                x["v_descale"], w.scale, w.causal)
        return
    qh, kh, vh, doh = (x[n][0, h] for n in ("q", "k", "v", "do"))
    m = workloads.block_mask(w)
    if m is not None:
        from oracle.block_sparse import block_sparse_backward, block_sparse_forward
        block_sparse_forward(qh, kh, vh, w.scale, m, w.causal)
        block_sparse_backward(qh, kh, vh, doh, w.scale, m, w.causal)
    else:
        oracle.attention_forward(qh, kh, vh, w.scale, w.causal)
        oracle.attention_backward(qh, kh, vh, doh, w.scale, w.causal)


def cpu_baseline(w, seconds: float):
    """The fp64 oracle (as it stands) on a bounded sample of the workload:
    whole heads, forward and backward, until about ``seconds`` of CPU work."""
    x = (workloads.make_fp8_inputs(w, B=1) if w.dtype == "e4m3"
         else workloads.make_inputs(w, with_grad_out=True, B=1))
    cores = os.cpu_count() or 1
    n_heads, flops, t0 = 0, 0.0, time.perf_counter()
    per_head = sum(step_flop_counts(w, B=1, H=1))
    while True:
        oracle_head_step(w, x, n_heads % w.H)
        n_heads += 1
        flops += per_head
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    return {"value": round(flops / el / 1e12, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_heads} head(s) of {w.name} (N={w.N}, d={w.d}), "
                      f"{'fwd+bwd' if w.backward else 'fwd'}, fp64 numpy "
                      f"on the host ({el:.1f} s)"}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return None
    w = workloads.WORKLOADS[args.workload]
    if w.nk:
        x = workloads.make_decode_inputs(w, B=1)
    elif w.dtype == "e4m3":
        x = workloads.make_fp8_inputs(w, B=1)
    else:
        x = workloads.make_inputs(w, with_grad_out=True, B=1)
    per_head = sum(step_flop_counts(w, B=1, H=1))
    passes = "fwd+bwd" if w.backward else "fwd"

    def step(i):
        oracle_head_step(w, x, i % w.H)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    value = per_head * args.steps / el / 1e12
    cores = os.cpu_count() or 1
    sample = f"1 head of {w.name} (N={w.N}, d={w.d}) {passes} per step, fp64 numpy oracle"
    return {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.describe(), "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "causal": w.causal, "passes": passes,
                       "timed_per_step": {"B": 1, "H": 1, "N": w.N, "d": w.d,
                                          "note": "one head of the workload per step "
                                                  "(heads cycle); value = its FLOPs / time"}},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_sweep(args, peaks):
    """Forward and backward TFLOP/s vs N at d = 128, causal and not, holding
    B*H*N = 262144 (one line per point; not the benchmark line)."""
    import exact_io_aware_99_b200 as fa
    peak = float(peaks["bf16_tflops"])
    for causal in (True, False):
        for N in (512, 1024, 2048, 4096, 8192, 16384):
            d = 128
            H = 16
            B = max(1, 262144 // (H * N))
            x = workloads.random_case(B, H, N, d, N, grad=True)
            q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
            o = torch.empty_like(q)
            lse = torch.empty((B, H, N), device="cuda")
            dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
            wb = fa.fa_backward_workspace_size(B, H, N, d)
            wsb = torch.empty(wb, device="cuda", dtype=torch.uint8)
            sc = 1 / math.sqrt(d)

            def f():
                fa.fa_forward(q, k, v, o, lse, B, H, N, d, sc, causal)

            def g():
                fa.fa_backward(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, sc, causal, wsb, wb)

            res = {}
            for name, fn, fl in (("fwd", f, perf.fwd_flops(B, H, N, d, causal)),
                                 ("bwd", g, perf.bwd_flops(B, H, N, d, causal))):
                for _ in range(3):
                    f()
                    fn()
                torch.cuda.synchronize()
                a, b = torch.cuda.Event(True), torch.cuda.Event(True)
                n = 10
                a.record()
                for _ in range(n):
                    fn()
                b.record()
                torch.cuda.synchronize()
                ms = a.elapsed_time(b) / n
                res[name] = fl / (ms * 1e-3) / 1e12
            print(json.dumps({"sweep": "d128", "causal": causal, "B": B, "H": H, "N": N,
                              "fwd_tflops": round(res["fwd"], 2),
                              "bwd_tflops": round(res["bwd"], 2),
                              "fwd_frac": round(res["fwd"] / peak, 4),
                              "bwd_frac": round(res["bwd"] / peak, 4)}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description="exact attention fwd+bwd benchmark (B200)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="causal_d128", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configs, the vs-N curve and the FP8/decode entries")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--sweep", action="store_true", help="print the TFLOP/s-vs-N sweep instead")
    ap.add_argument("--splits", type=int, default=0,
                    help="key splits for a decode workload (0: the library's default)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    peaks, kind = load_peaks()
    if args.impl == "reference":
        line = run_reference(args)
    elif args.sweep:
        run_sweep(args, peaks)
        return
    elif workloads.WORKLOADS[args.workload].nk:
        line = run_decode(args, peaks, kind)
    elif workloads.WORKLOADS[args.workload].dtype == "e4m3":
        line = run_fp8(args, peaks, kind)
    else:
        line = run_ours(args, peaks, kind)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
