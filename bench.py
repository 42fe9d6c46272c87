#!/usr/bin/env python
"""Benchmark of the Muon optimizer step on one B200 per process.

A step is the whole hot path over one batch of matrices: momentum + Nesterov +
Frobenius norm + cast (1 kernel), then 10 hybrid Newton-Schulz steps (3 grouped
GEMM kernels each), the last one fused with the RMS rescale, decoupled weight
decay and parameter update. Default workload: the dense transformer stack of
16 layers at d = 4096 (per layer Q, K, V, O 4096 x 4096, gate and up 4096 x
14336, down 14336 x 4096 on the transposed path: 112 fp32 matrices, W, G and M
resident in HBM, 46.7 GB, far larger than the 126 MB L2, so no explicit L2
flush between steps), bf16 Newton-Schulz operands. `--config batch64_1024`
runs 64 square 1024 x 1024 matrices instead.

Metric: Newton-Schulz TFLOP/s of the whole step, with the FLOPs the metric
defines, 10 (4 r^2 c + 2 r^3) per matrix (r = min(n, m), c = max(n, m)), and
the step time in ms. The roofline of the dominant kernel counts the FLOPs its
tiles execute (the symmetric stages skip the upper tiles). Multi-GPU: every
rank runs its own batch (independent problems, no data-path collective, weak
scaling); value = FLOPs of all ranks / the slowest rank's time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --mode distributed   # one workload shared by the ranks (strong scaling)
    python bench.py --impl reference     # the float64 CPU oracle, timed on a sample
"""

from __future__ import annotations

import argparse
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

METRIC = "Muon step ms & Newton–Schulz TFLOPS (% of B200 bf16 dense peak) per shape set"
UNIT = "TFLOP/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
HYBRID = ((3.4445, -4.7750, 2.0315),) * 8 + ((2.0, -1.5, 0.5),) * 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--mode", choices=["independent", "distributed"], default="independent",
                    help="independent: every rank steps its own copy of the workload (weak "
                         "scaling); distributed: the ranks share one workload, each stepping "
                         "the matrices it owns, then one all-gather of the weights (strong "
                         "scaling)")
    ap.add_argument("--config", default="dense_d4096")
    ap.add_argument("--precision", choices=["bf16", "fp32"], default="bf16")
    ap.add_argument("--scale-mode", choices=["shape", "unit_rms", "none"], default="shape",
                    help="update scale: sqrt(max(n, m)) gamma (default), unit RMS times gamma, or none")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches, not a CUDA graph")
    ap.add_argument("--stagewise", action="store_true",
                    help="one launch per Newton-Schulz stage instead of the chained launch")
    ap.add_argument("--chain-window", type=int, default=0,
                    help="matrices the chained launch keeps in flight (0: from the tile counts)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=6, help="matrices in the CPU-baseline sample")
    ap.add_argument("--no-adamw", action="store_true", help="skip the AdamW companion measurement")
    ap.add_argument("--count", type=int, default=None,
                    help="a smaller case of the workload for profiling (not a benchmark line): "
                         "this many layers (dense_d4096), experts (moe_64x3) or matrices (the "
                         "others)")
    return ap.parse_args()


def metric_flops(shapes, ns_steps=10):
    """FLOPs the metric defines: ns_steps * (4 r^2 c + 2 r^3) per matrix."""
    tot = 0.0
    for n, m in shapes:
        r, c = min(n, m), max(n, m)
        tot += ns_steps * (4.0 * r * r * c + 2.0 * r ** 3)
    return tot


def apply_bytes(shapes):
    """Algorithmic HBM bytes of one Apply launch: B (bf16 r x r) read once, the
    iterate (bf16 high + low parts, r x c) read once and written once:
    2 r^2 + 8 r c per matrix."""
    return sum(2.0 * min(n, m) ** 2 + 8.0 * min(n, m) * max(n, m) for n, m in shapes)


TINY_ELEMS = 4096  # matrices of at most this many elements: the tiny fp32 kernel


def one_cta_kind(n, m, precision="bf16"):
    """Launch kind of the one-CTA kernel that runs a matrix (5 small, 8 mid,
    9 tiny), or None when it takes the grouped stage kernels."""
    if precision != "bf16":
        return None
    r, c = min(n, m), max(n, m)
    if r * c <= TINY_ELEMS:
        return 9
    if r <= 128 and c <= 128:
        return 5
    if r <= 128 and c <= 512:
        return 8
    return None


def stage_bytes(kind, shapes, precision="bf16"):
    """Algorithmic HBM bytes of one launch of a grouped stage over these
    matrices: each operand read once, each result written once.
                   bf16 operands                               fp32 operands
      Gram (1)     X high part read, A written: 2rc + 2r^2     X read, A written: 4rc + 4r^2
      Poly (2)     A read, B written: 4r^2                     8r^2
      Apply (3)    B read, X high + low in and out: 2r^2 + 8rc B read, X in and out: 4r^2 + 8rc
      ApplyLast(4) B, X in, W read and written: 2r^2 + 12rc    4r^2 + 12rc"""
    f = 2.0 if precision == "bf16" else 4.0
    tot = 0.0
    for n, m in shapes:
        r, c = float(min(n, m)), float(max(n, m))
        tot += {1: f * r * c + f * r * r, 2: 2 * f * r * r, 3: f * r * r + 8 * r * c,
                4: f * r * r + 12 * r * c}[kind]
    return tot


def executed_stage_flops(kind, shapes, precision="bf16"):
    """FLOPs one launch of a grouped stage executes over these matrices. With
    bf16 operands the symmetric stages (Gram, Poly) run only the 128 x 128
    blocks on or below the diagonal, clipped to the matrix; the fp32 kernels
    and Apply run the whole product."""
    tot = 0.0
    for n, m in shapes:
        r, c = min(n, m), max(n, m)
        if kind in (3, 4) or precision != "bf16":
            tot += 2.0 * r * r * (r if kind == 2 else c)
            continue
        k = c if kind == 1 else r
        rb = -(-r // 128)
        for i in range(rb):
            rows = min(128, r - 128 * i)
            for j in range(i + 1):
                tot += 2.0 * rows * min(128, r - 128 * j) * k
    return tot


def dominant_roofline(kinds, per_kind_ms, shapes, peaks, precision="bf16", ns_steps=10):
    """Roofline record of the kernel kind with the largest total time.

    per_kind_ms maps a launch kind to the list of its launch durations (ms).
    Bytes and FLOPs are per launch and algorithmic: the grouped stages by
    stage_bytes / executed_stage_flops over the matrices they run; the
    elementwise kernel 16 B per element of every matrix; a one-CTA kernel
    12 B per element (iterate high and low parts in, W in and out) and every
    step's FLOPs. The bound is whichever of FLOPs at the sustained bf16 peak
    or bytes at the HBM copy bandwidth takes longer."""
    share = {k: sum(v) for k, v in per_kind_ms.items()}
    dom = max(share, key=lambda k: share[k])
    avg_ms = share[dom] / len(per_kind_ms[dom])
    stage = "stage_tc_kernel" if precision == "bf16" else "stage_simt_kernel"
    names = {0: "ew_kernel", 1: f"{stage}<Gram>", 2: f"{stage}<Poly>", 3: f"{stage}<Apply>",
             4: f"{stage}<ApplyLast>", 5: "ns_small_kernel", 8: "ns_mid_kernel",
             9: "ns_tiny_kernel", 6: "rms_reduce_kernel", 7: "finish_kernel",
             10: "stage_chain_kernel"}
    grouped = [(n, m) for n, m in shapes if one_cta_kind(n, m, precision) is None]
    if dom in (1, 2, 3, 4):
        flops = executed_stage_flops(dom, grouped, precision)
        nbytes = stage_bytes(dom, grouped, precision)
    elif dom == 10:
        # every Gram, Poly and Apply stage but the last Apply (fused with the
        # update, its own launch); bytes as if each stage read its operands
        # and wrote its results through HBM
        per = {k: (executed_stage_flops(k, grouped, precision), stage_bytes(k, grouped, precision))
               for k in (1, 2, 3)}
        flops = ns_steps * (per[1][0] + per[2][0] + per[3][0]) - per[3][0]
        nbytes = ns_steps * (per[1][1] + per[2][1] + per[3][1]) - per[3][1]
    elif dom in (5, 8, 9):
        mine = [(n, m) for n, m in shapes if one_cta_kind(n, m, precision) == dom]
        flops = sum(ns_steps * (4.0 * min(n, m) ** 2 * max(n, m) + 2.0 * min(n, m) ** 3)
                    for n, m in mine)
        nbytes = sum(12.0 * n * m for n, m in mine)
    else:
        flops = 0.0
        nbytes = sum(16.0 * n * m for n, m in shapes)
    tensor_peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    hbm_peak = float(peaks["hbm_gbs"])
    t_tensor = flops / (tensor_peak * 1e12)
    t_hbm = nbytes / (hbm_peak * 1e9)
    if t_hbm >= t_tensor:
        achieved = nbytes / (avg_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak}
    else:
        achieved = flops / (avg_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": achieved / tensor_peak}
    roof.update({"kind": dom, "kernel": names.get(dom, str(dom)), "launch_ms": avg_ms,
                 "flops_per_launch": flops, "bytes_per_launch": nbytes})
    return roof


def max_over_ranks(x, device, world):
    """The job-wide maximum of a per-rank number (the slowest rank's time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank, world, steps, ms_max):
    """Whole-job throughput: the FLOPs of every rank over the slowest rank's time."""
    return flops_per_rank * world * steps / (ms_max / 1e3) / 1e12


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count() or 1)
    except Exception:
        return os.cpu_count() or 1


def cpu_oracle_rate(wl_cpu_mats, hyper, budget_s=None):
    """Time the float64 oracle (as it stands) on a list of (W, G, M) numpy
    matrices; returns (TFLOP/s by the metric's count, seconds, matrices done)."""
    from oracle import muon_oracle

    t0 = time.perf_counter()
    done = []
    for W, G, M in wl_cpu_mats:
        muon_oracle.muon_step(W, G, M, lr=hyper["lr"], mu=hyper["mu"], wd=hyper["wd"],
                              gamma=hyper["gamma"], nesterov_on=hyper["nesterov"])
        done.append(W.shape)
        if budget_s is not None and time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return metric_flops(done) / dt / 1e12, dt, len(done)


def _nvml_uuid(local_rank):
    """NVML's name for the CUDA device, "GPU-<uuid>", or None."""
    try:
        import torch
        return "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        return None


class NvmlClockReader:
    """SM clock and clock-event reasons of one GPU, read through NVML every
    `period_s` seconds in a background thread, with host timestamps. Read-only
    queries; any NVML failure leaves the reader without samples."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, index, uuid=None, period_s=0.01, nvml=None):
        self.index, self.uuid, self.period_s = index, uuid, period_s
        self.nvml = nvml
        self.samples = []  # (monotonic time, SM MHz, reason bit mask)
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None

    def start(self):
        try:
            if self.nvml is None:
                import pynvml
                self.nvml = pynvml
            nv = self.nvml
            nv.nvmlInit()
            handle = None
            if self.uuid:
                try:
                    handle = nv.nvmlDeviceGetHandleByUUID(self.uuid)
                except Exception:
                    handle = None
            if handle is None:
                handle = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM))
            reasons = (getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None)
                       or nv.nvmlDeviceGetCurrentClocksThrottleReasons)
        except Exception:
            self.nvml = None
            return False

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append((time.monotonic(),
                                         float(nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)),
                                         int(reasons(handle))))
                except Exception:
                    return
                self._stop.wait(self.period_s)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return True

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2.0)
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self, t0, t1):
        """Median SM clock and the reasons seen between host times t0 and t1
        (None without samples there)."""
        win = [s for s in self.samples if t0 is not None and t1 is not None and t0 <= s[0] <= t1]
        if not win:
            return None
        reasons = sorted({nm for _, _, mask in win for nm, bit in self.REASONS if mask & bit})
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(win), "source": "nvml, timed region"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms from before
    the warm-up to the end of the timed region, and NVML read every 10 ms
    inside the timed region (used when it has samples there)."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, uuid=None, nvml=None):
        self.index = index
        self.proc = None
        self.path = None
        self.reader = NvmlClockReader(index, uuid=uuid, nvml=nvml)
        self.t0 = self.t1 = None

    def window_begin(self):
        self.t0 = time.monotonic()

    def window_end(self):
        self.t1 = time.monotonic()

    def start(self):
        self.reader.start()
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        self.reader.stop()
        smi = self._stop_smi()
        nv = self.reader.summary(self.t0, self.t1)
        if nv is None:
            return smi
        nv["smi_samples"] = smi.get("samples", 0)
        return nv

    def _stop_smi(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = [l.split(",") for l in open(self.path).read().splitlines() if l.strip()]
        os.unlink(self.path)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvidia-smi, warm-up and timed region"}


KERNEL_SOURCES = ("muon_step_b200/csrc/ns_tc.cu", "muon_step_b200/csrc/ptx_sm100.cuh",
                  "muon_step_b200/csrc/stage_common.cuh", "muon_step_b200/csrc/muon_internal.h")


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(config, kind=3):
    """Per-launch DRAM bytes of the dominant stage kernel (launch kind `kind`)
    from the committed ncu summary of this workload, or None when there is
    none, it covers another kernel, or the kernel sources changed since the
    counters were taken."""
    path = os.path.join(ROOT, "profiles", f"ns_stages_{config}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    k = re.search(r"^traffic_kind:\s*([0-9]+)\s*$", text, re.M)
    if (int(k.group(1)) if k else 3) != kind:
        return None
    m = re.search(r"^traffic_per_launch_bytes:\s*([0-9.eE+]+)\s*$", text, re.M)
    h = re.search(r"^kernel_source_sha256:\s*([0-9a-f]+)\s*$", text, re.M)
    if not m or not h or h.group(1) != kernel_source_hash():
        return None
    return float(m.group(1))


ADAMW_VOCAB = 32000


def time_adamw_companion(wl, steps, dev, stream, peaks, world):
    """The AdamW group a model with these matrices would carry: an embedding
    and a prediction head of ADAMW_VOCAB rows by the model width (the most
    common matrix dimension), plus two norm vectors per matrix. One launch per
    step, timed with CUDA events over `steps` steps; HBM-bound, 28 B/element."""
    import torch

    import muon_step_b200 as ms

    dims = {}
    for n, m in wl.shapes:
        for d in (n, m):
            dims[d] = dims.get(d, 0) + 1
    width = max(dims, key=lambda d: (dims[d], -d))
    sizes = [ADAMW_VOCAB * width, ADAMW_VOCAB * width] + [width] * (2 * wl.count)
    gen = torch.Generator(device=dev).manual_seed(1234)
    tensors = []
    for n in sizes:
        p = torch.randn(n, generator=gen, device=dev) * 0.02
        g = torch.randn(n, generator=gen, device=dev) * 1e-3
        tensors.append((p, g, torch.zeros_like(p), torch.zeros_like(p)))
    plan = ms.AdamWPlan(tensors)
    ws = plan.alloc_workspace()
    for t in range(1, 4):
        plan.execute(ws, step=t, stream=stream)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for t in range(4, 4 + steps):
        plan.execute(ws, step=t, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    t_ms = max_over_ranks(e0.elapsed_time(e1), dev, world) / steps
    elems = plan.numel
    gbs = 28.0 * elems / (t_ms / 1e3) / 1e9
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return {"elements": elems, "tensors": len(sizes), "width": width, "vocab": ADAMW_VOCAB,
            "ms_per_step": t_ms, "achieved_gbs": gbs, "frac_hbm": gbs / hbm,
            "bytes_per_element": 28, "gpu_launches_per_step": 1}


def run_reference(args, rank, world):
    """Reference arm: the float64 CPU oracle, timed on host cores, rank 0 only."""
    if rank != 0:
        return
    import numpy as np
    import workloads

    # a bounded sample of the workload: one matrix of its first shape per step
    wl = workloads.make(args.config, device="cpu", **_small_kwargs(args.config))
    mats = [(wl.W[k].double().numpy(), wl.G[k].double().numpy(), wl.M[k].double().numpy())
            for k in range(1)]
    h = wl.hyper
    for _ in range(args.warmup):
        cpu_oracle_rate(mats, h)
    times = []
    for _ in range(args.steps):
        rate, dt, _n = cpu_oracle_rate(mats, h)
        times.append(dt)
    tot = sum(times)
    value = metric_flops([mats[0][0].shape]) * args.steps / tot / 1e12
    cores = oracle_threads()
    sample = f"1 matrix {mats[0][0].shape[0]}x{mats[0][0].shape[1]} of {args.config} per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": args.config},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def count_kwargs(config, count):
    """Keyword that shrinks a workload to `count` units (None: full size)."""
    if count is None:
        return {}
    if config == "dense_d4096":
        return {"layers": count}
    if config == "moe_64x3":
        return {"experts": count}
    if config == "single_256x512":
        raise SystemExit("single_256x512 has one matrix")
    return {"count": count}


def _small_kwargs(config):
    # the reference arm needs only one matrix of the workload's shape
    if config == "batch64_1024":
        return {"count": 1}
    if config == "dense_d4096":
        return {"layers": 1}
    if config == "moe_64x3":
        return {"experts": 1}
    if config.startswith("sweep_"):
        return {"count": 1}
    return {}


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def run_distributed(args, rank, world, local_rank):
    """Strong scaling over one workload ("Muon 优化器完全拆解…", section
    "分布式工程"): every rank holds the whole workload (the same seeded W and G),
    owns whole matrices balanced by Newton-Schulz FLOPs, steps them with the
    single-GPU plan, and one all-gather hands the updated weights to every
    rank. Timed per step: the owned step and the exchange, each with CUDA
    events; value = the workload's FLOPs / the slowest rank's step time."""
    import datetime

    import torch
    import torch.distributed as dist

    import muon_step_b200 as ms
    import workloads
    from muon_step_b200.distributed import DistributedMuon

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs CUDA GPUs")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    timeout = datetime.timedelta(seconds=120)
    if world > 1:
        dist.init_process_group("nccl", timeout=timeout, device_id=dev)
    else:
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                                world_size=1, timeout=timeout, device_id=dev)
    wl = workloads.make(args.config, device=dev)
    h = wl.hyper
    opt = DistributedMuon([(wl.W[k], wl.G[k], wl.M[k]) for k in range(wl.count)],
                          precision=args.precision)
    hyper = dict(lr=h["lr"], momentum=h["mu"], weight_decay=h["wd"], gamma=h["gamma"],
                 nesterov=h["nesterov"])
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 0)):
        opt.step(**hyper)
    torch.cuda.synchronize()
    assert ms.sync_status() == 0
    clocks = ClockSampler(local_rank, uuid=_nvml_uuid(local_rank))
    clocks.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    clocks.window_begin()
    t0.record(stream)
    for k in range(args.steps):
        ev[k][0].record(stream)
        opt.compute(**hyper)
        ev[k][1].record(stream)
        opt.exchange()
        ev[k][2].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.window_end()
    dist.barrier()
    clk = clocks.stop()
    assert ms.sync_status() == 0
    ms_max = max_over_ranks(t0.elapsed_time(t1), dev, world)
    compute_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps, dev, world)
    exchange_ms = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps, dev, world)
    flops = metric_flops(wl.shapes, len(HYBRID))
    value = flops * args.steps / (ms_max / 1e3) / 1e12
    owned = [len(o) for o in opt.owned]
    launches = len(opt._plan.launches()) if getattr(opt, "_plan", None) is not None else 0
    if world > 1:
        launches += 4  # pack and unpack: a descriptor copy and the copy kernel each
    if rank == 0:
        xbytes = opt.exchange_bytes()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": args.precision, "data": "synthetic",
            "config": {"workload": args.config, "mode": "distributed", "matrices": wl.count,
                       "parallelism": f"owner-partitioned x{world}", "owned_per_rank": owned,
                       "metric_flops_per_step": flops},
            "compute_ms_per_step": compute_ms, "exchange_ms_per_step": exchange_ms,
            "exchange": {"collective": "all_gather (NCCL, in place)", "bytes_in_per_rank": xbytes,
                         "gbs_per_rank": (xbytes / (exchange_ms / 1e3) / 1e9) if exchange_ms > 0 else None},
            "gpu_launches": launches * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    del opt
    dist.barrier()
    dist.destroy_process_group()


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.mode == "distributed":
        return run_distributed(args, rank, world, local_rank)

    import datetime

    import torch
    import torch.distributed as dist

    import muon_step_b200 as ms
    import workloads

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs CUDA GPUs")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    wl = workloads.make(args.config, device=dev, **count_kwargs(args.config, args.count))
    h = wl.hyper
    params = [(wl.W[k], wl.G[k], wl.M[k]) for k in range(wl.count)]
    plan = ms.MuonPlan(params, precision=args.precision, scale_mode=args.scale_mode)
    plan.set_chaining(not args.stagewise, args.chain_window)
    ws = plan.alloc_workspace()
    kinds = plan.launches()
    ns_steps = len(HYBRID)
    stream = torch.cuda.current_stream()

    def step():
        plan.execute(ws, lr=h["lr"], momentum=h["mu"], weight_decay=h["wd"], gamma=h["gamma"],
                     nesterov=h["nesterov"], stream=stream)

    clocks = ClockSampler(local_rank, uuid=_nvml_uuid(local_rank))
    clocks.start()
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    assert ms.sync_status() == 0

    # ---- timed region: device time with events, per-launch events inside.
    # By default the K steps (with their event records) are captured once in
    # a CUDA graph and the timed region replays it.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(kinds))]
          for _ in range(args.steps)]
    for k in range(args.steps):
        for e in ev[k]:
            e.record(stream)  # create the cudaEvent_t handles outside any capture
    torch.cuda.synchronize()
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            graph.capture_begin()
            for k in range(args.steps):
                plan.set_events(ev[k], materialize=False)
                plan.execute(ws, lr=h["lr"], momentum=h["mu"], weight_decay=h["wd"],
                             gamma=h["gamma"], nesterov=h["nesterov"], stream=cap)
            graph.capture_end()
        stream.wait_stream(cap)
        plan.set_events(None)
        torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks.window_begin()
    t_start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for k in range(args.steps):
            plan.set_events(ev[k], materialize=False)
            step()
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.window_end()
    barrier()
    plan.set_events(None)
    clk = clocks.stop()
    ms_total = t_start.elapsed_time(t_end)
    status = ms.sync_status()
    if status != 0:
        raise SystemExit(f"device error status {status}")

    ms_max = max_over_ranks(ms_total, dev, world)
    ms_per_step = ms_max / args.steps
    flops_rank = metric_flops(wl.shapes, ns_steps)
    value = job_tflops(flops_rank, world, args.steps, ms_max)

    # per-kernel durations over the timed region
    per_kind = {}
    for k in range(args.steps):
        for i, kd in enumerate(kinds):
            per_kind.setdefault(kd, []).append(ev[k][2 * i].elapsed_time(ev[k][2 * i + 1]))
    avg = {kd: sum(v) / len(v) for kd, v in per_kind.items()}
    share = {kd: sum(v) for kd, v in per_kind.items()}
    tot_kernel = sum(share.values())

    peaks, peak_src = load_peaks()
    g_fl, p_fl, a_fl = plan.flops()
    tensor_peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    burst_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    roof = dominant_roofline(kinds, per_kind, wl.shapes, peaks, args.precision, ns_steps)
    roof["traffic"] = traffic_from_profile(args.config, roof["kind"])
    roof["peak_source"] = f"{peak_src} ({'sustained bf16' if roof['bound'] == 'tensor' else 'HBM copy'})"
    executed = (g_fl + p_fl + a_fl) / (ms_per_step / 1e3) / 1e12

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        G_dev = [grp[1] for grp in wl.groups.values()]
        W_dev = [grp[0] for grp in wl.groups.values()]
        G_host = [g.cpu().pin_memory() for g in G_dev]
        W_host = [torch.empty(w.shape, dtype=w.dtype, pin_memory=True) for w in W_dev]
        h2d = sum(g.numel() * 4 for g in G_host)
        d2h = sum(w.numel() * 4 for w in W_host)
        # A training loop's transfers overlap the optimizer on their own copy
        # streams, as here. G is needed only by the first kernel of a step and W
        # is rewritten only by the last, so each crosses PCIe through a device
        # staging copy: step k's gradients upload while step k - 1 runs, and
        # step k's weights download while step k + 1 runs. Every step still
        # moves its full inputs in and its result out inside the timed region.
        G_stage = [torch.empty_like(g) for g in G_dev]
        W_stage = [torch.empty_like(w) for w in W_dev]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        e_up, e_taken, e_staged, e_read = ev(), ev(), ev(), ev()

        def e2e_steps(nsteps):
            with torch.cuda.stream(up):
                for gh, gs in zip(G_host, G_stage):
                    gs.copy_(gh, non_blocking=True)
                e_up.record(up)
            e_read.record(down)
            for k in range(nsteps):
                stream.wait_event(e_up)
                for gs, gd in zip(G_stage, G_dev):
                    gd.copy_(gs, non_blocking=True)
                e_taken.record(stream)
                if k + 1 < nsteps:
                    with torch.cuda.stream(up):
                        up.wait_event(e_taken)
                        for gh, gs in zip(G_host, G_stage):
                            gs.copy_(gh, non_blocking=True)
                        e_up.record(up)
                step()
                stream.wait_event(e_read)  # the previous download has read the staging copy
                for wd_, ws_ in zip(W_dev, W_stage):
                    ws_.copy_(wd_, non_blocking=True)
                e_staged.record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(e_staged)
                    for wh, ws_ in zip(W_host, W_stage):
                        wh.copy_(ws_, non_blocking=True)
                    e_read.record(down)
            stream.wait_event(e_read)

        e2e_steps(2)
        torch.cuda.synchronize()
        e_s = torch.cuda.Event(enable_timing=True)
        e_e = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e_s.record(stream)
        e2e_steps(args.steps)
        e_e.record(stream)
        torch.cuda.synchronize()
        barrier()
        te = max_over_ranks(e_s.elapsed_time(e_e), dev, world)
        e2e = {"value": job_tflops(flops_rank, world, args.steps, te),
               "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": te / args.steps,
               "overlap": "copies on their own streams through device staging copies"}
        assert ms.sync_status() == 0

    # ---- AdamW companion group (separate timed region; not part of `value`)
    adamw = None
    if not args.no_adamw:
        adamw = time_adamw_companion(wl, args.steps, dev, stream, peaks, world)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ks = list(range(min(args.cpu_sample, wl.count)))
        mats = [(wl.W[k].double().cpu().numpy(), wl.G[k].double().cpu().numpy(),
                 wl.M[k].double().cpu().numpy()) for k in ks]
        rate, dt, done = cpu_oracle_rate(mats, h, budget_s=20.0)
        cpu = {"value": rate, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
               "sample": f"{done} of {wl.count} matrices of {args.config}, {dt:.1f} s of float64 numpy"}

    if rank == 0:
        names = {0: "elementwise", 1: "gram", 2: "poly", 3: "apply", 4: "apply_update", 5: "small",
                 6: "rms_reduce", 7: "update", 8: "mid", 9: "tiny", 10: "chain"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": args.precision,
            "data": "synthetic",
            "config": {"workload": args.config, "matrices": wl.count,
                       "shapes": sorted({f"{n}x{m}" for n, m in wl.shapes}),
                       "ns_steps": ns_steps, "precision": args.precision,
                       "scale_mode": args.scale_mode,
                       "l2": "inputs larger than L2 (no flush)" if wl.elements() * 12 > 126e6
                             else "inputs smaller than L2",
                       "metric_flops_per_step": flops_rank},
            "pct_of_peak": {"dense_eq_of_burst": value / burst_peak,
                            "executed_of_burst": executed / burst_peak,
                            "executed_of_sustained": executed / tensor_peak},
            "roofline": roof,
            "kernels_ms_avg": {names[k]: v for k, v in sorted(avg.items())},
            "kernels_share": {names[k]: v / tot_kernel for k, v in sorted(share.items())},
            "executed_tflops": executed,
            "gpu_launches": len(kinds) * args.steps,
            "cuda_graph": graph is not None,
            "chained": 10 in kinds,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "companion_adamw": adamw,
        }
        print(json.dumps(line), flush=True)
    del graph
    del plan
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
