#!/usr/bin/env python
"""Benchmark of one Muon optimizer step on B200: every Muon matrix of a parameter set
in one grouped call (momentum, Nesterov input, Frobenius norm, 5 Newton-Schulz
iterations, fused parameter update), timed with CUDA events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--parallel single|sharded|replicas]

Prints one JSON line (rank 0).  Under torchrun the default is the sharded data-parallel
step: each matrix is stepped on one owner rank (gradients averaged onto the owners, the
updated parameters broadcast back), so the whole job's work is fixed as N grows (strong
scaling) and the step time is the maximum over ranks.  `--parallel replicas` instead runs
an independent copy of the whole step on every rank (weak scaling).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from newton_schulz_11_b200 import inputs  # noqa: E402

DEFAULT_WORKLOAD = "gpt2-124m-72-matrices"
WIDE_WORKLOAD = "wide-4096-192-matrices"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# spec-sheet figures of one B200: HBM3e bandwidth and dense (not 2:4 sparse) bf16 tensor peak
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
KINDS = ("momentum", "norm", "gram", "poly", "apply", "apply_last")

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture of
# the benchmarked workload, keyed by kernel kind; valid only while the kernel sources hash to
# `source_hash` (kernel_source_hash: comments and layout do not count; see profiles/).
# Filled in from the committed ncu summary.
NCU_TRAFFIC = {"source_hash": "a482f71f2894de27", "workload": DEFAULT_WORKLOAD,
               "bytes_per_launch": {"gram": 211227904, "poly": 128570112, "apply": 552650496,
                                    "apply_last": 660730624}}
# the same for the AdamW path (workload gpt2-124m-adamw-params, one launch per step)
NCU_TRAFFIC_ADAMW = {"source_hash": "a482f71f2894de27", "bytes_per_launch": 893596672}


def _code_only(text: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace runs collapsed: what the
    compiler sees, so that an edit to a comment does not invalidate measured counters."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":  # string or character literal, copied through with its escapes
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash() -> str:
    """Hash of the kernel sources (newton_schulz_11_b200/csrc), comments and layout aside."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "newton_schulz_11_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ work model

def matrix_work(rows, cols):
    """Per matrix and iteration: algorithmic flops of the Gram (upper half), the
    polynomial (upper half) and the apply, plus the dense-equivalent total."""
    m, n = min(rows, cols), max(rows, cols)
    return {"gram": m * m * n, "poly": m ** 3, "apply": 2 * m * m * n, "dense": 4 * m * m * n + 2 * m ** 3}


def kind_bytes(w, kind, with_out=False):
    """Algorithmic HBM bytes of one launch of `kind` over the whole workload: every input
    the launch needs read once, every output written once (X is a bf16 hi and an 8-bit lo)."""
    pb = 2 if w.param_dtype == "bf16" else 4
    tot = 0
    for rows, cols in w.shapes:
        mn = rows * cols
        m = min(rows, cols)
        if kind == "momentum":
            tot += 15 * mn           # read g, m; write m; write hi (2 B), lo (1 B)
        elif kind == "norm":
            tot += 0
        elif kind == "gram":
            tot += 2 * mn + 2 * m * m    # read hi; write A
        elif kind == "poly":
            tot += 4 * m * m             # read A; write B
        elif kind == "apply":
            tot += 6 * mn + 2 * m * m    # read hi, lo and B; write hi, lo
        elif kind == "apply_last":
            tot += (3 + 2 * pb + (4 if with_out else 0)) * mn + 2 * m * m   # read hi, lo, B; W in/out; O
    return tot


def kind_flops(w, kind):
    if kind not in ("gram", "poly", "apply", "apply_last"):
        return 0
    key = "apply" if kind == "apply_last" else kind
    return sum(matrix_work(r, c)[key] for r, c in w.shapes)


def step_flops(w):
    alg = sum(sum(matrix_work(r, c)[k] for k in ("gram", "poly", "apply")) for r, c in w.shapes) * w.ns_steps
    dense = sum(matrix_work(r, c)["dense"] for r, c in w.shapes) * w.ns_steps
    return alg, dense


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="muon_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def mark(self, begin: bool):
        if begin:
            self.t0 = datetime.datetime.now()
        else:
            self.t1 = datetime.datetime.now()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                except ValueError:
                    continue
                rows.append((ts, parts))
        os.unlink(self.path)
        inside = [p for ts, p in rows if self.t0 and self.t1 and self.t0 <= ts <= self.t1]
        use = inside or [p for _, p in rows]
        sm = [float(p[1]) for p in use if p[1].replace(".", "").isdigit()]
        mx = [float(p[2]) for p in use if p[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in use:
            for name, v in zip(names, p[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(use), "samples_in_timed_region": len(inside)}


class NvmlSampler:
    """SM clock and clock-event reasons sampled in-process by NVML every `period` seconds on a
    thread, so that a timed region of a few tens of milliseconds still holds samples (the
    nvidia-smi loop above cannot sample faster than every few tens of milliseconds)."""

    REASONS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device_index, period=0.002):
        self.period = period
        self.samples = []
        self.t0 = self.t1 = None
        self._stop = threading.Event()
        self._thread = None
        self.handle = None
        self.max_mhz = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(gpu_id_for(device_index))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        except Exception:  # pragma: no cover - depends on the machine
            self.handle = None

    def _loop(self):
        nv, h = self.nv, self.handle
        while not self._stop.is_set():
            t = time.perf_counter()
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                why = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
            except Exception:  # pragma: no cover
                break
            self.samples.append((t, sm, why))
            time.sleep(self.period)

    def start(self):
        if self.handle is not None:
            self._thread = threading.Thread(target=self._loop, daemon=True)
            self._thread.start()

    def mark(self, begin: bool):
        if begin:
            self.t0 = time.perf_counter()
        else:
            self.t1 = time.perf_counter()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        self._stop.set()
        self._thread.join(timeout=5)
        inside = [x for x in self.samples if self.t0 is not None and self.t1 is not None and self.t0 <= x[0] <= self.t1]
        sm = [x[1] for x in inside]
        reasons = sorted({name for _, _, why in inside for name, bit in self.REASONS if why & bit})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples_in_timed_region": len(inside), "period_ms": self.period * 1e3, "source": "nvml"}


class Clocks:
    """Both samplers around one timed region: NVML in-process (the record used, every 2 ms)
    and the nvidia-smi loop of the profiling recipe (kept beside it)."""

    def __init__(self, device_index):
        self.nvml = NvmlSampler(device_index)
        self.smi = ClockSampler(gpu_id_for(device_index))

    def start(self):
        self.smi.start()
        self.nvml.start()

    def mark(self, begin: bool):
        self.nvml.mark(begin)
        self.smi.mark(begin)

    def stop(self):
        rec = self.nvml.stop()
        smi = self.smi.stop()
        if rec.get("samples_in_timed_region", 0) == 0:  # no NVML: fall back on nvidia-smi's record
            rec = dict(smi, source="nvidia-smi")
        rec["nvidia_smi"] = smi
        return rec


def gpu_id_for(device_index):
    import torch

    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid).replace("GPU-", "")
    except Exception:  # pragma: no cover
        return str(device_index)


# ------------------------------------------------------------------ CPU oracle timing

class OracleWorkload:
    """The fp64 oracle on the host cores over a workload's matrices: the same seeded draws
    as the GPU arm's, made on the host once per matrix and cached."""

    def __init__(self, w):
        import numpy as np

        import oracle

        self.np, self.oracle = np, oracle
        self.w = w
        self.coeffs = load_coeffs(w)
        self.step = inputs.first_step_index(w)
        self.cache = {}

    def work(self, i):
        r, c = self.w.shapes[i]
        mw = matrix_work(r, c)
        return (mw["gram"] + mw["poly"] + mw["apply"]) * self.w.ns_steps + 16 * r * c

    def data(self, i):
        if i not in self.cache:
            f64 = self.np.float64
            self.cache[i] = (inputs.weight_np(self.w, i).astype(f64), inputs.grad_np(self.w, self.step, i).astype(f64),
                             inputs.momentum_np(self.w, i).astype(f64))
        return self.cache[i]

    def run(self, idx):
        """Seconds the oracle's step (momentum, Newton-Schulz, update) takes on matrices idx."""
        w = self.w
        data = [self.data(i) for i in idx]
        t0 = time.perf_counter()
        for W, g, m in data:
            self.oracle.muon_step(W, g, m, lr=w.lr, beta=w.beta, weight_decay=w.weight_decay, nesterov=w.nesterov,
                                  coeffs=self.coeffs)
        return time.perf_counter() - t0

    def plan(self, runs, budget_s):
        """Matrices per run so that `runs` runs take about budget_s: the whole workload when it
        fits, else a window of consecutive matrices (taken cyclically), scaled to the whole
        workload by work.  Returns (list of index lists, total work, description)."""
        n = len(self.w.shapes)
        per_shape = {}
        for i, s in enumerate(self.w.shapes):
            if s not in per_shape:
                per_shape[s] = self.run([i]) / max(1, self.work(i))
        est = [per_shape[s] * self.work(i) for i, s in enumerate(self.w.shapes)]
        total = sum(self.work(i) for i in range(n))
        if runs * sum(est) <= budget_s:
            return [list(range(n))] * runs, total, f"the full step: all {n} matrices of {self.w.name}"
        per_run = budget_s / runs
        plans, start = [], 0
        for _ in range(runs):
            idx, t = [], 0.0
            while not idx or (t + est[start % n] <= per_run and len(idx) < n):
                idx.append(start % n)
                t += est[start % n]
                start += 1
            plans.append(idx)
        k = max(len(p) for p in plans)
        return plans, total, (f"per run up to {k} consecutive matrices of {self.w.name} (cyclically), "
                              f"scaled to all {n} by algorithmic work, to keep the run within {budget_s:.0f} s")

    def ms_per_step(self, idx, total):
        return self.run(idx) * 1e3 * total / sum(self.work(i) for i in idx)


def oracle_baseline_ms(w, budget_s=30.0):
    """cpu_baseline of the GPU arm: the oracle on one step of the workload (the whole step
    when it takes at most budget_s), best of two runs when they fit."""
    ow = OracleWorkload(w)
    plans, total, sample = ow.plan(1, budget_s)
    runs = [ow.ms_per_step(plans[0], total)]
    if runs[0] * 2e-3 <= budget_s:
        runs.append(ow.ms_per_step(plans[0], total))
    return min(runs), sample + (f", best of {len(runs)}" if len(runs) > 1 else "")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:  # pragma: no cover
        return os.cpu_count()


def load_coeffs(w):
    from newton_schulz_11_b200 import schedules

    if w.schedule == "polar5":
        return schedules.load("polar5")
    return [(3.4445, -4.7750, 2.0315)] * w.ns_steps


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(args, backend=None):
    """One process per GPU (torchrun env).  NCCL on GPUs; `backend="gloo"` runs the same
    rank logic on CPU processes (tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch
        import torch.distributed as dist

        backend = backend or "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return world, rank, local


def dist_max(x, world):
    """Max of a per-rank number over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ------------------------------------------------------------------ reference arm

def workload_of(args):
    w = inputs.WORKLOADS[args.workload]
    k = getattr(args, "matrices", 0)
    if k and k < len(w.shapes):
        w = inputs.scaled_workload(w, w.shapes[:k], name=f"{w.name}[:{k}]")
    return w


def parallel_mode(args, world):
    mode = getattr(args, "parallel", None)
    if mode in (None, "auto"):
        mode = "sharded" if world > 1 else "single"
    if mode == "single" and world > 1:
        mode = "replicas"
    return mode


def config_of(w, world, mode):
    """The `config` object both arms print for a workload."""
    return {"workload": w.name, "matrices": len(w.shapes), "params": w.n_params, "param_dtype": w.param_dtype,
            "ns_steps": w.ns_steps, "schedule": w.schedule,
            "l2": "inputs larger than L2 (grads+momentum+params ~%.2f GB)" % (w.n_params * 10 / 1e9),
            "parallelism": mode if world > 1 else "single"}


REFERENCE_BUDGET_S = 150.0


def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores: each of the W + K steps runs the oracle's
    step over the workload (all of it when W + K full steps fit in about REFERENCE_BUDGET_S,
    else a window of matrices scaled to the whole step by work); value = median over K."""
    if rank != 0:
        return
    w = workload_of(args)
    ow = OracleWorkload(w)
    plans, total, sample = ow.plan(args.warmup + args.steps, getattr(args, "budget_s", REFERENCE_BUDGET_S))
    for idx in plans[:args.warmup]:
        ow.run(idx)
    runs = [ow.ms_per_step(idx, total) for idx in plans[args.warmup:]]
    value = statistics.median(runs)
    cores = blas_threads()
    mode = parallel_mode(args, world)
    line = {
        "impl": "reference", "metric": "muon_step_ms", "value": round(value, 3), "unit": "ms",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(value, 3),
        "higher_is_better": False, "scaling": "weak" if mode == "replicas" else "strong", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "config": config_of(w, world, mode),
        "cpu_baseline": {"value": round(value, 3), "unit": "ms", "cores": cores, "kind": "oracle",
                         "sample": f"{sample}; median of {args.steps} steps after {args.warmup} warm-up steps"},
        "e2e": {"value": round(value, 3), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def roofline_of(flops, nbytes, ms, peaks, peak_src):
    """Roofline of one kernel from its algorithmic work per launch and its mean launch time.
    The binding bound is the one whose floor time (work / peak) is the longer; `frac` is that
    floor over the measured time.  The tensor denominator is the measured burst bf16 peak,
    fixed whatever the clocks did; the power-capped sustained peak and the spec-sheet figures
    are reported beside it."""
    t = ms * 1e-3
    tf = flops / t / 1e12 if flops else 0.0
    gbs = nbytes / t / 1e9
    f_t = tf / peaks["bf16_tflops"]
    f_h = gbs / peaks["hbm_gbs"]
    tensor = flops > 0 and f_t >= f_h
    return {"bound": "tensor" if tensor else "hbm", "achieved": round(tf if tensor else gbs, 1),
            "peak": peaks["bf16_tflops"] if tensor else peaks["hbm_gbs"], "unit": "TFLOP/s" if tensor else "GB/s",
            "frac": round(max(f_t, f_h), 4),
            "peak_source": f"{peak_src} {'burst bf16 GEMM' if tensor else 'copy bandwidth'}",
            "frac_tensor": round(f_t, 4), "frac_hbm": round(f_h, 4),
            "frac_tensor_of_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
            "frac_nominal": {"tensor": round(tf / NOMINAL_PEAKS["bf16_tflops"], 4),
                             "hbm": round(gbs / NOMINAL_PEAKS["hbm_gbs"], 4)},
            "achieved_tflops": round(tf, 1), "achieved_gbs": round(gbs, 1),
            "algorithmic_flops_per_launch": int(flops), "algorithmic_bytes_per_launch": int(nbytes),
            "ms_per_launch": round(ms, 4)}


def make_step(w, ps, gs, ms, *, mode, world, waves=2, workspace=None, local_step=None):
    """The step the bench times: one PreparedMuonStep over every matrix (single, replicas), or
    the sharded data-parallel step (ShardedMuon: gradients averaged onto each matrix's owner,
    the owners' grouped steps, parameters broadcast back).  Returns (step(), owned indices)."""
    hyper = dict(lr=w.lr, beta=w.beta, weight_decay=w.weight_decay, nesterov=w.nesterov, coeffs=load_coeffs(w))
    if mode == "sharded":
        from newton_schulz_11_b200.distributed import ShardedMuon

        if workspace is not None:
            hyper["workspace"] = workspace
        sh = ShardedMuon(ps, gs, ms, reduce_grads=world > 1, waves=waves, local_step=local_step, **hyper)
        return sh, list(sh.owned)
    from newton_schulz_11_b200 import api

    fn = api.PreparedMuonStep(ps, gs, ms, workspace=workspace, **hyper)
    return (lambda: fn()), list(range(len(ps)))


def time_steps(step, steps, world, device):
    """Milliseconds per step over `steps` steps, bracketed by a barrier and a device
    synchronisation on both sides, timed on the device (CUDA events on the current stream;
    wall clock for CPU ranks); the max over ranks."""
    import torch

    cuda = torch.device(device).type == "cuda"
    barrier(world)
    if cuda:
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            step()
        e1.record()
        torch.cuda.synchronize(device)
        ms = e0.elapsed_time(e1) / steps
    else:
        t0 = time.perf_counter()
        for _ in range(steps):
            step()
        ms = (time.perf_counter() - t0) * 1e3 / steps
    barrier(world)
    return dist_max(ms, world)


def base_line(w, world, mode, ms_step, args):
    """The contract's keys of our arm's JSON line."""
    return {"metric": "muon_step_ms", "value": round(ms_step, 4), "unit": "ms", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": False,
            "scaling": "weak" if mode == "replicas" else "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_of(w, world, mode)}


def flat_workload(w, dev, step):
    """The workload's grads, momentum and params in three flat device buffers, one 2-D view
    per matrix (so that the host copies of e2e are one copy each)."""
    import torch

    sizes = [r * c for r, c in w.shapes]
    offs = [0]
    for n in sizes:
        offs.append(offs[-1] + n)
    pdt = torch.bfloat16 if w.param_dtype == "bf16" else torch.float32
    G = torch.empty(offs[-1], dtype=torch.float32, device=dev)
    M = torch.empty(offs[-1], dtype=torch.float32, device=dev)
    P = torch.empty(offs[-1], dtype=pdt, device=dev)
    views = lambda flat: [flat[offs[i]: offs[i + 1]].view(*w.shapes[i]) for i in range(len(sizes))]  # noqa: E731
    gs, ms, ps = views(G), views(M), views(P)
    with torch.no_grad():
        for i in range(len(sizes)):
            gs[i].copy_(inputs.grad_torch(w, step, i, dev))
            ms[i].copy_(inputs.momentum_torch(w, i, dev))
            ps[i].copy_(inputs.weight_torch(w, i, dev))
    torch.cuda.synchronize(dev)
    return (G, M, P), (gs, ms, ps), views


def measure_wide(local, peaks, peak_src, steps=5, warmup=3):
    """The 4096-wide set (192 matrices, 5.9B parameters) on this GPU, inputs drawn on the
    device: step time, Newton-Schulz TFLOP/s and its fractions, with the clocks of its own
    timed region."""
    import torch

    from newton_schulz_11_b200 import api

    dev = torch.device("cuda", local)
    w = inputs.WORKLOADS[WIDE_WORKLOAD]
    free, _ = torch.cuda.mem_get_info(dev)
    need = w.n_params * 10 + api.workspace_size(w.shapes)
    if free < need * 1.1:
        return {"skipped": f"needs {need / 1e9:.0f} GB, {free / 1e9:.0f} GB free"}
    _, (gs, ms, ps), _ = flat_workload(w, dev, inputs.first_step_index(w))
    ws = api.Workspace(dev)
    step, _ = make_step(w, ps, gs, ms, mode="single", world=1, workspace=ws)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = Clocks(local)
    clocks.start()
    clocks.mark(True)
    ms_step = time_steps(step, steps, 1, dev)
    clocks.mark(False)
    clk = clocks.stop()
    code, where = api.device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} at {where} in the 4096-wide run")
    alg, dense = step_flops(w)
    tf = alg / (ms_step * 1e-3) / 1e12
    out = {"workload": w.name, "matrices": len(w.shapes), "params": w.n_params, "ms_per_step": round(ms_step, 2),
           "steps": steps, "warmup": warmup, "ns_tflops": round(tf, 1),
           "ns_tflops_dense_equiv": round(dense / (ms_step * 1e-3) / 1e12, 1),
           "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
           "frac_of_bf16_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
           "frac_of_nominal_bf16": round(tf / NOMINAL_PEAKS["bf16_tflops"], 4),
           "peak_source": peak_src, "clocks": clk,
           "note": "whole step (elementwise pass included) timed; NS flops over the step time"}
    del gs, ms, ps, step, ws
    torch.cuda.empty_cache()
    return out


def torch_comparator_step(w, grads, moms, params, coeffs):
    """The same step in plain PyTorch, the way the pages' listing runs it: for each shape
    class, the matrices stacked and every Newton-Schulz product a batched bf16 matmul
    (torch.bmm, cuBLAS), with X kept in bf16 between iterations; momentum, Nesterov input
    and update as torch elementwise ops.  A library comparator for timing on the same GPU:
    it is neither the product path nor the parity reference (the oracle is).  Returns
    step() and the stacked (g, m, W) per class (W updated in place)."""
    import torch

    groups = {}
    for i, shp in enumerate(w.shapes):
        groups.setdefault(tuple(shp), []).append(i)
    cls = []
    for (r, c), idx in groups.items():
        cls.append((torch.stack([grads[i] for i in idx]), torch.stack([moms[i] for i in idx]),
                    torch.stack([params[i] for i in idx]), r > c, math.sqrt(max(1.0, r / c))))

    def step():
        for g, m, p, tall, scale in cls:
            m.mul_(w.beta).add_(g)
            u = g.add(m, alpha=w.beta) if w.nesterov else m
            X = u.bfloat16()
            X = X / (torch.linalg.vector_norm(X, dim=(1, 2), keepdim=True) + 1e-7)
            if tall:
                X = X.mT
            for a, b, c in coeffs:
                A = X @ X.mT
                B = b * A + c * (A @ A)
                X = a * X + B @ X
            if tall:
                X = X.mT
            p.mul_(1.0 - w.lr * w.weight_decay).add_(X.to(p.dtype), alpha=-w.lr * scale)

    return step, cls


def measure_torch_comparator(w, local, ms_ours, steps=20, warmup=5):
    """Times torch_comparator_step on this GPU on the workload's own inputs."""
    import torch

    dev = torch.device("cuda", local)
    step0 = inputs.first_step_index(w)
    n = len(w.shapes)
    step, _ = torch_comparator_step(w, [inputs.grad_torch(w, step0, i, dev) for i in range(n)],
                                    [inputs.momentum_torch(w, i, dev) for i in range(n)],
                                    [inputs.weight_torch(w, i, dev) for i in range(n)], load_coeffs(w))
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    ms_t = time_steps(step, steps, 1, dev)
    alg, _ = step_flops(w)
    del step
    torch.cuda.empty_cache()
    return {"impl": "plain PyTorch: bf16 torch.bmm per shape class (cuBLAS), X kept in bf16",
            "ms_per_step": round(ms_t, 4), "steps": steps, "warmup": warmup,
            "ns_tflops": round(alg / (ms_t * 1e-3) / 1e12, 1), "time_ratio_to_ours": round(ms_t / ms_ours, 2),
            "note": "a library comparator on the same GPU and inputs; lower precision than this "
                    "library's path (X rounded to bf16 every iteration) and not parity-checked"}


def run_ours(args, world, rank, local):
    import ctypes

    import torch

    from newton_schulz_11_b200 import _lib, api, build

    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = workload_of(args)
    mode = parallel_mode(args, world)
    step0 = inputs.first_step_index(w)
    (G, M, P), (gs, ms, ps), views = flat_workload(w, dev, step0)
    ws = api.Workspace(dev)
    stream = torch.cuda.current_stream(dev)
    step, owned = make_step(w, ps, gs, ms, mode=mode, world=world, waves=args.waves, workspace=ws)
    # the kernels of this rank run on its own matrices (all of them unless sharded)
    w_local = w if len(owned) == len(w.shapes) else inputs.scaled_workload(
        w, [w.shapes[i] for i in owned], name=f"{w.name}[owned by rank {rank}]")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    L = _lib.lib()
    clocks = Clocks(local)
    clocks.start()
    # ---- timed region: K steps, inputs resident in HBM (larger than L2).  No per-kernel
    # events here: an event between two launches would stop their programmatic overlap.
    clocks.mark(True)
    ms_step = time_steps(step, args.steps, world, dev)
    clocks.mark(False)
    clk = clocks.stop()

    # ---- step-time spread: events between steps only (launches inside a step keep their
    # programmatic overlap); p10 / p50 / p90 over up to 200 steps
    spread_steps = max(1, min(args.steps, 200))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(spread_steps + 1)]
    torch.cuda.synchronize()
    evs[0].record(stream)
    for i in range(spread_steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    per_step = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(spread_steps))
    pct = lambda f: per_step[min(len(per_step) - 1, int(f * len(per_step)))]  # noqa: E731
    spread = {"p10": round(pct(0.10), 4), "p50": round(pct(0.50), 4), "p90": round(pct(0.90), 4),
              "steps": spread_steps}

    # ---- per-kernel breakdown: a second pass with an event pair around every launch
    prof_steps = max(1, min(args.steps, 50))
    torch.cuda.synchronize()
    _lib.check(L.muon_profile_begin(), "muon_profile_begin")
    for _ in range(prof_steps):
        step()
    torch.cuda.synchronize()
    kms = (ctypes.c_double * 6)()
    kcount = (ctypes.c_int64 * 6)()
    _lib.check(L.muon_profile_end(kms, kcount, 6), "muon_profile_end")
    launches_per_step = sum(kcount) // prof_steps

    # ---- end to end through host buffers: every step copies its grads in from pinned host
    # memory and its params out to pinned host memory.
    e2e_ms = None
    if not args.no_e2e:
        e2e_ms = run_e2e(w, mode, world, step, (G, M, P), (gs, ms, ps), views, ws, stream, args)

    code, where = api.device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} at wait site {where}")

    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    per_kind = {k: {"ms_total": kms[i], "launches": int(kcount[i])} for i, k in enumerate(KINDS)}
    dom = max(KINDS, key=lambda k: per_kind[k]["ms_total"])
    # The dominant kernel's work over all its launches in the profiled pass, divided by
    # their summed time (a workload of several waves has several launches per iteration).
    iters = {"momentum": 1, "norm": 1, "gram": w.ns_steps, "poly": w.ns_steps, "apply": w.ns_steps - 1,
             "apply_last": 1}

    def per_launch(kind):
        n = max(1, per_kind[kind]["launches"])
        return (kind_flops(w_local, kind) * iters[kind] * prof_steps / n,
                kind_bytes(w_local, kind) * iters[kind] * prof_steps / n, per_kind[kind]["ms_total"] / n)

    fl, by, dom_ms = per_launch(dom)
    roof = roofline_of(fl, by, dom_ms, peaks, peak_src)
    traffic = None
    if NCU_TRAFFIC["source_hash"] == kernel_source_hash() and NCU_TRAFFIC["workload"] == w_local.name:
        traffic = NCU_TRAFFIC["bytes_per_launch"].get(dom)
    roof = {**{k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac")}, "traffic": traffic,
            "kernel": dom, **{k: v for k, v in roof.items() if k not in ("bound", "achieved", "peak", "unit", "frac")}}
    _, ew_by, ew_ms = per_launch("momentum")
    ew = roofline_of(0, ew_by, ew_ms, peaks, peak_src)

    alg, dense = step_flops(w)
    jobs = world if mode == "replicas" else 1  # whole-job work per step
    tf = jobs * alg / (ms_step * 1e-3) / 1e12
    line = base_line(w, world, mode, ms_step, args)
    line.update({
        "ns_tflops": round(tf, 1),
        "ns_tflops_dense_equiv": round(jobs * dense / (ms_step * 1e-3) / 1e12, 1),
        # per GPU: the whole job's Newton-Schulz flops over the step time, over N GPUs' peaks
        "ns_frac_of_bf16_peak": round(tf / world / peaks["bf16_tflops"], 4),
        "ns_frac_of_bf16_sustained": round(tf / world / peaks["bf16_tflops_sustained"], 4),
        "ns_frac_of_nominal_bf16": round(tf / world / NOMINAL_PEAKS["bf16_tflops"], 4),
        "kernels": {k: {"ms_per_launch": round(v["ms_total"] / max(1, v["launches"]), 4),
                        "launches": v["launches"], "share": round(v["ms_total"] / max(1e-9, sum(
                            x["ms_total"] for x in per_kind.values())), 4)} for k, v in per_kind.items()},
        "roofline": roof,
        "elementwise": {"kernel": "muon_momentum_kernel", "achieved_gbs": ew["achieved_gbs"],
                        "frac_of_measured_hbm": ew["frac_hbm"], "frac_of_nominal_hbm": ew["frac_nominal"]["hbm"],
                        "algorithmic_bytes_per_launch": ew["algorithmic_bytes_per_launch"],
                        "ms_per_launch": ew["ms_per_launch"]},
        "clocks": clk,
        "e2e": None if e2e_ms is None else {
            "value": round(e2e_ms, 4), "unit": "ms", "h2d_bytes_per_step": G.numel() * 4,
            "d2h_bytes_per_step": P.numel() * P.element_size()},
        "gpu_launches": int(launches_per_step * args.steps),
        "profiled_steps": prof_steps,
        "ms_per_step_spread": spread,
        "peaks": {"source": peak_src, **peaks, "nominal": NOMINAL_PEAKS},
    })
    if mode == "sharded" and world > 1:
        line["sharding"] = {"owned_by_rank0": len(owned), "waves": args.waves,
                            "collectives": "NCCL reduce of fp32 grads onto owners, broadcast of bf16 params"}
    if world == 1 and not args.no_cpu_baseline:
        cms, sample = oracle_baseline_ms(w)
        line["cpu_baseline"] = {"value": round(cms, 1), "unit": "ms", "cores": blas_threads(), "kind": "oracle",
                                "sample": sample}
    if world == 1 and mode == "single" and not args.no_torch:
        line["torch_comparator"] = measure_torch_comparator(w, local, ms_step)
    if world == 1 and w.name == DEFAULT_WORKLOAD and not args.no_wide:
        del G, M, P, gs, ms, ps, step, ws
        torch.cuda.empty_cache()
        line["wide4096"] = measure_wide(local, peaks, peak_src)
    print(json.dumps(line), flush=True)


def run_e2e(w, mode, world, step, flats, views_, view_of, ws, stream, args):
    """Milliseconds per step through host buffers (max over ranks).  Single GPU: pipelined
    over two copy streams -- step t + 1's grads come in (into the other of two grad
    buffers) and step t's params go out (from a device snapshot taken right after the step)
    while step t + 1 runs.  Sharded: every step copies its grads in, steps, and copies the
    params out, in stream order."""
    import torch

    from newton_schulz_11_b200 import api

    G, M, P = flats
    gs, ms, ps = views_
    dev = G.device
    pin_g = torch.empty_like(G, device="cpu").pin_memory()
    pin_g.copy_(G.cpu())
    e2e_steps = max(2, min(args.steps, 50))
    if mode == "sharded":
        pin_p = torch.empty_like(P, device="cpu").pin_memory()

        def one():
            G.copy_(pin_g, non_blocking=True)
            step()
            pin_p.copy_(P, non_blocking=True)

        one()
        torch.cuda.synchronize()
        return time_steps(one, e2e_steps, world, dev)

    G2 = torch.empty_like(G)
    coeffs = load_coeffs(w)
    step2 = api.PreparedMuonStep(ps, view_of(G2), ms, lr=w.lr, beta=w.beta, weight_decay=w.weight_decay,
                                 nesterov=w.nesterov, coeffs=coeffs, workspace=ws)
    gbuf, steps_fn = (G, G2), (step, lambda: step2())
    snap = (torch.empty_like(P), torch.empty_like(P))
    pin_p = (torch.empty_like(P, device="cpu").pin_memory(), torch.empty_like(P, device="cpu").pin_memory())
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731

    def run(n):
        in_done, step_done, out_done = [None, None], [None, None], [None, None]
        for t in range(n):
            b = t % 2
            if step_done[b] is not None:
                s_in.wait_event(step_done[b])      # the step that read this grad buffer is done
            with torch.cuda.stream(s_in):
                gbuf[b].copy_(pin_g, non_blocking=True)
            in_done[b] = ev()
            in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            steps_fn[b]()
            if out_done[b] is not None:
                stream.wait_event(out_done[b])     # the snapshot's previous copy-out is done
            snap[b].copy_(P, non_blocking=True)
            step_done[b] = ev()
            step_done[b].record(stream)
            s_out.wait_event(step_done[b])
            with torch.cuda.stream(s_out):
                pin_p[b].copy_(snap[b], non_blocking=True)
            out_done[b] = ev()
            out_done[b].record(s_out)
        for e in out_done:
            if e is not None:
                stream.wait_event(e)

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    s_in.wait_event(f0)
    s_out.wait_event(f0)
    run(e2e_steps)
    f1.record(stream)
    torch.cuda.synchronize()
    out = dist_max(f0.elapsed_time(f1) / e2e_steps, world)
    barrier(world)
    return out


# ------------------------------------------------------------------ AdamW path

ADAMW_HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)
ADAMW_BYTES_PER_ELEM = 24  # bf16 p read + written, fp32 g read, fp32 m and v read + written


def adamw_layout():
    """(name, numel, offset) of each tensor in flat buffers; offsets are multiples of 8
    elements, so every view keeps 16-byte alignment (the vector path)."""
    out, off = [], 0
    for name, n in inputs.gpt2_124m_adamw_tensors():
        out.append((name, n, off))
        off += (n + 7) // 8 * 8
    return out, off


def adamw_oracle_sample_ms(step=2):
    """The fp64 oracle's AdamW step on a bounded sample (the first 2^21 elements of the token
    embedding), scaled to the whole parameter set by element count."""
    import numpy as np

    from oracle import adamw_oracle as ao

    layout, _ = adamw_layout()
    total = sum(n for _, n, _ in layout)
    k = 1 << 21
    rng = np.random.default_rng(0)
    p = 0.02 * rng.standard_normal(k)
    g = 1e-3 * rng.standard_normal(k)
    m = 0.1 * g
    v = 0.05 * g * g
    t0 = time.perf_counter()
    ao.adamw_step(p, g, m, v, step=step, **{"lr": ADAMW_HYPER["lr"], "beta1": ADAMW_HYPER["beta1"],
                                           "beta2": ADAMW_HYPER["beta2"], "eps": ADAMW_HYPER["eps"],
                                           "weight_decay": ADAMW_HYPER["weight_decay"]})
    dt = time.perf_counter() - t0
    sample = (f"the fp64 oracle's AdamW step on the first {k} elements of the token embedding, "
              f"scaled to all {total} elements")
    return dt * 1e3 * total / k, sample


def run_adamw(args, world, rank, local):
    import torch

    from newton_schulz_11_b200 import api, build

    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    layout, flat = adamw_layout()
    P = torch.empty(flat, dtype=torch.bfloat16, device=dev)
    G = torch.zeros(flat, dtype=torch.float32, device=dev)
    M = torch.zeros(flat, dtype=torch.float32, device=dev)
    V = torch.zeros(flat, dtype=torch.float32, device=dev)
    ps = [P[o:o + n] for _, n, o in layout]
    gs = [G[o:o + n] for _, n, o in layout]
    ms = [M[o:o + n] for _, n, o in layout]
    vs = [V[o:o + n] for _, n, o in layout]
    with torch.no_grad():
        for i, (_, n, o) in enumerate(layout):
            ps[i].copy_(inputs.adamw_param_torch(i, n, dev))
            gs[i].copy_(inputs.adamw_grad_torch(1, i, n, dev))
    numel = sum(n for _, n, _ in layout)
    stream = torch.cuda.current_stream(dev)
    adamw = api.PreparedAdamW(ps, gs, ms, vs, lr=ADAMW_HYPER["lr"], betas=(ADAMW_HYPER["beta1"], ADAMW_HYPER["beta2"]),
                              eps=ADAMW_HYPER["eps"], weight_decay=ADAMW_HYPER["weight_decay"])
    t = 0
    for _ in range(args.warmup):
        t += 1
        adamw(t, stream)
    torch.cuda.synchronize()
    clocks = Clocks(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark(True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        t += 1
        adamw(t, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    barrier(world)
    ms_step = dist_max(e0.elapsed_time(e1) / args.steps, world)
    clk = clocks.stop()
    e2e = None
    if not args.no_e2e:
        pin_g = G.cpu().pin_memory()
        pin_p = torch.empty_like(P, device="cpu").pin_memory()
        e2e_steps = max(1, min(args.steps, 50))
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        barrier(world)
        f0.record(stream)
        for _ in range(e2e_steps):
            t += 1
            G.copy_(pin_g, non_blocking=True)
            adamw(t, stream)
            pin_p.copy_(P, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize()
        e2e = {"value": round(dist_max(f0.elapsed_time(f1) / e2e_steps, world), 4), "unit": "ms",
               "h2d_bytes_per_step": G.numel() * 4, "d2h_bytes_per_step": P.numel() * 2}
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    launches = (len(layout) + 127) // 128
    by = ADAMW_BYTES_PER_ELEM * numel / launches
    gbs = by / (ms_step / launches * 1e-3) / 1e9
    line = {
        "metric": "adamw_step_ms", "value": round(ms_step, 4), "unit": "ms", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": inputs.ADAMW_WORKLOAD, "tensors": len(layout), "params": numel, "param_dtype": "bf16",
                   "l2": "inputs larger than L2 (%.2f GB moved per step)" % (ADAMW_BYTES_PER_ELEM * numel / 1e9),
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "traffic": NCU_TRAFFIC_ADAMW["bytes_per_launch"]
                     if NCU_TRAFFIC_ADAMW["source_hash"] == kernel_source_hash() else None,
                     "kernel": "muon_adamw_kernel",
                     "peak_source": peak_src + " copy", "algorithmic_bytes_per_launch": int(by)},
        "clocks": clk, "e2e": e2e, "gpu_launches": launches * args.steps,
    }
    if world == 1 and not args.no_cpu_baseline:
        cms, sample = adamw_oracle_sample_ms()
        line["cpu_baseline"] = {"value": round(cms, 1), "unit": "ms", "cores": blas_threads(), "kind": "oracle",
                                "sample": sample}
    print(json.dumps(line), flush=True)


def run_adamw_reference(args, world, rank):
    if rank != 0:
        return
    for _ in range(args.warmup):
        adamw_oracle_sample_ms()
    runs = [adamw_oracle_sample_ms() for _ in range(args.steps)]
    value = statistics.median(r[0] for r in runs)
    layout, _ = adamw_layout()
    line = {
        "impl": "reference", "metric": "adamw_step_ms", "value": round(value, 3), "unit": "ms", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(value, 3), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": inputs.ADAMW_WORKLOAD, "tensors": len(layout), "params": sum(n for _, n, _ in layout)},
        "cpu_baseline": {"value": round(value, 3), "unit": "ms", "cores": blas_threads(), "kind": "oracle",
                         "sample": runs[0][1]},
        "e2e": {"value": round(value, 3), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=inputs.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer pass (for workloads whose inputs do not fit pinned host memory)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", default="muon", choices=["muon", "adamw"],
                    help="muon: the Muon step (default); adamw: the AdamW step of the non-matrix parameters")
    ap.add_argument("--matrices", type=int, default=0,
                    help="run only the first K matrices of the workload (a small case of the same kernels)")
    ap.add_argument("--parallel", default="auto", choices=["auto", "single", "sharded", "replicas"],
                    help="N > 1: sharded data-parallel step (default) or independent replicas")
    ap.add_argument("--waves", type=int, default=2,
                    help="sharded: waves of owned matrices (a wave's broadcasts overlap the next wave's step)")
    ap.add_argument("--no-wide", action="store_true",
                    help="skip the 4096-wide measurement added to the default workload's line")
    ap.add_argument("--no-torch", action="store_true",
                    help="skip the plain-PyTorch (cuBLAS bf16 bmm) comparator timed beside the step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        (run_adamw_reference if args.path == "adamw" else run_reference)(args, world, rank)
        return
    world, rank, local = dist_setup(args)
    try:
        (run_adamw if args.path == "adamw" else run_ours)(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
