"""Benchmark: Kronecker-layer rows/s, forward + backward, on the tutorial layer
(N = 20000 rows, 1024 x 1024, m = 32 (p = q = 32), r = 4, fp32 I/O, half of S zeroed),
with the achieved fraction of the dominant kernel's roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--path tf32|f32|bf16]
    python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores

One step = forward (y = x W + bias) and backward (dX, dS, dA, dB, dbias) of one batch
through the C ABI.  With N > 1 GPUs (torchrun, NCCL) every rank runs the full batch
on its own GPU (weak scaling) and the factor gradients are summed across ranks with
one NCCL all-reduce per step, the data-parallel exchange.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Kron-layer rows/s fwd+bwd (1024², m=32, r=4) & achieved % of roofline"
UNIT = "rows/s"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the backward
# call's kernels (dX + parameter gradients) on the tutorial layer, from one ncu capture of
# this command (the step after the warm-up), valid only for the kernel sources whose
# SHA-256 prefix is recorded with it: any later change to them makes the figure null.  The
# write counters miss the part of dX still in L2 when the kernel ends.
_TRAFFIC = {
    "tf32": (81.99e6 + 27.75e6 + 163.99e6 + 0.19e6, "9e6816695f191714"),
    "bf16": (41.01e6 + 0.20e6 + 82.00e6 + 0.36e6, "9e6816695f191714"),
}


def _tc_sources_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "kronecker_factored_structured_b200", "csrc")
    for f in ("tc_fwd.cu", "tc_bwd.cu", "tc_ptx.cuh"):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic(path: str, workload: str):
    rec = _TRAFFIC.get(path)
    if rec is None or workload != "tutorial" or rec[1] != _tc_sources_sha():
        return None
    return rec[0]
WORKLOAD = "tutorial"
ROTATE = 3  # independent input sets cycled through, so the working set exceeds L2


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0, "source": "fallback"}


def _workload_desc(w):
    zero = f", {w.s_zero_entries} of {w.p * w.q} entries of S zeroed" if w.s_zero_entries else ""
    return (f"{w.name}: N={w.N} rows, {w.d_in}x{w.d_out} layer, p={w.p} q={w.q} "
            f"m1={w.m1} m2={w.m2}, r={w.r}, {w.dtype} I/O{zero}")


class _NvmlRegion:
    """SM clock and clock-event reasons read through NVML every `period` seconds by a
    background thread while the timed region runs (nvidia-smi's -lms sampling is too coarse
    for a region of tens of milliseconds).  Reads only; any NVML failure leaves it empty."""
    NAMES = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
             ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
             ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
             ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device: int, period: float = 0.002):
        self.samples, self.period, self.error = [], period, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device)
            self._nv = pynvml
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            except pynvml.NVMLError:
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(
                    f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0")
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # no NVML on this host: the nvidia-smi samples remain
            self._nv, self.error = None, f"{type(e).__name__}: {e}"

    def _run(self):
        nv, h = self._nv, self._h
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            self._stop.wait(self.period)

    def start(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._nv is not None:
            try:
                self._nv.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return None
        reasons = set()
        for _, bits in self.samples:
            for name, attr in self.NAMES:
                if bits & getattr(self._nv, attr):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz for mhz, _ in self.samples),
                "sm_max_mhz": float(self.max_mhz), "reasons": sorted(reasons),
                "samples": len(self.samples),
                "sampler": f"NVML every {self.period * 1e3:.0f} ms inside the timed region"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms around the timed region,
    and NVML every 2 ms inside it (begin_region / end_region); the NVML samples are the
    record when there are any."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def begin_region(self):
        self.nvml = _NvmlRegion(torch_current_device())
        # the launching thread holds the interpreter lock between library calls; a short
        # switch interval lets the sampler thread take its 2 ms samples on time
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(0.0002)
        self.nvml.start()

    def end_region(self):
        if getattr(self, "nvml", None) is not None:
            self.nvml.stop()
        if getattr(self, "_switch", None) is not None:
            sys.setswitchinterval(self._switch)

    def wait_started(self, timeout=5.0):
        """Block until nvidia-smi has printed its first sample (it takes ~0.5 s to start)."""
        import select
        if self.proc is None:
            return
        r, _, _ = select.select([self.proc.stdout], [], [], timeout)
        if r:
            self.first = self.proc.stdout.readline()

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in (getattr(self, "first", "") + out).splitlines() if ln.strip()]

    def summary(self):
        fine = self.nvml.summary() if getattr(self, "nvml", None) is not None else None
        if fine is not None:
            fine["nvidia_smi_samples"] = len(getattr(self, "lines", []) or [])
            return fine
        if not getattr(self, "lines", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def torch_current_device() -> int:
    import torch
    return torch.cuda.current_device()


def cpu_baseline(w, rows: int, threads: int | None = None):
    """Time the fp64 oracle (forward + backward) on the first `rows` rows."""
    import numpy as np

    import kron_workloads as kw
    import oracle
    if threads:
        oracle.set_threads(threads)
    f = {k: v.float().numpy().astype(np.float64) for k, v in kw.factors(w).items()}
    x = kw.rows(w, "x", 0, rows).float().numpy().astype(np.float64)
    G = kw.rows(w, "G", 0, rows).float().numpy().astype(np.float64)
    t0 = time.perf_counter()
    oracle.forward(x, f["S"], f["A"], f["B"], f["bias"])
    oracle.backward(x, f["S"], f["A"], f["B"], G)
    dt = time.perf_counter() - t0
    return rows / dt, dt, oracle.get_threads()


def run_reference(args, w):
    """--impl reference: the fp64 oracle on the host cores, a bounded row sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rows = args.ref_rows
    for _ in range(args.warmup):
        cpu_baseline(w, rows)
    t0 = time.perf_counter()
    threads = 1
    for _ in range(args.steps):
        _, _, threads = cpu_baseline(w, rows)
    dt = time.perf_counter() - t0
    value = rows * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": _workload_desc(w), "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"first {rows} of {w.N} rows per step, forward + backward"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def dense_context(fac, sets, path, steps, dev, graph=False):
    """Context only (not the product path): the same layer as a dense x @ W + bias with W
    materialised (sum_i kron(S*A_i, B_i)), forward and backward (dX = dY W^T, dW = x^T dY,
    dbias) as three cuBLAS GEMMs through torch, timed like the Kronecker step (CUDA events
    around `steps` back-to-back steps over the same rotated inputs).  TF32 tensor cores are
    allowed for the tf32 path and disallowed for f32."""
    import torch
    t = torch.bfloat16 if path == "bf16" else torch.float32
    C = (fac["S"].float()[None] * fac["A"].float())
    W = sum(torch.kron(C[i], fac["B"].float()[i]) for i in range(C.shape[0])).to(t)
    bias = fac["bias"].to(t)
    old = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = path == "tf32"
    try:
        def step(i):
            x, G = sets[i % len(sets)]
            y = torch.addmm(bias, x, W)
            dx = G @ W.t()
            dw = x.t() @ G
            db = G.sum(0)
            return y, dx, dw, db
        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        if graph:
            ms = _time_graph(step, steps, REPEATS)[0] / steps
        else:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for i in range(steps):
                step(i)
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / steps
    finally:
        torch.backends.cuda.matmul.allow_tf32 = old
    return {"what": "dense x @ W + bias forward and backward (dX, dW, dbias) with W "
                    "materialised, torch/cuBLAS, same inputs and timer; context only",
            "matmul": "tf32" if path == "tf32" else path, "ms_per_step": ms,
            "timer": "CUDA graph replay" if graph else "eager steps between CUDA events"}


REPEATS = 5  # repeats of each timed region; the median is reported (and the min)


def _path_supported(kfs, w, path):
    """True when the library has kernels for this workload on this path (the backward's
    workspace size is 0 exactly when no kernel of the path takes the shape)."""
    return kfs.workspace_size(max(w.N, 1), w.p, w.q, w.m1, w.m2, w.r, path) > 0


def _step_roofline(w, path, ms_step, peaks, flags):
    """Roofline time of one forward + backward step, max(bytes / HBM, flops / unit peak), and
    the achieved fraction of it.  The unit peak is the measured BF16 tensor rate for BF16, half
    of it for TF32 (the nominal TF32:BF16 ratio) and the derived FFMA rate for FP32."""
    from kronecker_factored_structured_b200 import accounting as acc
    elt = 2 if path == "bf16" else 4
    nbytes = w.N * acc.bytes_per_row(w.d_in, w.d_out, elt)
    skip = None
    if flags and w.s_zero_patches:
        skip = 1.0 - w.s_zero_patches / float((w.p // w.s_zero_patch) * (w.q // w.s_zero_patch))
    flops = w.N * acc.flops_per_row(w.p, w.q, w.m1, w.m2, w.r, skip_fraction=skip)
    if path == "f32":
        peak, unit, src = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6, "FFMA", "derived"
    else:
        bf = peaks["bf16_tflops"] * 1e12
        peak, unit, src = (bf, "bf16", peaks["source"]) if path == "bf16" else \
            (bf / 2, "tf32", peaks["source"] + " bf16 x 1/2")
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_fl = flops / peak
    t_roof = max(t_hbm, t_fl)
    return {"bound": "hbm" if t_hbm >= t_fl else ("alu" if path == "f32" else "tensor"),
            "roofline_us": t_roof * 1e6, "hbm_us": t_hbm * 1e6, "flops_us": t_fl * 1e6,
            "frac": t_roof / (ms_step / 1e3), "flop_peak": unit, "flop_peak_source": src,
            "bytes": nbytes, "flops": flops}


class _Problem:
    """Device tensors of one workload on one path: ROTATE (or fewer) independent (x, dY)
    input sets resident in HBM, the factors, outputs and workspace."""

    def __init__(self, kw, kfs, w, path, dev, rank=0, rotate=ROTATE):
        import torch
        self.w, self.path = w, path
        t_io = kfs.native.io_dtype(path)
        self.fac = {k: v.to(dev).to(t_io) for k, v in kw.factors(w).items()}
        self.sets = []
        for s in range(rotate):
            ws = dataclasses.replace(w, seed=w.seed + 1000 * s + 100000 * rank) if (s or rank) else w
            self.sets.append((kw.rows(ws, "x").to(dev).to(t_io), kw.rows(ws, "G").to(dev).to(t_io)))
        self.y = torch.empty(w.N, w.d_out, dtype=t_io, device=dev)
        self.wsb = torch.empty(max(kfs.workspace_size(w.N, w.p, w.q, w.m1, w.m2, w.r, path), 1),
                               dtype=torch.uint8, device=dev)


def _time_region(step, steps, repeats, world, dist, stream, clk=None):
    """Device time (ms) of `steps` back-to-back steps, measured `repeats` times between CUDA
    events on the launching stream, each repeat bracketed by a barrier and a synchronize;
    the max over ranks of each repeat.  Returns (median, min, all)."""
    import torch
    times = []
    for rep in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        if clk is not None and rep == 0:
            clk.begin_region()
        a.record(stream)
        for i in range(steps):
            step(i)
        b.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms = a.elapsed_time(b)
        if world > 1:
            t = torch.tensor([ms], device="cuda", dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        times.append(ms)
    if clk is not None:
        clk.end_region()
    return statistics.median(times), min(times), times


def _time_graph(step, steps, repeats):
    """Device time (ms) of `steps` steps captured once in a CUDA graph and replayed
    `repeats` times between CUDA events (launch overhead excluded: the per-call host work
    of the Python binding exceeds the device time of the small layers).  Returns (median,
    min, all)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        step(0)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=side):
            for i in range(steps):
                step(i)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    del g
    return statistics.median(times), min(times), times


def _split_calls(step, steps, stream):
    """Mean forward and backward call times (ms) from per-call events over `steps` steps
    (outside any timed region: the extra event records do not enter a reported value)."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True)
    marks = [(ev(), ev(), ev()) for _ in range(steps)]
    for i in range(steps):
        step(i, marks[i])
    torch.cuda.synchronize()
    return (statistics.mean(a.elapsed_time(b) for a, b, _ in marks),
            statistics.mean(b.elapsed_time(c) for _, b, c in marks))


def _make_step(kfs, pr, flags, stream, grads, world=1, dp=None, flat=None, det=False):
    def step(i, timing=None):
        x, G = pr.sets[i % len(pr.sets)]
        if timing is not None:
            timing[0].record(stream)
        kfs.forward(x, pr.fac["S"], pr.fac["A"], pr.fac["B"], pr.fac["bias"], dtype=pr.path,
                    flags=flags, out=pr.y)
        if timing is not None:
            timing[1].record(stream)
        kfs.backward(x, pr.fac["S"], pr.fac["A"], pr.fac["B"], G, dtype=pr.path, flags=flags,
                     workspace=pr.wsb, grads=grads)
        if timing is not None:
            timing[2].record(stream)
        if world > 1:
            dp.allreduce_grads(flat, deterministic=det)
    return step


# Further legs of the default run (rank 0 alone, N = 1): the tutorial layer on the other two
# paths, then every other configuration on its own tensor-core path where the library has
# one (the workload's BF16 I/O, or TF32 for fp32 I/O), else on the exact-FP32 path for the
# fp32 workloads.  (workload, path or None for the workload's own, skip-zero-blocks flag)
LEGS = [("tutorial", "f32", 0), ("tutorial", "bf16", 0),
        ("gpt2_c_fc_r1", None, 0), ("gpt2_c_fc_r4", None, 0),
        ("gpt2_c_proj_r1", None, 0), ("gpt2_c_proj_r4", None, 0),
        ("stress", None, 0), ("stress", None, 1)] + \
       [(f"sweep_m{m}_r{r}", None, 0) for m in (8, 16, 64, 128) for r in (1, 2, 8)]


def _tc_forward_leg(kfs, pr, w, steps, peaks):
    """TF32 forward call alone on the fp32 tensors of `pr`, replayed from a CUDA graph;
    None when the library has no TF32 forward kernel for the shape."""
    fac = pr.fac

    def fwd(i):
        x, _ = pr.sets[i % len(pr.sets)]
        kfs.forward(x, fac["S"], fac["A"], fac["B"], fac["bias"], dtype="tf32", out=pr.y)
    try:
        fwd(0)
    except kfs.KronError:
        return None
    med, mn, _ = _time_graph(fwd, steps, REPEATS)
    ms = med / steps
    nbytes = w.N * 4 * (w.d_in + w.d_out)
    flops = w.N * 2 * w.r * (w.p * w.m1 * w.m2 + w.p * w.q * w.m2)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_fl = flops / (peaks["bf16_tflops"] * 1e12 / 2)
    t_roof = max(t_hbm, t_fl)
    return {"path": "tf32", "ms_per_call": ms, "ms_per_call_min": mn / steps,
            "timer": "CUDA graph replay", "roofline": {
                "bound": "hbm" if t_hbm >= t_fl else "tensor", "roofline_us": t_roof * 1e6,
                "hbm_us": t_hbm * 1e6, "flops_us": t_fl * 1e6, "frac": t_roof / (ms / 1e3),
                "flop_peak": "tf32 (measured bf16 x 1/2)", "bytes": nbytes, "flops": flops}}


def run_extras(kfs, steps, dev):
    """The two utilities built around the layer, timed on one GPU (rank 0):
    - the Van Loan rank-r fit of a dense W of the GPT-2 c_fc shape (768 x 3072, C_i 24 x 48,
      B_i 32 x 64) that is an exact sum of 4 Kronecker products, r = 4, k = 12, two power steps:
      time per fit (CUDA events around back-to-back fits) and the fit's relative Frobenius
      error (exact rank: rounding only);
    - the triple Kronecker layer with A 32 x 32, B 4 x 4, C 8 x 8, r = 4 (blocks of 32 x 32, the
      tutorial layer's tensor-core kernels) on 20000 rows, TF32: forward + backward step time
      from a CUDA-graph replay."""
    import torch
    from kronecker_factored_structured_b200 import native
    out = {}
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    p, q, m1, m2, r = 24, 48, 32, 64, 4
    C = torch.randn(r, p, q, device=dev, generator=g) / p ** 0.5
    B = torch.randn(r, m1, m2, device=dev, generator=g) / m1 ** 0.5
    W = sum(torch.kron(C[i], B[i]) for i in range(r)).float().contiguous()
    omega = torch.randn(12, m1 * m2, device=dev, generator=g)
    fit = native.vanloan_fit(W, p, q, m1, m2, r, k=12, omega=omega)
    torch.cuda.synchronize()
    times = []
    for _ in range(REPEATS):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(10):
            fit = native.vanloan_fit(W, p, q, m1, m2, r, k=12, omega=omega)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) / 10)
    Wf = sum(torch.kron(fit["A"][i], fit["B"][i]) for i in range(r))
    out["vanloan"] = {"what": "kron_vanloan_fit of a 768 x 3072 W of Kronecker rank 4 "
                              "(GPT-2 c_fc factor shapes), r = 4, k = 12, 2 power steps",
                      "ms_per_fit": statistics.median(times),
                      "rel_frobenius_error": float((Wf - W).norm() / W.norm()),
                      "alpha": float(fit["alpha"][0])}
    del W, Wf, fit, omega, C, B
    N, p, q, m1, m2, s1, s2, r = 20000, 32, 32, 4, 4, 8, 8, 4
    A3 = torch.randn(r, p, q, device=dev, generator=g) / p ** 0.5
    B3 = torch.randn(r, m1, m2, device=dev, generator=g) / m1 ** 0.5
    C3 = torch.randn(r, s1, s2, device=dev, generator=g) / s1 ** 0.5
    bias = 0.1 * torch.randn(q * m2 * s2, device=dev, generator=g)
    xs = [torch.randn(N, p * m1 * s1, device=dev, generator=g) for _ in range(ROTATE)]
    Gs = [torch.randn(N, q * m2 * s2, device=dev, generator=g) for _ in range(ROTATE)]

    def step(i):
        native.forward3(xs[i % ROTATE], A3, B3, C3, bias, dtype="tf32")
        native.backward3(xs[i % ROTATE], A3, B3, C3, Gs[i % ROTATE], dtype="tf32")
    step(0)
    torch.cuda.synchronize()
    med, _, _ = _time_graph(step, steps, REPEATS)
    ms = med / steps
    out["kron3"] = {"what": "triple Kronecker layer, A 32x32, B 4x4, C 8x8, r = 4, N = 20000, "
                            "TF32, forward + backward (CUDA-graph replay)",
                    "ms_per_step": ms, "rows_per_s": N / (ms / 1e3)}
    del xs, Gs
    torch.cuda.empty_cache()
    return out


def ks_permute_bmm_step(x, G, w, bias, pattern):
    """The Kronecker-sparse factor's forward and backward the way the page "Fast Inference
    with Kronecker-Sparse Matrices" describes earlier GPU kernels: permute x (and dY) into
    a*d contiguous slices, batched GEMMs, permute back.  Returns (y, dX, dw, dbias) with dw in
    the [a][d][b][c] layout.  Context for the bench only (torch ops; any device)."""
    import torch
    a, b, c, d = pattern
    N = x.shape[0]
    W3 = w.reshape(a * d, b, c)
    xt = x.view(N, a, b, d).permute(1, 3, 0, 2).reshape(a * d, N, b)
    y = torch.bmm(xt, W3).view(a, d, N, c).permute(2, 0, 3, 1).reshape(N, a * c * d) + bias
    Gt = G.view(N, a, c, d).permute(1, 3, 0, 2).reshape(a * d, N, c)
    dx = torch.bmm(Gt, W3.transpose(1, 2)).view(a, d, N, b).permute(2, 0, 3, 1).reshape(
        N, a * b * d)
    dw = torch.bmm(xt.transpose(1, 2), Gt).view(a, d, b, c)
    db = G.sum(0)
    return y, dx, dw, db


def ks_bmm_context(fac, sets, pattern, steps, dev):
    """Context only (not the product path): `ks_permute_bmm_step` (FP32 cuBLAS through torch,
    TF32 off) on the same inputs, forward + backward per step, replayed from a CUDA graph."""
    import torch
    old = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        def step(i):
            x, G = sets[i % len(sets)]
            return ks_permute_bmm_step(x, G, fac["w"], fac["bias"], pattern)
        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        ms = _time_graph(step, steps, REPEATS)[0] / steps
    finally:
        torch.backends.cuda.matmul.allow_tf32 = old
    return {"what": "permute + batched GEMM + permute back (torch/cuBLAS FP32, TF32 off), "
                    "forward and backward (dX, dw, dbias), same inputs, CUDA graph replay; "
                    "context only", "ms_per_step": ms}


KS_LEGS = ["ks_monarch_bd", "ks_monarch_tr", "ks_butterfly", "ks_gpt2m_up", "ks_block128"]


def run_ks_leg(kw, kfs, name, steps, warmup, peaks, dev, stream):
    """One Kronecker-sparse factor (include/ks_linear.h): forward + backward through the C
    ABI, exact FP32, CUDA-graph replay of `steps` steps (median of REPEATS), with the
    roofline max(bytes / HBM, flops / FFMA) and the permute + batched-GEMM context."""
    import torch
    from kronecker_factored_structured_b200 import accounting as acc
    from kronecker_factored_structured_b200 import native
    w = kw.ks_get(name)
    a, b, c, d = w.pattern
    fac = {k: v.to(dev) for k, v in kw.ks_factors(w).items()}
    rotate = ROTATE if w.N * (w.d_in + w.d_out) * 4 < 126e6 else 1
    sets = []
    for s in range(rotate):
        ws = dataclasses.replace(w, seed=w.seed + 1000 * s) if s else w
        sets.append((kw.rows(ws, "x").to(dev), kw.rows(ws, "G").to(dev)))
    y = torch.empty(w.N, w.d_out, device=dev)
    grads = {"dX": torch.empty(w.N, w.d_in, device=dev), "dw": torch.empty_like(fac["w"]),
             "dbias": torch.empty(w.d_out, device=dev)}
    wsb = torch.empty(native.ks_workspace_size(w.N, a, b, c, d), dtype=torch.uint8, device=dev)

    def step(i, timing=None):
        x, G = sets[i % len(sets)]
        if timing is not None:
            timing[0].record(stream)
        native.ks_forward(x, fac["w"], fac["bias"], out=y)
        if timing is not None:
            timing[1].record(stream)
        native.ks_backward(x, fac["w"], G, workspace=wsb, grads=grads)
        if timing is not None:
            timing[2].record(stream)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    med, mn, _ = _time_graph(step, steps, REPEATS)
    t_fwd, t_bwd = _split_calls(step, steps, stream)
    ms = med / steps
    nbytes = w.N * acc.bytes_per_row(w.d_in, w.d_out, 4)
    flops = w.N * acc.ks_flops_per_row(a, b, c, d)
    ffma = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6
    t_hbm, t_fl = nbytes / (peaks["hbm_gbs"] * 1e9), flops / ffma
    fwd_bytes = w.N * acc.bytes_per_row(w.d_in, w.d_out, 4, backward=False)
    leg = {"workload": f"Kronecker-sparse factor, pattern (a, b, c, d) = {w.pattern}, "
                       f"{w.d_in} -> {w.d_out}, N = {w.N}, fp32",
           "name": name, "path": "f32", "N": w.N, "steps": steps, "repeats": REPEATS,
           "timer": "CUDA graph replay of the steps", "ms_per_step": ms,
           "ms_per_step_min": mn / steps, "rows_per_s": w.N / (ms / 1e3),
           "fwd_ms": t_fwd, "bwd_ms": t_bwd, "call_split_timer": "eager, per-call events",
           "l2": f"{len(sets)} input set(s), {len(sets) * w.N * (w.d_in + w.d_out) * 4 / 1e6:.0f} MB",
           "forward_hbm_frac": (fwd_bytes / (peaks["hbm_gbs"] * 1e9)) / (t_fwd / 1e3),
           "roofline": {"bound": "hbm" if t_hbm >= t_fl else "alu",
                        "roofline_us": max(t_hbm, t_fl) * 1e6, "hbm_us": t_hbm * 1e6,
                        "flops_us": t_fl * 1e6, "frac": max(t_hbm, t_fl) / (ms / 1e3),
                        "flop_peak": "FFMA", "flop_peak_source": "derived", "bytes": nbytes,
                        "flops": flops}}
    ctx = ks_bmm_context(fac, sets, w.pattern, steps, dev)
    ctx["ks_speedup"] = ctx["ms_per_step"] / ms
    leg["context_bmm"] = ctx
    del sets, y, grads, wsb, fac
    torch.cuda.empty_cache()
    return leg


def run_leg(kw, kfs, name, path, flags, steps, warmup, peaks, dev, stream):
    """One further leg: the workload's forward + backward step, median of REPEATS timed
    regions of `steps` steps; a dict for the JSON line's "legs" list."""
    import torch
    w = kw.get(name)
    if path is None:
        path = "bf16" if w.dtype == "bf16" else "tf32"
    if not _path_supported(kfs, w, path):
        if w.dtype == "bf16":
            return {"workload": name, "path": path, "flags": flags,
                    "status": "unsupported: no tensor-core kernel for this shape"}
        alt = "f32"
        note = f"no {path} kernel for this shape: exact-FP32 path"
        path = alt
    else:
        note = None
    if path == "bf16" and w.dtype != "bf16":
        w = dataclasses.replace(w, dtype="bf16")
    rotate = ROTATE if w.N * (w.d_in + w.d_out) * (2 if path == "bf16" else 4) < 126e6 else 1
    pr = _Problem(kw, kfs, w, path, dev, rotate=rotate)
    f32 = torch.float32
    grads = {"dX": torch.empty(w.N, w.d_in, dtype=pr.y.dtype, device=dev),
             "dS": torch.empty(w.p, w.q, dtype=f32, device=dev),
             "dA": torch.empty(w.r, w.p, w.q, dtype=f32, device=dev),
             "dB": torch.empty(w.r, w.m1, w.m2, dtype=f32, device=dev),
             "dbias": torch.empty(w.d_out, dtype=f32, device=dev)}
    step = _make_step(kfs, pr, flags, stream, grads)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    # the leg's figure: the steps replayed from one CUDA graph (device time); the same
    # steps issued eagerly from Python are reported beside it
    med, mn, _ = _time_graph(step, steps, REPEATS)
    med_e, _, _ = _time_region(step, steps, REPEATS, 1, None, stream)
    t_fwd, t_bwd = _split_calls(step, steps, stream)
    ms = med / steps
    leg = {"workload": _workload_desc(w), "name": name, "path": path, "flags": flags,
           "N": w.N, "steps": steps, "repeats": REPEATS, "timer": "CUDA graph replay of the steps",
           "ms_per_step": ms, "ms_per_step_min": mn / steps, "rows_per_s": w.N / (ms / 1e3),
           "ms_per_step_eager": med_e / steps,
           "fwd_ms": t_fwd, "bwd_ms": t_bwd, "call_split_timer": "eager, per-call events",
           "l2": f"{len(pr.sets)} input set(s), "
                 f"{len(pr.sets) * w.N * (w.d_in + w.d_out) * (2 if path == 'bf16' else 4) / 1e6:.0f} MB",
           "roofline": _step_roofline(w, path, ms, peaks, flags)}
    if note:
        leg["note"] = note
    if note and path == "f32":
        # the step runs exact FP32; where the TF32 forward has a tensor-core kernel for the
        # shape, its forward call is timed alone the same way, against the forward roofline
        fwd_tc = _tc_forward_leg(kfs, pr, w, steps, peaks)
        if fwd_tc is not None:
            leg["forward_tf32"] = fwd_tc
    if name.startswith("gpt2"):
        ctx = dense_context(pr.fac, pr.sets, path, steps, dev, graph=True)
        ctx["kron_speedup"] = ctx["ms_per_step"] / ms
        leg["context_dense"] = ctx
    del pr, grads
    torch.cuda.empty_cache()
    return leg


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--path", default=None, help="tf32 | f32 | bf16 (default: headline path)")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--ref-rows", type=int, default=1024)
    ap.add_argument("--cpu-rows", type=int, default=None,
                    help="oracle rows for cpu_baseline (default: the whole batch when it is "
                         "at most 20000 rows of 1024 + 1024 values, else 1024)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-context", action="store_true",
                    help="skip the dense-layer context timing (cuBLAS through torch)")
    ap.add_argument("--no-legs", action="store_true",
                    help="time only the headline workload (no further legs)")
    ap.add_argument("--legs", default=None,
                    help="comma-separated workload names of the further legs (default: all)")
    ap.add_argument("--leg-steps", type=int, default=20)
    ap.add_argument("--skip-zero-blocks", action="store_true",
                    help="pass KRON_FLAG_SKIP_ZERO_BLOCKS (drop products with a zero S entry)")
    ap.add_argument("--deterministic-exchange", action="store_true",
                    help="N > 1: sum the ranks' gradients in rank order after an all-gather "
                         "(bitwise reproducible) instead of one all-reduce")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    import kron_workloads as kw
    w = kw.get(args.workload)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist

    import kronecker_factored_structured_b200 as kfs
    from kronecker_factored_structured_b200 import accounting as acc
    from kronecker_factored_structured_b200 import dp

    # default path: the workload's own I/O type (bf16 workloads run the BF16 path)
    path = args.path or ("bf16" if w.dtype == "bf16" else "tf32")
    flags = 1 if args.skip_zero_blocks else 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if path == "bf16" and w.dtype != "bf16":
        w = dataclasses.replace(w, dtype="bf16")
    kfs.native.load()

    # ---- inputs resident in HBM: ROTATE independent (x, G) sets, factors shared ----
    pr = _Problem(kw, kfs, w, path, dev, rank=rank)
    p, q, m1, m2, r, N = w.p, w.q, w.m1, w.m2, w.r, w.N
    t_io = kfs.native.io_dtype(path)
    elt = 2 if path == "bf16" else 4
    grads = {"dX": torch.empty(N, p * m1, dtype=t_io, device=dev)}
    # parameter gradients as views of one flat buffer: the one exchange of the data-parallel
    # backward is a single all-reduce of it
    flat, views = dp.flat_grad_buffer(p, q, m1, m2, r, device=dev)
    grads.update(views)
    stream = torch.cuda.current_stream()
    step = _make_step(kfs, pr, flags, stream, grads, world, dp, flat, args.deterministic_exchange)
    fac, sets, wsb = pr.fac, pr.sets, pr.wsb

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    # extra device memory of one step beyond the caller's tensors (inputs, outputs and the
    # workspace are all allocated above): the library allocates nothing itself
    torch.cuda.reset_peak_memory_stats(dev)
    base_bytes = torch.cuda.memory_allocated(dev)
    step(0)
    torch.cuda.synchronize()
    peak_extra = torch.cuda.max_memory_allocated(dev) - base_bytes

    # ---- timed region: REPEATS x (K steps between two events on the launching stream) ----
    with ClockSampler(torch.cuda.current_device()) as clk:
        clk.wait_started()
        ms_med, ms_min, ms_all = _time_region(step, args.steps, REPEATS, world, dist, stream, clk)
    # ---- the split into forward and backward call (outside the timed region) ----
    t_fwd, t_bwd = _split_calls(step, args.steps, stream)
    # ---- for information (one GPU): the same steps replayed from one CUDA graph ----
    graph_ms = _time_graph(step, args.steps, REPEATS)[0] / args.steps if world == 1 else None
    ms_step = ms_med / args.steps
    value = world * N * args.steps / (ms_med / 1e3)

    # ---- end to end through the public API with pinned host buffers ----
    xh = [s[0].cpu().pin_memory() for s in sets]
    gh = [s[1].cpu().pin_memory() for s in sets]
    yh = torch.empty(N, q * m2, dtype=t_io).pin_memory()
    dxh = torch.empty(N, p * m1, dtype=t_io).pin_memory()
    fh = torch.empty_like(flat, device="cpu").pin_memory()
    xd, gd = torch.empty_like(sets[0][0]), torch.empty_like(sets[0][1])

    def e2e_step(i):
        xd.copy_(xh[i % len(sets)], non_blocking=True)
        gd.copy_(gh[i % len(sets)], non_blocking=True)
        kfs.forward(xd, fac["S"], fac["A"], fac["B"], fac["bias"], dtype=path, flags=flags,
                    out=pr.y)
        kfs.backward(xd, fac["S"], fac["A"], fac["B"], gd, dtype=path, flags=flags, workspace=wsb,
                     grads=grads)
        if world > 1:
            dp.allreduce_grads(flat, deterministic=args.deterministic_exchange)
        yh.copy_(pr.y, non_blocking=True)
        dxh.copy_(grads["dX"], non_blocking=True)
        fh.copy_(flat, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 20))
    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    e2e_med, _, _ = _time_region(e2e_step, e2e_steps, 3, world, dist, stream)
    e2e_value = world * N * e2e_steps / (e2e_med / 1e3)
    h2d = xh[0].numel() * xh[0].element_size() + gh[0].numel() * gh[0].element_size()
    d2h = yh.numel() * yh.element_size() + dxh.numel() * dxh.element_size() + fh.numel() * 4
    del xh, gh, yh, dxh, fh, xd, gd

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    # ---- roofline of the dominant call (the backward) ----
    peaks = _peaks()
    bwd_bytes = N * elt * (2 * p * m1 + q * m2)
    bwd_flops = N * (acc.flops_per_row(p, q, m1, m2, r) - acc.flops_per_row(p, q, m1, m2, r, False))
    on_tc = path != "f32"
    # kernels of this library per step: tuned tensor-core kernels of the tutorial shape:
    # forward, dX, parameter gradients (with their fused reduction); CUDA cores on the
    # tutorial shape: forward, dX, parameter-gradient partials, reduction
    tutorial_shape = (p, q, m1, m2, r) == (32, 32, 32, 32, 4)
    compiled_f32 = path == "f32" and tutorial_shape and not flags
    launches_per_step = 4 if compiled_f32 or (on_tc and not tutorial_shape) else 3
    if not on_tc:
        peak = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12   # FFMA TFLOP/s at max clock
        achieved = bwd_flops / (t_bwd / 1e3) / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": None,
                "kernel": "backward call on the CUDA cores (dX, parameter-gradient partials, "
                          "reduction)",
                "peak_source": "derived: 148 SMs x 128 FFMA/clk x 2 x max SM clock"}
    else:
        achieved = bwd_bytes / (t_bwd / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": _traffic(path, args.workload),
                "kernel": "backward call: dX kernel + parameter-gradient kernel",
                "peak_source": peaks["source"]}

    step_bytes = N * acc.bytes_per_row(p * m1, q * m2, elt)
    step_flops = N * acc.flops_per_row(p, q, m1, m2, r)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": path, "data": "synthetic",
        "config": {"workload": _workload_desc(w), "N": N, "p": p, "q": q, "m1": m1, "m2": m2,
                   "r": r, "path": path, "parallelism": f"dp{world}",
                   "exchange": ("all-gather, rank-ordered sum" if args.deterministic_exchange
                                else "all-reduce") if world > 1 else None,
                   "skip_zero_blocks": bool(flags),
                   "l2": f"inputs rotated over {len(sets)} independent (x, dY) sets "
                         f"({len(sets) * N * elt * (p * m1 + q * m2) / 1e6:.0f} MB > 126 MB L2)"},
        "repeats": {"n": REPEATS, "ms_per_step": [t / args.steps for t in ms_all],
                    "median": ms_step, "min": ms_min / args.steps},
        "fwd_ms": t_fwd, "bwd_ms": t_bwd,
        "graph": None if graph_ms is None else {
            "ms_per_step": graph_ms, "rows_per_s": N / (graph_ms / 1e3),
            "what": "the same steps captured once in a CUDA graph and replayed (information; "
                    "value is the eager figure, the same at every GPU count)"},
        "tflops": step_flops / (ms_step / 1e3) / 1e12,
        "gbs": step_bytes / (ms_step / 1e3) / 1e9,
        "step_roofline_frac_hbm": (step_bytes / (peaks["hbm_gbs"] * 1e9)) / (ms_step / 1e3),
        "roofline": roof,
        "gpu_launches": REPEATS * args.steps * launches_per_step,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "clocks": clk.summary(),
    }
    line["memory"] = {"workspace_bytes": int(wsb.numel()), "peak_extra_bytes_per_step": int(peak_extra)}
    if not args.no_context:
        ctx = dense_context(fac, sets, path, max(10, min(args.steps, 100)), dev)
        ctx["kron_ms_per_step"] = ms_step
        ctx["kron_speedup"] = ctx["ms_per_step"] / ms_step
        line["context_dense"] = ctx
    del pr, sets, fac, grads, flat, views, step
    torch.cuda.empty_cache()
    if world == 1 and not args.no_legs:
        names = args.legs.split(",") if args.legs else None
        legs = []
        for name, lpath, lflags in LEGS:
            if names is not None and name not in names:
                continue
            legs.append(run_leg(kw, kfs, name, lpath, lflags, max(3, min(args.steps, args.leg_steps)),
                                args.warmup, peaks, dev, stream))
        line["legs"] = legs
        line["ks_legs"] = [run_ks_leg(kw, kfs, name, max(3, min(args.steps, args.leg_steps)),
                                      args.warmup, peaks, dev, stream)
                           for name in KS_LEGS if names is None or name in names]
        line["extras"] = run_extras(kfs, max(3, min(args.steps, args.leg_steps)), dev)
    if world == 1 and not args.no_cpu_baseline:
        cpu_rows = args.cpu_rows or (N if N * (w.d_in + w.d_out) <= 20000 * 2048 else 1024)
        rows_s, dt, cores = cpu_baseline(w, cpu_rows)
        line["cpu_baseline"] = {"value": rows_s, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"first {cpu_rows} of {N} rows, forward + "
                                          f"backward, {dt:.1f} s"}
        # the same oracle on one host thread, on a smaller sample (about 16x slower per row)
        import oracle
        all_threads = oracle.get_threads()
        rows1 = max(64, min(cpu_rows, 1024))
        try:
            rows_s1, dt1, _ = cpu_baseline(w, rows1, threads=1)
        finally:
            oracle.set_threads(all_threads)
        line["cpu_baseline_single_thread"] = {
            "value": rows_s1, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"first {rows1} of {N} rows, forward + backward, {dt1:.1f} s"}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
