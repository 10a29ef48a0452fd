"""Benchmark of the Titans memory's chunk-wise update + retrieve on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one titans_mem_forward over the whole workload: every (batch, head) unit
runs all its chunks (update + retrieve) in one persistent kernel launch. The default
workload is the 760M-class layer shape: MLP memory 64 -> 256 -> 64, B=8, H=16,
T=4096, chunk 64. Inputs are seeded synthetic data (titans_long_term_b200.synth),
resident in HBM before the timed region. Units are independent, so under torchrun
every rank runs its own B*H units (weak scaling, no data-path collective); the
elapsed time is the max over ranks.

Prints one JSON line (rank 0). ``--impl reference`` times the fp64 CPU oracle (the
reference arm for this method) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

from titans_long_term_b200 import mem, synth  # noqa: E402

METRIC = "memory tokens/sec (update+retrieve) per B200; % bf16 tensor-core peak"
KERNEL_NAMES = {mem.PATH_TC_MLP64: "chunk_fwd_tc_mlp64", mem.PATH_CUDA_CORES: "chunk_fwd_cuda_cores",
                mem.PATH_TC_PHASED: "chunk_fwd_tc_phased", mem.PATH_TC_DEEP: "chunk_fwd_tc_deep",
                mem.PATH_DEEP_CUDA_CORES: "chunk_fwd_deep_cuda_cores"}
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def flops_per_head_token(w) -> float:
    """Algorithmic FLOPs: MLP 18 d h (key forward 4dh, backprop to the hidden units 2dh, four
    weighted outer-product sums 8dh, query retrieval 4dh); linear 8 d^2."""
    return 18.0 * w.d * w.h if w.h else 8.0 * w.d * w.d


def stream_bytes_per_head_token(w) -> float:
    """k, q, v in, y out (input dtype) + three fp32 gates."""
    e = 2 if w.dtype == "bf16" else 4
    return 4 * w.d * e + 12


def state_bytes_per_unit(w) -> float:
    """W and S read once and written once per call (fp32): 4 x |W| x 4 B, |W| = |W1| + |W2|."""
    n = 2 * w.d * w.h if w.h else w.d * w.d
    return 4 * n * 4


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clocks and clock-event reasons around and inside the timed region: nvidia-smi samples
    every 50 ms from start() to stop(), and NVML reads (read-only queries) about every millisecond
    between mark_start() and mark_stop(), so that a timed region of a few milliseconds still has
    samples of its own."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t_start = self.t_stop = None
        self.nvml = None       # pynvml module once initialised
        self.nvml_rows = []    # (sm MHz, event-reason bitmask) inside the timed region
        self._poll = None
        self._polling = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._handle = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self._max_sm = float(pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM))
            self.nvml = pynvml
        except Exception:  # no NVML: nvidia-smi samples only
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._reader = threading.Thread(target=self._read, daemon=True)
        self._reader.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def _poll_nvml(self):
        nv, h = self.nvml, self._handle
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while self._polling:
            try:
                self.nvml_rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), int(reasons(h))))
            except Exception:
                return
            time.sleep(0.005)

    def mark_start(self):
        self.t_start = time.time()
        if self.nvml is not None:
            self._polling = True
            self._poll = threading.Thread(target=self._poll_nvml, daemon=True)
            self._poll.start()

    def mark_stop(self):
        if self._poll is not None:
            self._polling = False
            self._poll.join(timeout=1.0)
        self.t_stop = time.time()

    def stop(self):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass

    def _nvml_reasons(self, mask: int):
        nv = self.nvml
        names = {"hw_slowdown": "HwSlowdown", "hw_thermal_slowdown": "HwThermalSlowdown",
                 "sw_thermal_slowdown": "SwThermalSlowdown", "sw_power_cap": "SwPowerCap",
                 "hw_power_brake_slowdown": "HwPowerBrakeSlowdown"}
        out = set()
        for key, suffix in names.items():
            bit = getattr(nv, "nvmlClocksEventReason" + suffix, None) or getattr(nv, "nvmlClocksThrottleReason" + suffix, 0)
            if mask & bit:
                out.add(key)
        return out

    def summary(self):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        inside = [p for ts, p in rows if self.t_start and self.t_stop and self.t_start - 0.1 <= ts <= self.t_stop + 0.1]
        use = inside or [p for _, p in rows]
        if not use and not self.nvml_rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for p in use if num(p[1]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in use:
            for name, val in zip(names, p[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        for _, mask in self.nvml_rows:
            reasons |= self._nvml_reasons(mask)
        nvml_sm = [float(c) for c, _ in self.nvml_rows]
        out = {"sm_mhz": statistics.median(nvml_sm) if nvml_sm else (statistics.median(sm) if sm else None),
               "sm_max_mhz": num(use[0][2]) if use else getattr(self, "_max_sm", None), "reasons": sorted(reasons),
               "samples": len(use), "samples_in_timed_region": len(inside) + len(nvml_sm),
               "nvml_samples_in_timed_region": len(nvml_sm)}
        if use:
            out["power_w_max"] = max((num(p[3]) or 0.0) for p in use)
        if nvml_sm:
            out["sm_mhz_min_in_timed_region"] = min(nvml_sm)
        return out


# ---------------------------------------------------------------- oracle (CPU baseline / reference arm)

def oracle_rate(w) -> float:
    """Head-tokens per second of the fp64 oracle on this host, from a short calibration run."""
    import oracle
    cores = oracle.threads()
    cal = synth.make_inputs(w, units=range(min(w.units, cores)), T=min(w.T, 2 * w.chunk))
    st = {n: cal[n] for n in cal if n[0] in "WS"}
    t = time.perf_counter()
    oracle.forward(*(cal[n] for n in ("k", "q", "v", "alpha", "eta", "theta")), st, w.chunk)
    return cal["k"].shape[0] * cal["k"].shape[1] / max(time.perf_counter() - t, 1e-6)


def oracle_sample(w, core_seconds: float = 15.0, units_cap: int = 0, rate: float = 0.0):
    """Time the fp64 oracle (token loop, OpenMP over units, all host cores) on a bounded
    sample of the workload: the first U units x the first T tokens, sized from a short
    calibration run (or the given rate, head-tokens/s) to about `core_seconds` of CPU work."""
    import oracle
    cores = oracle.threads()
    rate = rate or oracle_rate(w)
    want = rate * core_seconds / cores  # head-tokens for the target wall time
    units = min(w.units, units_cap or w.units, max(1, cores))
    T = int(min(w.T, max(w.chunk, (want / units) // w.chunk * w.chunk)))
    while units < min(w.units, units_cap or w.units) and units * T < want and T == w.T:
        units = min(w.units, units * 2)
    inp = synth.make_inputs(w, units=range(units), T=T)
    st = {n: inp[n] for n in inp if n[0] in "WS"}
    t = time.perf_counter()
    oracle.forward(*(inp[n] for n in ("k", "q", "v", "alpha", "eta", "theta")), st, w.chunk)
    dt = time.perf_counter() - t
    return {"value": units * T / w.H / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{units} units x {T} tokens of {w.name} (fp64 token loop), {dt:.2f} s wall",
            "seconds": dt, "cpu_model": cpu_model()}


def cpu_model() -> str:
    """The host CPU's model name (/proc/cpuinfo), or "unknown"."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def reference_arm(args, w, rank, world):
    """The reference arm: the oracle as it stands, on this host's cores, one bounded sample per
    step (sized so that warm-up + steps take about two minutes), rank 0 only."""
    if rank != 0:
        return
    import oracle
    per_step = 120.0 * oracle.threads() / max(1, args.steps + args.warmup)
    per_step = min(per_step, 30.0 * oracle.threads())
    rate = oracle_rate(w)  # calibrated once, so that many short steps stay cheap
    for _ in range(args.warmup):
        oracle_sample(w, core_seconds=per_step / 4, rate=rate)
    vals, base = [], None
    for _ in range(args.steps):
        base = oracle_sample(w, core_seconds=per_step, rate=rate)
        vals.append(base["value"])
    value = statistics.median(vals)
    base["value"] = value
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * w.B * w.T / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "impl": "reference",
            "config": {"workload": w.name, "memory": f"MLP {w.d}-{w.h}-{w.d} SiLU" if w.h else f"linear {w.d}",
                       "B": w.B, "H": w.H, "T": w.T, "chunk": w.chunk, "units": w.units,
                       "inputs": synth.describe(w)},
            "cpu_baseline": base,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- multi-rank helpers

def rank_units(w, rank: int):
    """Units of one rank: rank r runs units [r * B*H, (r + 1) * B*H) of a (world * B) x H batch, so
    every rank processes its own data and per-GPU work stays fixed as ranks are added (weak scaling)."""
    return list(range(rank * w.units, (rank + 1) * w.units))


def max_over_ranks(value: float, device, world: int) -> float:
    """Max of a per-rank duration over all ranks (the job is as slow as its slowest rank)."""
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- our arm

def our_arm(args, w, rank, world, local_rank):
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    units = rank_units(w, rank)
    inp = synth.make_inputs(w, units=units)
    toks = {n: inp[n].reshape(w.B, w.H, w.T, w.d).to(dev) for n in ("k", "q", "v")}
    gates = {n: inp[n].reshape(w.B, w.H, w.T).to(dev) for n in ("alpha", "eta", "theta")}
    state0 = {n: inp[n].reshape(w.B, w.H, *inp[n].shape[1:]).to(dev) for n in inp if n[0] in "WS"}
    state = {n: t.clone() for n, t in state0.items()}
    y = torch.empty_like(toks["k"])
    m = mem.Memory(w.d, w.h, w.chunk, w.dtype, w.B, w.H)
    path = m.path()
    stream = torch.cuda.current_stream(dev)

    def step():
        m.forward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state, y=y)

    for _ in range(args.warmup):
        step()
    m.sync_status()
    if world > 1:
        torch.distributed.barrier()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    phys = vis.split(",")[local_rank] if vis else str(local_rank)
    clocks = ClockSampler(int(phys) if phys.isdigit() else local_rank)
    if rank == 0:
        clocks.start()
    # Device-timed region: K launches, one event pair per launch on the launching stream.
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clocks.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark_stop()
    if world > 1:
        torch.distributed.barrier()
    m.sync_status()
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), dev, world)
    launch_ms = [a.elapsed_time(b) for a, b in evs]

    # End-to-end through the public API from pinned host memory: titans_mem_forward_host copies
    # the step's inputs in and y out segment by segment, overlapping the copies with the
    # forward (the device arrays above serve as its staging buffers).
    host = {n: inp[n].reshape(t_.shape).pin_memory() for n, t_ in list(toks.items()) + list(gates.items())}
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    h2d = sum(t_.numel() * t_.element_size() for t_ in host.values())
    d2h = y_host.numel() * y_host.element_size()
    e_steps = max(3, min(args.steps, 20))
    staging = dict(toks, **gates, y=y)

    def e2e_step():
        m.forward_host(host["k"], host["q"], host["v"], host["alpha"], host["eta"], host["theta"], state, y_host,
                       staging)

    e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e_steps, dev, world)
    m.sync_status()
    if rank == 0:
        clocks.stop()
    if rank != 0:
        return

    ms = elapsed_ms / args.steps
    tokens = world * w.B * w.T
    value = tokens / (ms / 1e3)
    peaks, which = load_peaks()
    avg_launch = statistics.mean(launch_ms)
    flops = flops_per_head_token(w) * w.units * w.T
    achieved = flops / (avg_launch / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    algo_bytes = stream_bytes_per_head_token(w) * w.units * w.T + state_bytes_per_unit(w) * w.units
    traffic = None
    prof = os.path.join(HERE, "profiles", "traffic.json")
    if os.path.exists(prof):
        tr = json.load(open(prof)).get(w.name)
        if tr and tr.get("kernel_sha") == kernel_sha():
            traffic = tr["bytes_per_launch"]
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp32",
        "data": "synthetic (seeded; k, v, q projections of one x_t)",
        "config": {"workload": w.name, "inputs": synth.describe(w),
                   "memory": f"MLP {w.d}-{w.h}-{w.d} SiLU" if w.h else f"linear {w.d}x{w.d}",
                   "B": w.B, "H": w.H, "T": w.T, "chunk": w.chunk, "units_per_gpu": w.units,
                   "kernel": KERNEL_NAMES.get(path, str(path)),
                   "l2": "inputs larger than L2 (k, q, v, y, state = %.0f MB per step)" % (algo_bytes / 1e6)},
        "head_tokens_per_s": value * w.H,
        "pct_bf16_peak": 100.0 * achieved / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"bf16_tflops ({which})", "kernel": KERNEL_NAMES.get(path, str(path)),
                     "flops_per_launch": flops, "avg_launch_ms": avg_launch,
                     "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peak),
                     "algorithmic_bytes_per_launch": algo_bytes,
                     "hbm_gbs_at_algorithmic_bytes": algo_bytes / (avg_launch / 1e3) / 1e9},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "api": "titans_mem_forward_host (pinned host buffers, ~16 overlapped segments)"},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    if world == 1 and not args.no_extras:
        del toks, gates, state0, state, y, host, y_host, staging, m
        torch.cuda.empty_cache()
        line["results"] = extra_results(args, dev)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(w)
    print(json.dumps(line), flush=True)


FP32_FMA_TFLOPS_NOMINAL = 148 * 128 * 2 * 1.965e9 / 1e12  # SMs x FMA lanes x 2 FLOP x max SM clock


def time_launches(fn, stream, steps: int, warmup: int):
    """Device time of `steps` calls of fn after `warmup` untimed ones: CUDA events on the launching
    stream around the whole run and around each launch. Returns (total ms, [per-launch ms])."""
    for _ in range(warmup):
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(steps):
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1), [a.elapsed_time(b) for a, b in evs]


def forward_measure(w, dev, steps: int, warmup: int, T=None):
    """titans_mem_forward over the whole workload (or its first T tokens per unit), inputs resident in
    HBM; one launch per step. Returns a result record with the dominant kernel's roofline."""
    T = w.T if T is None else T
    inp = synth.make_inputs(w, T=T)
    toks = {n: inp[n].reshape(w.B, w.H, T, w.d).to(dev) for n in ("k", "q", "v")}
    gates = {n: inp[n].reshape(w.B, w.H, T).to(dev) for n in ("alpha", "eta", "theta")}
    state = {n: inp[n].reshape(w.B, w.H, *inp[n].shape[1:]).to(dev) for n in inp if n[0] in "WS"}
    del inp
    y = torch.empty_like(toks["k"])
    m = mem.Memory(w.d, w.h, w.chunk, w.dtype, w.B, w.H)
    path = m.path()
    stream = torch.cuda.current_stream(dev)
    fn = lambda: m.forward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state, y=y)
    total, per = time_launches(fn, stream, steps, warmup)
    m.sync_status()
    ms = total / steps
    avg = statistics.mean(per)
    peaks, which = load_peaks()
    flops = flops_per_head_token(w) * w.units * T
    achieved = flops / (avg / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    algo_bytes = stream_bytes_per_head_token(w) * w.units * T + state_bytes_per_unit(w) * w.units
    kernel = KERNEL_NAMES.get(path)
    sms = min(w.units, 148)
    rec = {"workload": w.name, "value": w.B * T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
           "steps": steps, "warmup": warmup, "head_tokens_per_s": w.B * T * w.H / (ms / 1e3),
           "config": {"memory": f"MLP {w.d}-{w.h}-{w.d} SiLU" if w.h else f"linear {w.d}x{w.d}", "B": w.B,
                      "H": w.H, "T": w.T, "T_timed": T, "chunk": w.chunk, "units": w.units,
                      "inputs": synth.describe(w)},
           "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                        "frac": achieved / peak, "traffic": None, "peak_source": f"bf16_tflops ({which})",
                        "kernel": kernel, "flops_per_launch": flops, "avg_launch_ms": avg,
                        "sms_used": sms, "frac_of_sms_used": achieved / (peak * sms / 148),
                        "algorithmic_bytes_per_launch": algo_bytes},
           "gpu_launches": steps}
    if path == mem.PATH_CUDA_CORES:
        rec["roofline"]["note"] = "CUDA-core fp32 FMA kernel; frac is against the bf16 tensor-core peak the work is bound by"
        rec["roofline"]["frac_of_fp32_fma_nominal"] = achieved / FP32_FMA_TFLOPS_NOMINAL
    del toks, gates, state, y, m
    torch.cuda.empty_cache()
    return rec


def decode_measure(w, dev, steps: int, warmup: int):
    """One step = one titans_mem_step (single-token update + retrieve) for every decode unit
    (decode_B x H), starting from seeded states; bound by HBM: each unit reads and writes its
    four fp32 state matrices once per step. Returns (result record, list of per-launch ms)."""
    n = w.decode_B * w.H
    src = synth.decode_state_rows(w)
    st0 = synth.make_inputs(w, units=sorted(set(src.tolist())), T=1)
    pos = {u: i for i, u in enumerate(sorted(set(src.tolist())))}
    idx = torch.as_tensor([pos[int(u)] for u in src])
    state = {nm: st0[nm][idx].reshape(w.decode_B, w.H, *st0[nm].shape[1:]).contiguous().to(dev)
             for nm in st0 if nm[0] in "WS"}
    K = max(steps, 1)
    steps_in = [synth.decode_step_inputs(w, s) for s in range(min(K, 16))]
    dev_in = [{k: v.reshape(w.decode_B, w.H, *v.shape[1:]).to(dev) for k, v in d.items()} for d in steps_in]
    m = mem.Memory(w.d, w.h, 1, w.dtype, w.decode_B, w.H)
    y = torch.empty_like(dev_in[0]["k"])
    it = [0]

    def step():
        g = dev_in[it[0] % len(dev_in)]
        it[0] += 1
        m.step(g["k"], g["q"], g["v"], g["alpha"], g["eta"], g["theta"], state, y=y)

    total, per = time_launches(step, torch.cuda.current_stream(dev), K, warmup)
    m.sync_status()
    ms = total / K
    avg = statistics.mean(per)
    peaks, which = load_peaks()
    state_bytes = n * 2 * (4 * w.d * w.h * 4)  # W1, W2, S1, S2 (fp32, d*h each): read once, written once
    io_bytes = n * (4 * w.d * (2 if w.dtype == "bf16" else 4) + 12)
    gbs = (state_bytes + io_bytes) / (avg / 1e3) / 1e9
    rec = {"workload": w.name + " decode", "value": w.decode_B / (ms / 1e3), "unit": "tokens/s",
           "ms_per_step": ms, "steps": K, "warmup": warmup,
           "config": {"decode_B": w.decode_B, "H": w.H, "units": n, "inputs": synth.describe(w),
                      "l2": "state larger than L2 (%.2f GB per step)" % (state_bytes / 1e9)},
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm_gbs"], "traffic": None, "peak_source": f"hbm_gbs ({which})",
                        "kernel": "step_mlp_cluster", "bytes_per_launch": state_bytes + io_bytes,
                        "avg_launch_ms": avg},
           "gpu_launches": K}
    del state, dev_in, y, m
    torch.cuda.empty_cache()
    return rec


def decode_arm(args, w, rank, world, local_rank):
    """--phase decode: one JSON line for the decode step alone (every rank runs its own decode batch)."""
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    rec = decode_measure(w, dev, args.steps, args.warmup)
    ms = max_over_ranks(rec["ms_per_step"], dev, world)
    if rank != 0:
        return
    cfg = dict(rec["config"], workload=rec["workload"])
    print(json.dumps({
        "metric": "decode tokens/sec (single-token update+retrieve, every head) per B200",
        "value": world * w.decode_B / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": rec["steps"],
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded)", "config": cfg,
        "roofline": rec["roofline"], "gpu_launches": rec["gpu_launches"]}), flush=True)


def _dev_inputs(w, dev, T=None, units=None):
    """Seeded inputs of a workload on the device, shaped [B, H, ...] (units = B*H)."""
    T = w.T if T is None else T
    inp = synth.make_inputs(w, T=T)
    toks = {n: inp[n].reshape(w.B, w.H, T, w.d).to(dev) for n in ("k", "q", "v")}
    gates = {n: inp[n].reshape(w.B, w.H, T).to(dev) for n in ("alpha", "eta", "theta")}
    state = {n: inp[n].reshape(w.B, w.H, *inp[n].shape[1:]).to(dev) for n in inp if n[0] in "WS"}
    return toks, gates, state


def _cuda_core_roofline(flops, avg_ms, kernel, units, note):
    """Roofline record of a CUDA-core kernel: fp32 FMA work against the nominal fp32 FMA peak
    (148 SMs x 128 lanes x 2 FLOP x 1.965 GHz) and the SMs its one-CTA-per-unit grid can use."""
    achieved = flops / (avg_ms / 1e3) / 1e12
    sms = min(units, 148)
    return {"bound": "alu", "achieved": achieved, "peak": FP32_FMA_TFLOPS_NOMINAL, "unit": "TFLOP/s",
            "frac": achieved / FP32_FMA_TFLOPS_NOMINAL, "traffic": None,
            "peak_source": "fp32 FMA nominal (148 SMs x 128 lanes x 2 FLOP x 1.965 GHz)", "kernel": kernel,
            "flops_per_launch": flops, "avg_launch_ms": avg_ms, "sms_used": sms,
            "frac_of_sms_used": achieved / (FP32_FMA_TFLOPS_NOMINAL * sms / 148), "note": note}


def deep_flops_per_head_token(d, h, layers) -> float:
    """Algorithmic FLOPs of a deep memory per head-token, with P = the weights of one state copy:
    key forward 2P, retrieval 2P, back-propagation to every hidden layer 2(P - d h), and the c- and
    d-weighted outer products 4P. At 2 layers this is the 2-layer memory's 18 d h."""
    P = sum(o * i for o, i in synth.deep_shapes(d, h, layers))
    return 10 * P - 2 * d * h


def extension_results(dev, steps: int, warmup: int):
    """The extension rows, each timed on its own workload: the memory-as-a-gate output and chunk-shared
    gates on the benchmarked kernel, the linear memory's cross-chunk scan, the deep memory and the
    backward (outer-loop gradients) of the 2-layer memory."""
    out = {}
    peaks, which = load_peaks()
    # memory-as-a-gate output and chunk-shared gates: the 760M-class workload on the tensor-core kernel
    w = synth.WORKLOADS["mlp-d64-b8h16-t4k"]
    toks, gates, state = _dev_inputs(w, dev)
    attn = synth.make_attn(w).reshape(w.B, w.H, w.T, w.d).to(dev)
    st0 = {n: t.clone() for n, t in state.items()}
    flops = flops_per_head_token(w) * w.units * w.T
    for name, chunk_gates in (("gated_output", False), ("chunk_gates", True)):
        m = mem.Memory(w.d, w.h, w.chunk, w.dtype, w.B, w.H, chunk_gates=chunk_gates)
        g = gates if not chunk_gates else {n: t[..., ::w.chunk].contiguous() for n, t in gates.items()}
        st = {n: t.clone() for n, t in st0.items()}
        o = torch.empty_like(toks["k"])
        if name == "gated_output":
            fn = lambda: m.forward_gated(toks["k"], toks["q"], toks["v"], g["alpha"], g["eta"], g["theta"], attn, st, o=o)
        else:
            fn = lambda: m.forward(toks["k"], toks["q"], toks["v"], g["alpha"], g["eta"], g["theta"], st, y=o)
        total, per = time_launches(fn, torch.cuda.current_stream(dev), steps, warmup)
        m.sync_status()
        avg = statistics.mean(per)
        achieved = flops / (avg / 1e3) / 1e12
        out[name] = {"workload": w.name, "value": w.B * w.T / (total / steps / 1e3), "unit": "tokens/s",
                     "ms_per_step": total / steps, "steps": steps,
                     "config": {"path": KERNEL_NAMES.get(m.path()), "chunk_gates": chunk_gates,
                                "gated_output": name == "gated_output"},
                     "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                                  "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                                  "peak_source": f"bf16_tflops ({which})", "kernel": KERNEL_NAMES.get(m.path()),
                                  "avg_launch_ms": avg},
                     "gpu_launches": steps}
        del m, st, o
    del toks, gates, state, st0, attn
    torch.cuda.empty_cache()

    # linear memory, one 65,536-token stream: the three-kernel cross-chunk scan against the chunk loop
    wl = synth.Workload("linear-d64-t64k", 64, 0, 1, 1, 65536, 16, "fp32", 20250106, recipe="stated")
    toks, gates, state = _dev_inputs(wl, dev)
    rec = {}
    for scan in (False, True):
        m = mem.Memory(wl.d, 0, wl.chunk, wl.dtype, 1, 1, chunk_scan=scan)
        st = {n: t.clone() for n, t in state.items()}
        fn = lambda: m.forward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], st)
        total, per = time_launches(fn, torch.cuda.current_stream(dev), max(3, steps // 2), warmup)
        m.sync_status()
        rec[scan] = (total / max(3, steps // 2), statistics.mean(per))
        del m, st
    flops = 8.0 * wl.d * wl.d * wl.T
    out["linear_scan"] = {
        "workload": wl.name, "value": wl.T / (rec[True][0] / 1e3), "unit": "tokens/s", "ms_per_step": rec[True][0],
        "chunk_loop_ms": rec[False][0], "speedup_vs_chunk_loop": rec[False][0] / rec[True][0],
        "config": {"memory": "linear 64x64", "units": 1, "T": wl.T, "chunk": wl.chunk, "mode": "fp32",
                   "inputs": synth.describe(wl)},
        "roofline": _cuda_core_roofline(flops, rec[True][1], "linear_scan_compose/segments/run", 148,
                                        "fp32 on CUDA cores; FLOPs are the chunk recurrence's 8 d^2 per token, "
                                        "not the scan's extra composition work"),
        "gpu_launches": 3 * max(3, steps // 2)}
    del toks, gates, state
    torch.cuda.empty_cache()

    # deep memory (4 layers, 64 -> 256 -> 256 -> 256 -> 64): the 760M-class layer shape on the tensor-core
    # kernel, and the 8-unit 2K-token workload on both kernels
    L = 4
    for key, wname, kernels in (("deep_memory", "mlp-d64-b8h16-t4k", (False,)),
                                ("deep_memory_8units", "mlp-d64-b2h4-t2k", (False, True))):
        w = synth.WORKLOADS[wname]
        toks, gates, _ = _dev_inputs(w, dev)
        dst = {n: t.reshape(w.B, w.H, -1).to(dev) for n, t in synth.make_deep_state(w, L).items()}
        flops = deep_flops_per_head_token(w.d, w.h, L) * w.units * w.T
        rec = None
        for cuda_cores in kernels:
            m = mem.Memory(w.d, w.h, w.chunk, w.dtype, w.B, w.H, layers=L, cuda_cores=cuda_cores)
            st = {n: t.clone() for n, t in dst.items()}
            fn = lambda: m.forward_deep(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], st)
            n_deep = steps if not cuda_cores else 3
            total, per = time_launches(fn, torch.cuda.current_stream(dev), n_deep, 1 if cuda_cores else warmup)
            m.sync_status()
            avg = statistics.mean(per)
            if cuda_cores:
                rec["cuda_cores"] = {"ms_per_step": total / n_deep, "roofline": _cuda_core_roofline(
                    flops, avg, "chunk_fwd_deep_cuda_cores", w.units, "fp32 on CUDA cores, one CTA per unit")}
                rec["speedup_vs_cuda_cores"] = (total / n_deep) / rec["ms_per_step"]
            else:
                achieved = flops / (avg / 1e3) / 1e12
                rec = {"workload": f"{w.name} deep L={L}", "value": w.B * w.T / (total / n_deep / 1e3), "unit": "tokens/s",
                       "ms_per_step": total / n_deep, "steps": n_deep,
                       "config": {"memory": f"deep {L}-layer {w.d}-{w.h}-{w.h}-{w.h}-{w.d} SiLU", "units": w.units,
                                  "T": w.T, "chunk": w.chunk,
                                  "flops_per_head_token": deep_flops_per_head_token(w.d, w.h, L),
                                  "inputs": synth.describe(w)},
                       "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                                    "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                                    "peak_source": f"bf16_tflops ({which})", "kernel": "chunk_fwd_tc_deep",
                                    "flops_per_launch": flops, "avg_launch_ms": avg},
                       "gpu_launches": n_deep}
            del m, st
        out[key] = rec
        del dst, toks, gates
        torch.cuda.empty_cache()

    # backward of the 2-layer memory (gradients of <dy, y> with respect to every input): the 760M-class
    # workload on the tensor-core backward, and the 8-unit 2K-token workload on both backward kernels
    for key, wname, kernels in (("backward", "mlp-d64-b8h16-t4k", (False,)),
                                ("backward_8units", "mlp-d64-b2h4-t2k", (False, True))):
        w = synth.WORKLOADS[wname]
        toks, gates, state = _dev_inputs(w, dev)
        dy = torch.randn(toks["k"].shape, generator=torch.Generator().manual_seed(5)).to(toks["k"].dtype).to(dev)
        flops = 2 * flops_per_head_token(w) * w.units * w.T
        rec = None
        for cuda_cores in kernels:
            m = mem.Memory(w.d, w.h, w.chunk, w.dtype, w.B, w.H, cuda_cores=cuda_cores)
            fn = lambda: m.backward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"],
                                    state, dy)
            nb = 3
            total, per = time_launches(fn, torch.cuda.current_stream(dev), nb, 1)
            m.sync_status()
            avg = statistics.mean(per)
            if cuda_cores:
                rec["cuda_cores"] = {"ms_per_step": total / nb, "roofline": _cuda_core_roofline(
                    flops, avg, "mlp_backward_kernel", w.units,
                    "fp32 on CUDA cores, one CTA per unit (TITANS_FLAG_CUDA_CORES)")}
                rec["speedup_vs_cuda_cores"] = (total / nb) / rec["ms_per_step"]
            else:
                achieved = flops / (avg / 1e3) / 1e12
                sms = min(w.units, 148)
                rec = {"workload": f"{w.name} backward", "value": w.B * w.T / (total / nb / 1e3), "unit": "tokens/s",
                       "ms_per_step": total / nb, "steps": nb,
                       "config": {"memory": f"MLP {w.d}-{w.h}-{w.d} SiLU", "units": w.units, "T": w.T,
                                  "chunk": w.chunk, "flops_per_head_token": 2 * flops_per_head_token(w),
                                  "inputs": synth.describe(w)},
                       "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                                    "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                                    "peak_source": f"bf16_tflops ({which})",
                                    "kernel": "chunk_fwd_tc_mlp64<true> + mlp_backward_tc_kernel",
                                    "flops_per_launch": flops, "avg_launch_ms": avg, "sms_used": sms,
                                    "frac_of_sms_used": achieved / (peaks["bf16_tflops"] * sms / 148),
                                    "note": "one titans_mem_backward call: the forward with chunk-start "
                                            "checkpoints, then the backward pass; FLOPs counted as twice the "
                                            "forward's 18 d h per head-token"},
                       "gpu_launches": 2 * nb}
            del m
        out[key] = rec
        del toks, gates, state, dy
        torch.cuda.empty_cache()
    return out


def deep_arm(args, w, rank, world, local_rank):
    """--phase deep: one JSON line for the deep memory (every rank runs its own B*H units)."""
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    L = args.layers
    toks, gates, _ = _dev_inputs(w, dev)
    dst = {n: t.reshape(w.B, w.H, -1).to(dev) for n, t in synth.make_deep_state(w, L).items()}
    m = mem.Memory(w.d, w.h, w.chunk, w.dtype, w.B, w.H, layers=L)
    fn = lambda: m.forward_deep(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], dst)
    total, per = time_launches(fn, torch.cuda.current_stream(dev), args.steps, args.warmup)
    m.sync_status()
    ms = max_over_ranks(total / args.steps, dev, world)
    if rank != 0:
        return
    peaks, which = load_peaks()
    flops = deep_flops_per_head_token(w.d, w.h, L) * w.units * w.T
    achieved = flops / (statistics.mean(per) / 1e3) / 1e12
    print(json.dumps({
        "metric": "deep memory tokens/sec (update+retrieve) per B200; % bf16 tensor-core peak",
        "value": world * w.B * w.T / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded)",
        "config": {"workload": f"{w.name} deep L={L}", "layers": L, "units": w.units, "T": w.T, "chunk": w.chunk,
                   "path": KERNEL_NAMES.get(m.path(), m.path())},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "traffic": None, "peak_source": f"bf16_tflops ({which})",
                     "kernel": "chunk_fwd_tc_deep", "flops_per_launch": flops, "avg_launch_ms": statistics.mean(per)},
        "gpu_launches": args.steps}), flush=True)


def backward_arm(args, w, rank, world, local_rank):
    """--phase backward: one JSON line for titans_mem_backward (every rank runs its own B*H units)."""
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    toks, gates, state = _dev_inputs(w, dev)
    dy = torch.randn(toks["k"].shape, generator=torch.Generator().manual_seed(5)).to(toks["k"].dtype).to(dev)
    m = mem.Memory(w.d, w.h, w.chunk, w.dtype, w.B, w.H)
    fn = lambda: m.backward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state, dy)
    total, per = time_launches(fn, torch.cuda.current_stream(dev), args.steps, args.warmup)
    m.sync_status()
    ms = max_over_ranks(total / args.steps, dev, world)
    if rank != 0:
        return
    peaks, which = load_peaks()
    flops = 2 * flops_per_head_token(w) * w.units * w.T
    achieved = flops / (statistics.mean(per) / 1e3) / 1e12
    tc = m.backward_path() == mem.PATH_TC_BACKWARD
    kernel = "chunk_fwd_tc_mlp64<true> + mlp_backward_tc_kernel" if tc else "mlp_backward_kernel"
    print(json.dumps({
        "metric": "backward tokens/sec (gradients of every input) per B200; % bf16 tensor-core peak",
        "value": world * w.B * w.T / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded)",
        "config": {"workload": f"{w.name} backward", "units": w.units, "T": w.T, "chunk": w.chunk, "kernel": kernel},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "traffic": None, "peak_source": f"bf16_tflops ({which})",
                     "kernel": kernel, "flops_per_launch": flops, "avg_launch_ms": statistics.mean(per)},
        "gpu_launches": (2 if tc else 1) * args.steps}), flush=True)


def extra_results(args, dev):
    """The other workloads' numbers, nested in the one JSON line (rank 0 of a 1-GPU run):
    the 2048-unit decode step (HBM-bound), the 16-unit long stream (occupancy-limited: one
    CTA per unit) and the wide memory's prefill."""
    out = {}
    steps = max(3, min(args.steps, 20))
    wide = synth.WORKLOADS["mlp-d128-b4h8-t16k"]
    out["decode"] = decode_measure(wide, dev, steps, args.warmup)
    out["long_stream"] = forward_measure(synth.WORKLOADS["mlp-d64-b1h16-t1m"], dev, max(3, min(args.steps, 5)),
                                         args.warmup)
    out["wide_prefill"] = forward_measure(wide, dev, max(3, min(args.steps, 5)), args.warmup)
    out.update(extension_results(dev, max(3, min(args.steps, 10)), args.warmup))
    return out


def kernel_sha() -> str:
    """sha1 (first 12 hex digits) of the tensor-core kernel's source with `//` comments and
    blank lines removed, so that the stored DRAM counters stay matched to the code across
    comment-only edits and go stale on any code change."""
    import hashlib
    import re
    p = os.path.join(HERE, "titans_long_term_b200", "csrc", "chunk_tc_mlp64.cu")
    lines = [re.sub(r"\s*//.*$", "", ln).rstrip() for ln in open(p).read().splitlines()]
    code = "\n".join(ln for ln in lines if ln)
    return hashlib.sha1(code.encode()).hexdigest()[:12]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, choices=list(synth.WORKLOADS),
                    help="default: mlp-d64-b8h16-t4k for --phase forward, mlp-d128-b4h8-t16k for decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the nested decode / long-stream / wide-prefill results of a 1-GPU run")
    ap.add_argument("--phase", choices=["forward", "decode", "deep", "backward"], default="forward",
                    help="forward: the chunk-wise update + retrieve (default); decode: titans_mem_step; "
                         "deep: the deep memory's chunk-wise forward (--layers) on the tensor-core kernel; "
                         "backward: titans_mem_backward of the 2-layer memory")
    ap.add_argument("--layers", type=int, default=4, help="depth of the deep memory for --phase deep")
    ap.add_argument("--decode-b", type=int, default=0, help="decode batch (default: the workload's, 256)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload is None:
        args.workload = "mlp-d128-b4h8-t16k" if args.phase == "decode" else "mlp-d64-b8h16-t4k"
    w = synth.WORKLOADS[args.workload]
    if args.phase == "decode" and not (w.decode_B or args.decode_b):
        ap.error(f"workload {w.name} has no decode batch: pass --decode-b")
    if args.phase == "decode" and args.decode_b:
        import dataclasses
        w = dataclasses.replace(w, decode_B=args.decode_b)
    if args.impl == "reference":
        reference_arm(args, w, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.phase == "decode":
            decode_arm(args, w, rank, world, local_rank)
        elif args.phase == "deep":
            deep_arm(args, w, rank, world, local_rank)
        elif args.phase == "backward":
            backward_arm(args, w, rank, world, local_rank)
        else:
            our_arm(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
