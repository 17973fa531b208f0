"""Benchmark of the DualQuant BCD solver on B200: weight-elements x BCD-iterations per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl dq|reference]

A step is one full solve (RTN init, all BCD iterations, final codes and MSE) of
the workload's synthetic matrix, already resident in HBM.  L2 is flushed
(a 512 MB write, then a 512 MB read so that no dirty line is left to write
back) before every step, outside the timed events.  With N > 1
(torchrun) every rank solves its own replica of the workload (no data-path
collective: the solver does not shard) and the value is the sum over ranks
divided by the slowest rank's time.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
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

from calibration_free_weight_dualquant_b200 import binding, synth  # noqa: E402

DEFAULT_WORKLOAD = "nvfp4_g16_gateup_14336x4096"
METRIC = "weight-elems x BCD-iters/sec"
UNIT = "elem*iter/s"
L2_FLUSH_BYTES = 512 << 20


class L2Flush:
    """Empties L2 between timed steps: a 512 MB write (every line of L2 replaced), then a 512 MB read of a
    second buffer, so that the dirty lines of the write are written back here, untimed, instead of during
    the next timed step."""

    def __init__(self, dev):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.w.fill_(1)
        self.sink = self.r.amax()
KERNEL_SOURCES = ["calibration_free_weight_dualquant_b200/csrc/dq_solver.cu",
                  "calibration_free_weight_dualquant_b200/csrc/dq_device.cuh",
                  "calibration_free_weight_dualquant_b200/csrc/dq_fast.cuh",
                  "calibration_free_weight_dualquant_b200/csrc/dq_iter.cuh",
                  "calibration_free_weight_dualquant_b200/csrc/dq_internal.h",
                  "calibration_free_weight_dualquant_b200/csrc/dq_capi.cu"]


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


def profile_traffic(workload: str):
    """DRAM bytes per pass of k_iter (one BCD iteration) from the committed ncu summary, if it was taken of
    the current kernel source.  One k_iter launch runs all T passes, so the summary stores its launch's
    dram bytes divided by the passes it ran."""
    path = os.path.join(ROOT, "profiles", "k_iter_%s.json" % workload)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_hash") != kernel_hash():
        return None
    return d.get("dram_bytes_per_pass")


class ClockSampler:
    """SM clocks, power and clock-event (throttle) reasons sampled while the timed region runs.

    Samples come from NVML (nvidia-ml-py) every ~2 ms in a background thread, so even a timed
    region of a few tens of milliseconds carries many samples; where NVML is unavailable,
    nvidia-smi is polled every 100 ms instead.  Entering waits for the first sample."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h: nvmlClocksEventReason*)
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, device: torch.device):
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.uuid = None
        self.proc = None
        self.stop = None
        self.samples = []  # (sm_mhz, max_mhz, reasons set)
        self.lines = []
        self.armed = 0
        self.source = None

    def _nvml_loop(self, nvml, h):
        mx = float(nvml.nvmlDeviceGetMaxClockInfo(h, nvml.NVML_CLOCK_SM))
        get_reasons = getattr(nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nvml.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                sm = float(nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM))
                bits = int(get_reasons(h))
                self.samples.append((sm, mx, {k for k, v in self.REASON_BITS.items() if bits & v}))
            except Exception:
                pass
            time.sleep(0.002)

    def _reader(self):
        for line in self.proc.stdout:
            if line.strip():
                self.lines.append(line)

    def __enter__(self):
        import threading
        self.stop = threading.Event()
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            h = nvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else nvml.nvmlDeviceGetHandleByIndex(0)
            self.thread = threading.Thread(target=self._nvml_loop, args=(nvml, h), daemon=True)
            self.source = "nvml, 2 ms"
            self.thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 5.0:
                time.sleep(0.001)
            self.armed = len(self.samples)
            return self
        except Exception:
            self.source = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid or "0", "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.source = "nvidia-smi, 100 ms"
        self.thread = threading.Thread(target=self._reader, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
            time.sleep(0.01)
        self.armed = len(self.lines)  # samples taken before the timed region are dropped
        return self

    def __exit__(self, *a):
        if self.source and self.source.startswith("nvml"):
            self.stop.set()
            self.thread.join(timeout=5)
            self.samples = self.samples[self.armed:]
            return
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)
        self.lines = self.lines[self.armed:]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            self.samples.append((sm, mx, {nm for nm, v in zip(names, parts[5:9]) if v.lower().startswith("active")}))

    def summary(self) -> dict:
        sm = [x[0] for x in self.samples]
        reasons = set()
        for x in self.samples:
            reasons |= x[2]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": self.samples[-1][1] if self.samples else None, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return rank, world, local, dist
    return 0, 1, 0, None


def max_over_ranks(x: float, dist) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist):
    if dist is not None:
        dist.barrier()


def cpu_baseline(wl, budget_s: float = 12.0, W=None) -> dict:
    """The oracle, as it stands, on a bounded row sample of the workload on the host cores."""
    import oracle
    W = synth.make_weight(wl) if W is None else W
    cores = oracle.num_threads()
    rows = max(8, min(wl.rows, 64))
    while True:
        Win, wdt = synth.to_oracle_input(W[:rows].contiguous())
        t0 = time.perf_counter()
        oracle.solve(Win, wdt, wl.fmt, wl.group, wl.iters, wl.col_dtype)
        dt = time.perf_counter() - t0
        if dt > budget_s / 4 or rows >= wl.rows:
            break
        rows = min(wl.rows, int(rows * max(2.0, (budget_s / 4) / max(dt, 1e-3))))
    value = rows * wl.cols * wl.iters / dt
    # the same oracle on one core, on a smaller row sample (a few seconds)
    rows1 = max(8, min(rows, int(rows * (budget_s / 3) / max(dt * cores, 1e-3))))
    Win1, wdt1 = synth.to_oracle_input(W[:rows1].contiguous())
    oracle.set_num_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.solve(Win1, wdt1, wl.fmt, wl.group, wl.iters, wl.col_dtype)
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(cores)
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "first %d of %d rows x %d cols, all %d iterations, %.2f s" % (rows, wl.rows, wl.cols, wl.iters,
                                                                                  dt),
            "single_core": {"value": rows1 * wl.cols * wl.iters / dt1, "cores": 1,
                            "sample": "first %d rows, %.2f s" % (rows1, dt1)}}


def run_reference(args, wl, rank, world, dist, set_name=None):
    """Reference arm: the CPU oracle on the host cores, one bounded row sample per step (for the
    Llama set: rows of its layer-0 gate matrix, drawn with the set's generator)."""
    if rank != 0:
        return
    import oracle
    W = synth.make_weight_device(wl, "cpu") if set_name else synth.make_weight(wl)
    rows = max(8, min(wl.rows, args.ref_rows))
    Win, wdt = synth.to_oracle_input(W[:rows].contiguous())
    t0 = time.perf_counter()
    oracle.solve(Win, wdt, wl.fmt, wl.group, wl.iters, wl.col_dtype)
    t_one = time.perf_counter() - t0
    budget_s = 90.0  # the whole timed run stays within a couple of minutes
    if args.steps * t_one > budget_s:
        rows = max(8, int(rows * budget_s / (args.steps * t_one)))
        Win, wdt = synth.to_oracle_input(W[:rows].contiguous())
    for _ in range(args.warmup):
        oracle.solve(Win, wdt, wl.fmt, wl.group, wl.iters, wl.col_dtype)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.solve(Win, wdt, wl.fmt, wl.group, wl.iters, wl.col_dtype)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = rows * wl.cols * wl.iters * args.steps / tot
    cores = oracle.num_threads()
    sample = "first %d of %d rows x %d cols, all %d iterations per step" % (rows, wl.rows, wl.cols, wl.iters)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": set_config(set_name, world) if set_name else config_of(wl, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores,
                                                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(wl, world) -> dict:
    return {"workload": wl.name, "rows": wl.rows, "cols": wl.cols, "format": wl.fmt, "group": wl.group,
            "iters": wl.iters, "w_dtype": wl.wdtype, "col_dtype": wl.col_dtype,
            "l2": "flushed before each step (512 MB write, then 512 MB read: no dirty line left; untimed)", "parallelism": "replicas x%d" % world}


# beta-folded activation quantization of a prefill batch: (format, group, tokens, in-features)
ACT_WORKLOADS = {
    "act_nvfp4_8192x4096": ("nvfp4", 16, 8192, 4096),
    "act_mxint4_8192x14336": ("mxint4", 32, 8192, 14336),
    "act_int4_8192x4096": ("int4", 64, 8192, 4096),
}


def run_act(args, name, rank, world, local, dist):
    """dq_act_quant on a synthetic prefill batch (X [tokens, cols] bf16, b [cols] bf16); a step is one call.
    The oracle arm (--impl reference) times oracle.act_quant on a row sample."""
    fmt, g, T, K = ACT_WORKLOADS[name]
    cfg = {"workload": name, "tokens": T, "cols": K, "format": fmt, "group": g, "x_dtype": "bf16",
           "col_dtype": "bf16", "l2": "flushed before each step (512 MB write, then 512 MB read: no dirty line left; untimed)",
           "parallelism": "replicas x%d" % world}
    metric, unit = "activation elems/sec", "elem/s"
    X = synth.make_activations(T, K, seed=77 + rank)
    b = synth.make_col_scales(K, seed=78)
    if args.impl == "reference":
        if rank != 0:
            return
        import oracle
        rows = max(1, min(T, 256))
        Xin, xdt = synth.to_oracle_input(X[:rows].contiguous())
        bv = b.to(torch.float64).numpy()
        for _ in range(args.warmup):
            oracle.act_quant(Xin, xdt, bv, fmt, g)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle.act_quant(Xin, xdt, bv, fmt, g)
        dt = time.perf_counter() - t0
        value = rows * K * args.steps / dt
        line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": cfg,
                "cpu_baseline": {"value": value, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
                                 "sample": "first %d of %d tokens per step" % (rows, T)},
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    binding.load_library()
    Xd, bd = X.to(dev), b.to(dev)
    out = binding.dq_act_quant(Xd, bd, fmt, g)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def timed(steps):
        ts = []
        for _ in range(steps):
            flush()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            binding.dq_act_quant(Xd, bd, fmt, g, out=out, workspace=out["workspace"], stream=stream, check=False)
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return ts

    timed(args.warmup)
    barrier(dist)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        ts = timed(args.steps)
    barrier(dist)
    total_ms = max_over_ranks(sum(ts), dist)
    med_ms = max_over_ranks(statistics.median(ts), dist)
    if rank != 0:
        return
    asz = 2 if fmt == "int4" else 1
    alg = T * K * 2 + T * K // 2 + T * (K // g) * asz + K * 2  # X read once, codes and scales written
    peaks = measured_peaks()
    achieved = alg / (med_ms * 1e-3) / 1e9
    line = {"metric": metric, "value": world * T * K * args.steps / (total_ms * 1e-3), "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": cfg,
            "roofline": {"bound": "hbm", "kernel": "k_act_nv" if fmt == "nvfp4" else "k_act", "achieved": achieved,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": None, "algorithmic_bytes_per_launch": alg, "peak_source": peaks["source"],
                         "note": "one call = one launch (NVFP4: amax pass, grid barrier, quantization pass); algorithmic bytes count one read of X"},
            "e2e": None, "gpu_launches": (2 if fmt == "nvfp4" else 1) * args.steps, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def set_config(name, world) -> dict:
    fmt = synth.LLAMA_SETS[name]
    wl = synth.llama_set(fmt)[0]
    return {"workload": name, "matrices": len(synth.llama_set(fmt)), "elements": synth.llama_set_elements(),
            "format": fmt, "group": wl.group, "iters": wl.iters, "w_dtype": wl.wdtype, "col_dtype": wl.col_dtype,
            "l2": "inputs (14 GB) far larger than L2", "parallelism": "replicas x%d" % world}


def algorithmic_bytes_per_iter(wl) -> int:
    wsz = 4 if wl.wdtype == "f32" else 2
    asz = 2 if wl.fmt == "int4" else 1
    nb = wl.cols // wl.group
    return wl.rows * wl.cols * wsz + 2 * wl.rows * nb * asz + 2 * wl.cols * 2


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(synth.WORKLOADS) + sorted(synth.LLAMA_SETS) + sorted(ACT_WORKLOADS))
    ap.add_argument("--impl", default="dq", choices=["dq", "reference"])
    ap.add_argument("--ref-rows", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--rows", type=int, help="override the workload's rows (profiling cases)")
    ap.add_argument("--cols", type=int, help="override the workload's cols (profiling cases)")
    ap.add_argument("--iters", type=int, help="override the workload's BCD iterations")
    args = ap.parse_args()
    if args.workload in ACT_WORKLOADS:
        rank, world, local, dist = dist_setup(args.gpus)
        try:
            run_act(args, args.workload, rank, world, local, dist)
        finally:
            if dist is not None:
                dist.destroy_process_group()
        return
    if args.workload in synth.LLAMA_SETS:
        rank, world, local, dist = dist_setup(args.gpus)
        try:
            if args.impl == "reference":
                run_reference(args, synth.llama_set(synth.LLAMA_SETS[args.workload])[4], rank, world, dist,
                              set_name=args.workload)
            else:
                run_dq_set(args, args.workload, rank, world, local, dist)
        finally:
            if dist is not None:
                dist.destroy_process_group()
        return
    wl = synth.WORKLOADS[args.workload]
    if args.rows or args.cols or args.iters:
        import dataclasses
        rows = args.rows or wl.rows
        cols = args.cols or wl.cols
        iters = args.iters or wl.iters
        wl = dataclasses.replace(wl, name="%s@%dx%d_T%d" % (wl.name, rows, cols, iters), rows=rows, cols=cols,
                                 iters=iters)
    rank, world, local, dist = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, wl, rank, world, dist)
            return
        run_dq(args, wl, rank, world, local, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


def run_dq(args, wl, rank, world, local, dist):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    binding.load_library()
    W = synth.make_weight(wl, seed=wl.seed + 7919 * rank)
    Wd = W.to(dev)
    T = wl.iters
    out = binding.alloc_outputs(wl.rows, wl.cols, wl.fmt, wl.group, wl.col_dtype, T, dev)
    ws = torch.empty(binding.workspace_bytes(wl.rows, wl.cols, wl.fmt, wl.group), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def solve(iters, o=out, full=False):
        binding.dq_solve(Wd, wl.fmt, wl.group, iters, wl.col_dtype, out=o, workspace=ws, stream=stream, check=False,
                         full_passes=full)

    def timed(iters, steps, o=out, full=False):
        ts = []
        for _ in range(steps):
            flush()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            solve(iters, o, full)
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return ts

    for _ in range(args.warmup):
        flush()
        solve(T)
    torch.cuda.synchronize()
    st = binding.load_library().dq_sync_status(ws.data_ptr(), stream.cuda_stream)
    if st != 0:
        raise binding.DQError(st, "bench warm-up")

    barrier(dist)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        step_ms = timed(T, args.steps)
    torch.cuda.synchronize()
    barrier(dist)
    total_ms = max_over_ranks(sum(step_ms), dist)
    exact_paths = binding.diagnostics(ws, stream)
    n_active = binding.active_block_columns(ws, stream)

    # steady-state iteration time of the dominant kernel (k_iter): (t(T) - t(0)) / T, median of runs
    out0 = binding.alloc_outputs(wl.rows, wl.cols, wl.fmt, wl.group, wl.col_dtype, 0, dev)
    t0s = timed(0, max(3, args.steps), out0)
    tTs = step_ms
    iter_ms = (statistics.median(tTs) - statistics.median(t0s)) / T
    iter_ms = max_over_ranks(iter_ms, dist)
    # ablation: every iteration over every block-column (no skipping of block-columns at a fixed point)
    full_ms = None
    if T > 0:
        solve(T, full=True)
        full_ms = (statistics.median(timed(T, max(3, min(args.steps, 5)), full=True)) - statistics.median(t0s)) / T
        full_ms = max_over_ranks(full_ms, dist)

    e2e_line = None
    if not args.no_e2e:
        e2e_line = run_e2e(args, wl, W, T, dev, stream, flush, dist, world)
    if rank != 0:
        return
    elems = wl.rows * wl.cols
    value = world * elems * T * args.steps / (total_ms * 1e-3)
    peaks = measured_peaks()
    alg = algorithmic_bytes_per_iter(wl)
    achieved = alg / (iter_ms * 1e-3) / 1e9
    traffic = profile_traffic(wl.name)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32+f64", "data": "synthetic",
        "config": config_of(wl, world),
        "final_mse": float(out["mse"][-1].item()),
        "ms_per_iter": iter_ms,
        "roofline": {"bound": "hbm", "kernel": "k_iter", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "algorithmic_bytes_per_pass": alg, "passes_per_launch": T, "peak_source": peaks["source"],
                     "note": "achieved = algorithmic bytes of one BCD iteration (W read once, block scales read "
                             "and written, column scales) / measured time per iteration; block-columns at a "
                             "fixed point are skipped and not read, so traffic per iteration is below that"},
        "work": {"block_columns_processed": n_active, "block_columns_x_iters": T * (wl.cols // wl.group),
                 "active_fraction": n_active / max(1, T * (wl.cols // wl.group))},
        "ablation_full_passes": None if full_ms is None else {
            "ms_per_iter": full_ms, "achieved_gbs": alg / (full_ms * 1e-3) / 1e9,
            "frac": alg / (full_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "note": "same solve with dq_options.full_passes: every iteration processes every block-column"},
        "e2e": e2e_line,
        # per solve: k_stats, k_init, one k_iter for all T iterations, the final k_iter pass
        "gpu_launches": args.steps * (4 if T > 0 else 3),
        "exact_paths_last_step": exact_paths,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)


def run_dq_set(args, name, rank, world, local, dist):
    """The whole 224-matrix Llama-3.1-8B linear set per step, queued on one stream by dq_solve_batched."""
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    binding.load_library()
    fmt = synth.LLAMA_SETS[name]
    wls = synth.llama_set(fmt)
    T, g, cd = wls[0].iters, wls[0].group, wls[0].col_dtype
    Ws = [synth.make_weight_device(wl, dev, seed=wl.seed + 7919 * rank) for wl in wls]
    outs = [binding.alloc_outputs(wl.rows, wl.cols, fmt, g, cd, T, dev) for wl in wls]
    outs0 = [binding.alloc_outputs(wl.rows, wl.cols, fmt, g, cd, 0, dev) for wl in wls]
    ws = torch.empty(max(binding.workspace_bytes(wl.rows, wl.cols, fmt, g) for wl in wls), dtype=torch.uint8,
                     device=dev)
    status = torch.zeros(len(wls), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(iters, steps, o):
        ts = []
        for _ in range(steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            binding.dq_solve_batched(Ws, fmt, g, iters, cd, outs=o, workspace=ws, status=status, stream=stream,
                                     check=False)
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return ts

    timed(T, args.warmup, outs)
    torch.cuda.synchronize()
    if int(status.abs().sum()) != 0:
        raise binding.DQError(int(status.max()), "bench warm-up (Llama set)")
    barrier(dist)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        step_ms = timed(T, args.steps, outs)
    torch.cuda.synchronize()
    barrier(dist)
    total_ms = max_over_ranks(sum(step_ms), dist)
    t0s = timed(0, max(3, min(args.steps, 10)), outs0)
    iter_ms = max_over_ranks((statistics.median(step_ms) - statistics.median(t0s)) / T, dist)
    if rank != 0:
        return
    elems = synth.llama_set_elements()
    value = world * elems * T * args.steps / (total_ms * 1e-3)
    peaks = measured_peaks()
    alg = sum(algorithmic_bytes_per_iter(wl) for wl in wls)
    achieved = alg / (iter_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32+f64", "data": "synthetic",
        "config": set_config(name, world),
        "final_mse_layer0_q": float(outs[0]["mse"][-1].item()),
        "ms_per_iter": iter_ms,
        "roofline": {"bound": "hbm", "kernel": "k_iter", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "algorithmic_bytes_per_pass": alg, "passes_per_launch": T, "peak_source": peaks["source"],
                     "note": "per iteration of the whole set (224 launches of k_iter)"},
        "e2e": None,
        "gpu_launches": args.steps * len(wls) * (4 if T > 0 else 3),
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(wls[4], W=synth.make_weight_device(wls[4], "cpu"))
        cb["extrapolated_full_set_s"] = elems * T / cb["value"]
        cb["sample"] += "; the whole set's CPU time is extrapolated by element count"
        line["cpu_baseline"] = cb
    print(json.dumps(line), flush=True)


def run_e2e(args, wl, W, T, dev, stream, flush, dist, world):
    """Same metric through the public host-buffer API: pinned W in, outputs back, copies timed."""
    Wh = W.pin_memory()
    host_out = binding.alloc_outputs(wl.rows, wl.cols, wl.fmt, wl.group, wl.col_dtype, T, "cpu")
    for k in host_out:
        host_out[k] = host_out[k].pin_memory()
    dws = torch.empty(binding.host_workspace_bytes(wl.rows, wl.cols, W.dtype, wl.fmt, wl.group, T),
                      dtype=torch.uint8, device=dev)
    binding.solve(Wh, wl.fmt, wl.group, T, wl.col_dtype, out=host_out, device_workspace=dws)
    e2e_ms = []
    for _ in range(max(3, args.steps // 2)):
        flush()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        binding.solve(Wh, wl.fmt, wl.group, T, wl.col_dtype, out=host_out, device_workspace=dws)
        e1.record(stream)
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    e2e_total = max_over_ranks(sum(e2e_ms), dist)
    nb = binding.output_nbytes(wl.rows, wl.cols, wl.fmt, wl.group, wl.col_dtype)
    h2d = W.numel() * W.element_size()
    d2h = nb["codes"] + nb["block_scales"] + nb["col_scales"] + nb["tensor_scale"] + 8 * (T + 1)
    e2e_value = world * wl.rows * wl.cols * T * len(e2e_ms) / (e2e_total * 1e-3)
    return {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


if __name__ == "__main__":
    main()
