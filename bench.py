#!/usr/bin/env python3
"""Benchmark of the fused add + RMSNorm + dynamic-quant operator on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload c2] [--no-cpu-baseline] [--no-workloads]

A step is one call of the operator (arnq_run) over one
batch of the workload: by default the 8192 x 4096 bf16 configuration
(x1 ~ N(0,1), x2 ~ N(0,0.5), gamma, beta, smooth1, outputMask [True, False],
INT8).  Inputs are seeded synthetic data resident in HBM before timing.  The
timed region is exactly K steps between a barrier + synchronize on both
sides, timed with CUDA events on the launching stream; three buffer sets are
rotated so that every step reads inputs that are not in L2 (each set is
larger than L2 by itself).  `value` is whole-job HBM GB/s of algorithmic
bytes; with N GPUs (launched by torchrun, one process per GPU) every rank
processes its own batch of the same size (weak scaling; rows are independent,
so there is no data-path collective) and the time is the maximum over ranks.

Also printed, on the same JSON line: rows/s, the roofline of the kernel
(achieved GB/s from the mean per-launch CUDA-event duration against the
measured copy bandwidth, and the DRAM traffic per launch recorded by ncu for
this kernel source), five more timed regions of K calls (the figure's
spread), the same K calls with the opt-in early parameter loads, the
end-to-end figure through the public call with host buffers (every step's
H2D copies, the call and the D2H copy of its outputs inside the timed region;
two buffer sets so that one step's copy-in overlaps the previous step's
copy-out), SM clocks sampled by NVML during the timed region, and the CPU
oracle's throughput on a bounded sample (rank 0, one GPU only).  The
`workloads` object carries the other configurations measured in the same
run: the large ones as device time per call of calls back to back (median of
five regions, with the early-parameter figure), the no-add operator on the
8192 x 4096 inputs, and the small, latency-bound ones as device time per call
from a CUDA graph of back-to-back calls (L2-cold and L2-hot) and as host time
per call.  The timed loops call arnq_run through ctypes with arguments
marshalled once, and each timed region is queued behind a short device-side
delay, so that the host's launches are not what is timed.

--impl reference times the CPU oracle (the only other implementation of the
operator; there is no runnable reference library) on the host cores.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused add-RMSNorm-dynquant HBM GB/s and rows/s on 1 B200 (% of HBM peak)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
DEFAULT_WORKLOAD = "c2"


# ---------------------------------------------------------------- byte accounting

def algorithmic_bytes(rows, n, dtype, qdtype, has_beta, has_s1, has_s2, on1, on2,
                      has_x2=True, x_out=True):
    """Bytes the operator must move: x1, x2 read and xOut written (2 B/element
    each), codes (1 or 1/2 B/element) and one fp32 scale per row for every
    produced output, and each parameter vector (gamma, beta, smooth1, smooth2)
    read once per call."""
    esz = 2
    per_row = n * esz * (2 if has_x2 else 1)
    if x_out and has_x2:
        per_row += n * esz
    code = n if qdtype == "int8" else n // 2
    per_row += (code + 4) * (int(on1) + int(on2))
    params = n * esz * (1 + int(has_beta) + int(has_s1) + int(has_s2))
    return rows * per_row + params


def workload_bytes(w, on1, on2):
    return algorithmic_bytes(w.rows, w.n, w.dtype, w.qdtype, w.beta is not None,
                             w.smooth1 is not None, w.smooth2 is not None, on1, on2)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    """Hash of the device code (the kernel template and its instantiation table)."""
    h = hashlib.sha256()
    for f in ("int4_quant_b200/csrc/arnq_kernels.cuh", "int4_quant_b200/csrc/arnq_table.h"):
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name, plan=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source with the same launch plan; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(workload_name)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    if plan is not None and e.get("plan") is not None and e["plan"] != plan:
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks (NVML)

class ClockSampler:
    """Samples SM clock and throttle reasons with NVML every `period` seconds."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.002):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in self.REASONS.items():
                    if r & bit and k != "gpu_idle":
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU oracle timing

def time_oracle(w, on1, on2, target_cpu_s=12.0, threads=None):
    """Times the (unmodified, single-threaded) oracle over row chunks of the
    workload run concurrently on `threads` host threads (ctypes releases the
    GIL).  Returns (GB/s, rows/s, threads, sample description)."""
    import oracle
    oracle.build()
    threads = threads or os.cpu_count() or 1
    chunk = 64

    def run_rows(r0, r1):
        oracle.add_rms_norm_dynamic_quant_v2(
            w.x1[r0:r1], w.x2[r0:r1], w.gamma, w.beta, w.smooth1, w.smooth2, eps=w.eps,
            mask=w.mask, qdtype=w.qdtype, dtype=w.dtype)

    t0 = time.perf_counter()
    run_rows(0, chunk)
    per_row = (time.perf_counter() - t0) / chunk
    total_rows = int(max(threads * chunk, min(target_cpu_s / per_row, 64 * w.rows)))
    jobs = []
    r = 0
    while r < total_rows:
        a = r % w.rows
        b = min(a + chunk, w.rows)
        jobs.append((a, b))
        r += b - a
    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda ab: run_rows(*ab), jobs))
    dt = time.perf_counter() - t0
    rows_done = sum(b - a for a, b in jobs)
    nbytes = workload_bytes(w, on1, on2) * rows_done / w.rows
    sample = (f"{rows_done} rows of the {w.rows}x{w.n} workload (chunks of {chunk} rows, "
              f"cycled) on {threads} host threads")
    return nbytes / dt / 1e9, rows_done / dt, threads, sample


# ---------------------------------------------------------------- reference arm

def run_reference(args, w, on1, on2):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    # size each step so that the whole run stays within about a minute
    t0 = time.perf_counter()
    oracle.add_rms_norm_dynamic_quant_v2(w.x1[:32], w.x2[:32], w.gamma, w.beta, w.smooth1,
                                         w.smooth2, eps=w.eps, mask=w.mask, qdtype=w.qdtype,
                                         dtype=w.dtype)
    per_row = (time.perf_counter() - t0) / 32
    budget = 60.0 / max(1, args.steps + args.warmup)
    rows = int(max(threads, min(w.rows, budget * threads / per_row)))
    bounds = np.linspace(0, rows, threads + 1).astype(int)

    def part(k):
        a, b = bounds[k], bounds[k + 1]
        if b > a:
            oracle.add_rms_norm_dynamic_quant_v2(
                w.x1[a:b], w.x2[a:b], w.gamma, w.beta, w.smooth1, w.smooth2, eps=w.eps,
                mask=w.mask, qdtype=w.qdtype, dtype=w.dtype)

    pool = cf.ThreadPoolExecutor(max_workers=threads)

    def step(i):  # the first `rows` rows of the workload, split over the host threads
        list(pool.map(part, range(threads)))

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    pool.shutdown()
    nbytes = workload_bytes(w, on1, on2) * rows / w.rows
    value = nbytes * args.steps / dt / 1e9
    sample = f"{rows} rows of the {w.rows}x{w.n} workload per step on {threads} host threads"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "rows_per_step": rows, "n": w.n, "io_dtype": w.dtype,
                   "qdtype": w.qdtype},
        "rows_per_s": rows * args.steps / dt,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm

def launches_per_call(plan):
    """Kernels one arnq_run call launches: the row kernel alone, whether a row
    has one CTA or a cluster (each row is settled inside the kernel)."""
    return 1


def max_over_ranks(value_ms, dist, device):
    """The slowest rank's time: every rank passes its own and gets the max."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value_ms)
    import torch
    t = torch.tensor([float(value_ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_step, steps, world, total_ms):
    """Whole-job throughput: every rank moves bytes_per_step per step (replicas)."""
    return bytes_per_step * steps * world / (total_ms / 1e3) / 1e9


# Device-side delay queued in front of a timed region (clock cycles, about
# 2 ms at 1.9 GHz): the host enqueues the timed calls while the GPU waits, so
# the first event does not also time the host's launch of the first calls.
HOST_AHEAD_CYCLES = 4_000_000


def hold_device(torch):
    """Queues HOST_AHEAD_CYCLES of device-side delay on the current stream
    (a torch kernel outside the timed region: it runs before the first event)."""
    torch.cuda._sleep(HOST_AHEAD_CYCLES)


def outputs_of(w):
    """(y1 produced, y2 produced) for a workload, by the outputMask rules."""
    on1 = w.mask is None or w.mask[0]
    on2 = (w.mask is not None and w.mask[1]) or (w.mask is None and w.smooth1 is not None
                                                 and w.smooth2 is not None)
    return on1, on2


def sets_for(w, on1, on2, min_bytes=None, cap=2048):
    """Buffer sets to rotate so that a call's inputs have left L2 before they are
    read again: at least 3, and enough that the sets together move min_bytes."""
    if min_bytes is None:
        return 3
    per = workload_bytes(w, on1, on2)
    return int(min(cap, max(3, -(-min_bytes // per))))


class DeviceRun:
    """One workload resident on the device: `nsets` rotated buffer sets, the
    parameters, a zeroed workspace, and the arnq_run arguments of every set
    marshalled once (ctypes), so that a timed loop spends its host time in
    the library's own launch path."""

    def __init__(self, w, dev, stream, nsets=3):
        import ctypes
        import torch
        from int4_quant_b200 import _abi as A
        import int4_quant_b200 as q
        self.w, self.dev, self.stream, self.A = w, dev, stream, A
        self.on1, self.on2 = outputs_of(w)
        TDT = {"bf16": torch.bfloat16, "fp16": torch.float16}[w.dtype]
        self.dt_code = A.ARNQ_BF16 if w.dtype == "bf16" else A.ARNQ_FP16
        self.q_code = A.ARNQ_INT8 if w.qdtype == "int8" else A.ARNQ_INT4
        self.mc = q.mask_code(w.mask)

        def to_dev(bits):
            if bits is None:
                return None
            t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
            return t.to(dev).view(TDT)

        cb = w.n if w.qdtype == "int8" else w.n // 2
        self.params = [to_dev(a) for a in (w.gamma, w.beta, w.smooth1, w.smooth2)]
        x1d, x2d = to_dev(w.x1), to_dev(w.x2)
        self.sets = []
        for i in range(nsets):
            self.sets.append(dict(
                x1=x1d if i == 0 else x1d.clone(), x2=x2d if i == 0 else x2d.clone(),
                y1=torch.empty((w.rows, cb), dtype=torch.uint8, device=dev) if self.on1 else None,
                s1=torch.empty((w.rows,), dtype=torch.float32, device=dev) if self.on1 else None,
                y2=torch.empty((w.rows, cb), dtype=torch.uint8, device=dev) if self.on2 else None,
                s2=torch.empty((w.rows,), dtype=torch.float32, device=dev) if self.on2 else None,
                xo=torch.empty((w.rows, w.n), dtype=TDT, device=dev)))
        st, self.ws_bytes = A.arnq_workspace_size(w.rows, w.n, self.dt_code, self.q_code, self.mc,
                                                  w.smooth1 is not None, w.smooth2 is not None)
        if st != A.ARNQ_OK:
            raise A.ArnqError(st, "arnq_workspace_size")
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.fn = A.lib().arnq_run
        self.args = [self._args(s, stream) for s in self.sets]
        st, self.plan = A.arnq_make_plan(self.sets[0]["x1"], self.sets[0]["x2"], *self.params,
                                         w.rows, w.n, self.dt_code, self.mc, self.q_code,
                                         self.sets[0]["y1"], self.sets[0]["y2"],
                                         self.sets[0]["xo"])
        if st != A.ARNQ_OK:
            raise A.ArnqError(st, "arnq_make_plan")
        self.bytes = workload_bytes(w, self.on1, self.on2)

    def _args(self, s, stream):
        import ctypes
        A = self.A
        p = A._ptr
        return (p(s["x1"]), p(s["x2"]), *[p(t) for t in self.params], self.w.rows, self.w.n,
                self.dt_code, ctypes.c_float(self.w.eps), self.mc, self.q_code, p(s["y1"]),
                p(s["s1"]), p(s["y2"]), p(s["s2"]), p(s["xo"]), p(self.ws), self.ws_bytes,
                A._stream(stream))

    def with_plan(self, **fields):
        """The same buffers, launched through arnq_run_planned with a plan whose
        given fields are set (the library chooses the others)."""
        import copy
        import ctypes
        other = copy.copy(self)
        pl = self.A.arnq_plan()
        for k, v in fields.items():
            setattr(pl, k, v)
        other.plan_request = pl  # the struct the marshalled pointer refers to
        other.fn = self.A.lib().arnq_run_planned
        other.args = [tuple(a) + (ctypes.addressof(pl),) for a in self.args]
        return other

    def launch(self, i, args=None):
        st = self.fn(*(args or self.args)[i % len(self.sets)])
        if st:
            raise self.A.ArnqError(st, "arnq_run")

    def status(self):
        """(code, row, counters) of the workspace status block (synchronizes)."""
        h = self.ws[:32].cpu().numpy().view(np.int32)
        return int(h[0]), int(h[2:4].view(np.int64)[0]), [int(v) for v in h[4:7]]

    def check_status(self):
        code, row, ctr = self.status()
        if code != 0 or any(ctr):
            raise RuntimeError(f"{self.w.name}: device status {code} (row {row}), counters {ctr}")

    def timed(self, steps, warmup):
        """Mean device time of one call over `steps` calls back to back (one CUDA
        event pair on the launching stream: the calls are programmatic
        dependents of one another, and an event between two would separate
        them), after `warmup` calls."""
        import torch
        for i in range(warmup):
            self.launch(i)
        torch.cuda.synchronize(self.dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        hold_device(torch)
        e0.record(self.stream)
        for i in range(steps):
            self.launch(i)
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return e0.elapsed_time(e1) / steps

    def graph_timed(self, calls, replays=20):
        """Device time of one call when `calls` calls (rotating the buffer sets)
        run back to back from a CUDA graph: no host enqueue in the way, as a
        decode loop captured in a graph sees it.  Returns the median over
        replays of (replay time / calls) in ms."""
        import torch
        side = torch.cuda.Stream(self.dev)
        args = [self._args(s, side) for s in self.sets]
        side.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(side):
            for i in range(3):
                self.launch(i, args)
        torch.cuda.synchronize(self.dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(calls):
                self.launch(i, args)
        g.replay()
        torch.cuda.synchronize(self.dev)
        out = []
        for _ in range(replays):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            g.replay()
            e1.record(self.stream)
            torch.cuda.synchronize(self.dev)
            out.append(e0.elapsed_time(e1) / calls)
        del g
        return statistics.median(out)

    def host_us(self, calls=2000):
        """Host time of one call of arnq_run (argument checks, plan lookup and
        launch), from Python through ctypes, calls issued back to back."""
        import torch
        for i in range(10):
            self.launch(i)
        t0 = time.perf_counter()
        for i in range(calls):
            self.launch(i)
        t1 = time.perf_counter()
        torch.cuda.synchronize(self.dev)
        return (t1 - t0) / calls * 1e6


def time_no_add(w, dev, stream, peak, calls=200, regions=5):
    """The no-add operator (arnq_rms_norm_dynamic_quant: x normalised as given,
    one output, no xOut) on workload w's x1, gamma, beta and smooth1: device
    time per call of `calls` calls back to back on 3 rotated L2-cold sets."""
    import ctypes
    import torch
    from int4_quant_b200 import _abi as A
    TDT = {"bf16": torch.bfloat16, "fp16": torch.float16}[w.dtype]
    dt = A.ARNQ_BF16 if w.dtype == "bf16" else A.ARNQ_FP16
    qd = A.ARNQ_INT8 if w.qdtype == "int8" else A.ARNQ_INT4

    def to_dev(bits):
        if bits is None:
            return None
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(TDT)

    cb = w.n if w.qdtype == "int8" else w.n // 2
    x0 = to_dev(w.x1)
    g, b, s1 = to_dev(w.gamma), to_dev(w.beta), to_dev(w.smooth1)
    sets = [dict(x=x0 if i == 0 else x0.clone(),
                 y=torch.empty((w.rows, cb), dtype=torch.uint8, device=dev),
                 s=torch.empty((w.rows,), dtype=torch.float32, device=dev)) for i in range(3)]
    st, nb = A.arnq_workspace_size(w.rows, w.n, dt, qd, A.ARNQ_MASK_ABSENT, s1 is not None, False)
    if st != A.ARNQ_OK:
        raise A.ArnqError(st, "arnq_workspace_size")
    ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
    fn = A.lib().arnq_rms_norm_dynamic_quant
    P = A._ptr
    args = [(P(t["x"]), P(g), P(b), P(s1), w.rows, w.n, dt, ctypes.c_float(w.eps), qd, P(t["y"]),
             P(t["s"]), P(ws), nb, A._stream(stream)) for t in sets]
    out = []
    for _ in range(regions):
        for i in range(20):
            fn(*args[i % 3])
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        hold_device(torch)
        e0.record(stream)
        for i in range(calls):
            if fn(*args[i % 3]):
                raise RuntimeError("arnq_rms_norm_dynamic_quant failed")
        e1.record(stream)
        torch.cuda.synchronize(dev)
        out.append(e0.elapsed_time(e1) / calls)
    if int(ws[:4].view(torch.int32).item()) != 0:
        raise RuntimeError("no-add run: device status set")
    ms = statistics.median(out)
    nbytes = algorithmic_bytes(w.rows, w.n, w.dtype, w.qdtype, w.beta is not None,
                               w.smooth1 is not None, False, True, False, has_x2=False,
                               x_out=False)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"us_per_call": ms * 1e3, "us_per_call_min_max": [min(out) * 1e3, max(out) * 1e3],
            "gbs": gbs, "frac": gbs / peak, "bytes_per_call": nbytes,
            "rows_per_s": w.rows / (ms / 1e3),
            "timing": f"{calls} calls back to back, 3 sets; median of {regions} timed regions",
            "workload": "rms_norm_dynquant_" + w.name.split("add_rmsnorm_dynquant_", 1)[-1]}


def workload_entry(run, ms, peak, how):
    """One line of the `workloads` object: a call's time, throughput, roofline."""
    gbs = run.bytes / (ms / 1e3) / 1e9
    return {"us_per_call": ms * 1e3, "gbs": gbs, "frac": gbs / peak,
            "rows_per_s": run.w.rows / (ms / 1e3), "bytes_per_call": run.bytes,
            "plan": run.plan.as_dict(), "timing": how}


SMALL = ("c1", "c5a", "c5b", "c5c")     # latency-bound: device time per call from a graph
LARGE = ("c2", "c3", "c4", "c5d")       # the >= 80 % roofline class


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads' lines (the `workloads` object)")
    ap.add_argument("--sets", type=int, default=3, help="rotated buffer sets")
    ap.add_argument("--repeats", type=int, default=5,
                    help="further timed regions of K steps after the first (spread only)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from int4_quant_b200 import workloads as wl
    w = wl.CONFIGS[args.workload]()
    on1, on2 = outputs_of(w)
    if args.impl == "reference":
        return run_reference(args, w, on1, on2)

    import torch
    import torch.distributed as dist
    import int4_quant_b200 as q
    from int4_quant_b200 import _abi as A

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if args.gpus > 1:
            sys.exit("for --gpus N > 1 launch with torch.distributed.run (one process per GPU)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        # every rank runs its own batch of the full workload (weak scaling)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    A.lib()
    stream = torch.cuda.current_stream(dev)
    run = DeviceRun(w, dev, stream, nsets=args.sets)
    plan = run.plan

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---- warm-up
    for i in range(args.warmup):
        run.launch(i)
    barrier()

    # ---- timed region: exactly K steps, back to back on the stream (one event
    # pair around all of them: an event between two calls would separate the
    # programmatically dependent launches and time the host's enqueue rate)
    K = args.steps
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local, period=0.0005)
    clocks.start()
    barrier()
    hold_device(torch)
    ev0.record(stream)
    for i in range(K):
        run.launch(i)
    ev1.record(stream)
    barrier()
    clocks.stop()
    total_ms = ev0.elapsed_time(ev1)
    # the same K steps timed again (spread of the figure; `value` is the first)
    repeats = []
    for _ in range(args.repeats):
        for i in range(args.warmup):
            run.launch(i)
        barrier()
        r0 = torch.cuda.Event(enable_timing=True)
        r1 = torch.cuda.Event(enable_timing=True)
        hold_device(torch)
        r0.record(stream)
        for i in range(K):
            run.launch(i)
        r1.record(stream)
        barrier()
        repeats.append(r0.elapsed_time(r1) / K)
    run.check_status()
    # the same K steps with the parameters promised constant (plan
    # early_params; an opt-in, reported beside the default path's figure)
    early_ms = []
    er = run.with_plan(early_params=1)
    for _ in range(max(1, args.repeats)):
        for i in range(args.warmup):
            er.launch(i)
        barrier()
        r0 = torch.cuda.Event(enable_timing=True)
        r1 = torch.cuda.Event(enable_timing=True)
        hold_device(torch)
        r0.record(stream)
        for i in range(K):
            er.launch(i)
        r1.record(stream)
        barrier()
        early_ms.append(r0.elapsed_time(r1) / K)
    er.check_status()
    local_ms = total_ms
    total_ms = max_over_ranks(total_ms, dist, dev)

    nbytes = run.bytes
    value = job_gbs(nbytes, K, world, total_ms)
    rows_per_s = w.rows * K * world / (total_ms / 1e3)
    # this rank's mean duration of one call (its kernels run back to back)
    mean_launch_ms = local_ms / K
    achieved = nbytes / (mean_launch_ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()

    # ---- end to end through the public call, host buffers, copies timed
    e2e_steps = max(1, args.e2e_steps)
    TDT = {"bf16": torch.bfloat16, "fp16": torch.float16}[w.dtype]
    x1p = torch.from_numpy(np.ascontiguousarray(w.x1).view(np.int16)).view(TDT).pin_memory()
    x2p = torch.from_numpy(np.ascontiguousarray(w.x2).view(np.int16)).view(TDT).pin_memory()
    params = run.params
    # two device buffer sets and two pinned host output sets: step k uses set
    # k % 2, so the copy-in of step k+1 and the copy-out of step k overlap the
    # calls (three streams, ordered by events)
    sets_e = run.sets[:2]
    outs_h = []
    for ge in sets_e:
        outs_h.append({k: torch.empty(ge[k].shape, dtype=ge[k].dtype).pin_memory()
                       for k in ("y1", "s1", "y2", "s2", "xo") if ge[k] is not None})
    h2d = x1p.numel() * 2 * 2
    d2h = sum(t.numel() * t.element_size() for t in outs_h[0].values())
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_comp = [None, None]  # the call of set j done (its inputs read, outputs written)
    ev_out = [None, None]   # the copy-out of set j done (its outputs read)

    def e2e_step(k):
        j = k % 2
        ge, oh = sets_e[j], outs_h[j]
        if ev_comp[j] is not None:
            s_in.wait_event(ev_comp[j])
        with torch.cuda.stream(s_in):
            ge["x1"].copy_(x1p, non_blocking=True)
            ge["x2"].copy_(x2p, non_blocking=True)
        ev_in = torch.cuda.Event()
        ev_in.record(s_in)
        stream.wait_event(ev_in)
        if ev_out[j] is not None:
            stream.wait_event(ev_out[j])
        q.add_rms_norm_dynamic_quant(
            ge["x1"], ge["x2"], params[0], params[1], params[2], params[3], eps=w.eps,
            output_mask=w.mask, qdtype=w.qdtype, stream=stream,
            out={"y1": ge["y1"], "scale1": ge["s1"], "y2": ge["y2"], "scale2": ge["s2"],
                 "x_out": ge["xo"]})
        ev_comp[j] = torch.cuda.Event()
        ev_comp[j].record(stream)
        s_out.wait_event(ev_comp[j])
        with torch.cuda.stream(s_out):
            for key, t in oh.items():
                t.copy_(ge[key], non_blocking=True)
        ev_out[j] = torch.cuda.Event()
        ev_out[j].record(s_out)

    for k in range(2):
        e2e_step(k)
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    s_in.wait_event(e_start)
    for k in range(e2e_steps):
        e2e_step(k)
    for j in range(2):
        stream.wait_event(ev_out[j])
    e_end.record(stream)
    barrier()
    e2e_ms = e_start.elapsed_time(e_end)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    e2e_value = job_gbs(nbytes, e2e_steps, world, e2e_ms)
    headline_plan = plan.as_dict()
    del run
    torch.cuda.empty_cache()

    # ---- the other workloads, in the same run (this rank alone; device time of
    # one call).  Large ones: K' calls back to back, 3 rotated sets (each call's
    # inputs have left L2 when they come round again).  Small ones (latency):
    # a CUDA graph of back-to-back calls, on L2-cold rotated sets and on one
    # L2-hot set; plus the host time of one call.
    workloads = None
    wl_clocks = ClockSampler(local, period=0.002)
    if not args.no_workloads:
        workloads = {}
        wl_clocks.start()
        for name in LARGE:
            if name == args.workload:
                continue
            wr = DeviceRun(wl.CONFIGS[name](), dev, stream, nsets=3)
            ck = ClockSampler(local, period=0.002)
            ck.start()
            regions = [wr.timed(steps=200, warmup=20) for _ in range(5)]
            ck.stop()
            wr.check_status()
            ms = statistics.median(regions)
            e = workload_entry(wr, ms, peak, "200 calls back to back, 3 sets; median of 5 "
                                             "timed regions")
            e["us_per_call_min_max"] = [min(regions) * 1e3, max(regions) * 1e3]
            e["clocks"] = ck.summary()
            if e["clocks"]["sm_mhz"]:
                e["us_x_ghz"] = ms * e["clocks"]["sm_mhz"]  # ms * MHz = us * GHz
            # the same calls with the parameters promised constant (plan
            # early_params: loaded before the wait for the preceding call)
            ep = wr.with_plan(early_params=1)
            e["early_params_us_per_call"] = statistics.median(
                [ep.timed(steps=200, warmup=20) for _ in range(3)]) * 1e3
            ep.check_status()
            e["workload"] = wr.w.name
            workloads[name] = e
            del wr
            torch.cuda.empty_cache()
        # the no-add operator on the 8192 x 4096 workload's x1 and parameters
        workloads["c2_no_add"] = time_no_add(wl.CONFIGS["c2"](), dev, stream, peak)
        torch.cuda.empty_cache()
        for name in SMALL:
            ww = wl.CONFIGS[name]()
            o1, o2 = outputs_of(ww)
            nsets = sets_for(ww, o1, o2, min_bytes=300 << 20)
            wr = DeviceRun(ww, dev, stream, nsets=nsets)
            cold = wr.graph_timed(calls=nsets)
            wr.check_status()
            e = workload_entry(wr, cold, peak, f"CUDA graph of {nsets} calls on {nsets} rotated "
                                                f"sets (L2-cold), median of 20 replays")
            hot_run = DeviceRun(ww, dev, stream, nsets=1)
            hot = hot_run.graph_timed(calls=256)
            hot_run.check_status()
            e["hot_us_per_call"] = hot * 1e3
            e["host_us_per_call"] = hot_run.host_us()
            e["workload"] = ww.name
            workloads[name] = e
            del wr, hot_run
            torch.cuda.empty_cache()
        wl_clocks.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, rps, cores, sample = time_oracle(w, on1, on2)
        cpu = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample,
               "rows_per_s": rps}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_ms / K,
        "ms_per_step_repeats": ({"median": statistics.median(repeats), "min": min(repeats),
                                 "max": max(repeats), "regions": len(repeats),
                                 "rank": "this rank (rank 0)"} if repeats else None),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded numpy PCG64, rounded to the input dtype; no dataset exists)",
        "config": {
            "workload": w.name, "rows": w.rows, "n": w.n, "io_dtype": w.dtype,
            "qdtype": w.qdtype, "output_mask": w.mask, "beta": w.beta is not None,
            "smooth1": w.smooth1 is not None, "smooth2": w.smooth2 is not None, "eps": w.eps,
            "l2": f"{args.sets} rotated buffer sets, inputs {2 * w.rows * w.n * 2 / 1e6:.0f} MB "
                  f"per set (> 126 MB L2)",
            "timing": f"CUDA events around the K calls, queued behind a "
                      f"{HOST_AHEAD_CYCLES}-cycle device delay outside the timed region",
            "plan": headline_plan,
            "parallelism": f"replicas x{world} (rows independent; no collective)",
        },
        "early_params": {"ms_per_step": statistics.median(early_ms), "regions": len(early_ms),
                         "gbs": nbytes / (statistics.median(early_ms) / 1e3) / 1e9,
                         "note": "opt-in (plan early_params / constant_params=True): gamma, "
                                 "beta and smooth loaded before the wait for the preceding "
                                 "call; valid when that work does not write them"},
        "rows_per_s": rows_per_s,
        "bytes_per_step": nbytes,
        "frac_of_nominal_hbm": value / world / NOMINAL_HBM_GBS,
        "roofline": {
            "bound": "hbm",
            "achieved": achieved,
            "peak": peak,
            "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": recorded_traffic(w.name, headline_plan),
            "peak_kind": peak_kind,
            "kernel": "arnq::rows_kernel (one launch per arnq_run call; each CTA settles "
                      "its rows from their records after its last row)",
            "mean_call_us": mean_launch_ms * 1e3,
            "launches_per_call": launches_per_call(plan),
        },
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "ms_per_step": e2e_ms / e2e_steps,
                "pipeline": "two buffer sets: copy-in of step k+1 and copy-out of step k "
                            "overlap, each step's outputs read back to pinned host memory"},
        "gpu_launches": K * launches_per_call(plan),
        "clocks": clocks.summary(),
        "workloads": workloads,
        "workloads_clocks": wl_clocks.summary() if workloads is not None else None,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
