#!/usr/bin/env python
"""Throughput of multi-LoRA delta application on B200.

One step = the whole hot path over one batch: group the batch's rows by
adapter id (lora_build_segments) and apply every linear layer's LoRA delta
(lora_add_linear, which runs the fused shrink/expand kernels).  Inputs are
synthetic, seeded, with the shapes of the workload named in ``config``.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed on the host

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun);
every rank applies the deltas of its own batch (rows are independent, so the
path shards with no collective on the data path) and the step time is the
maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "multi-LoRA delta tokens/s + achieved HBM GB/s (% of B200 peak), SGMV & BGMV"
UNIT = "tokens/s"
HEADLINE = "multislice_8b"
SWEEP = ["decode_qproj", "prefill", "mixed_70b"]
# Runs of at least this many rows become contiguous tiles (the tensor-core SGMV
# kernel); 0 = gathered tiles only.  A serving engine knows whether a batch
# holds prompts: decode-only batches are grouped without contiguous tiles.
MIN_RUN = {"tiny": 0, "decode_qproj": 0, "multislice_8b": 0, "prefill": 64, "mixed_70b": 64}
# Rows per gathered tile.  The fused kernel reads a tile's adapter once for all of its
# rows, but a tile's shrink runs on one SM and its expand items wait for it: 16-row
# tiles keep that critical path short, and the adapter repeats of a popular adapter's
# tiles are mostly L2 hits (64-row tiles were 8 % slower on the Llama-3-8B decode set).
ROWS_PER_TILE = 16
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


# ----------------------------------------------------------------------------- helpers
def code_digest(path):
    """sha256 of a C++/CUDA source with comments and blank space removed: edits to
    comments leave it unchanged, any change to the code does not."""
    import hashlib
    import re
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()


def measured_traffic(workload, n_layers):
    """DRAM bytes of one step's fused-kernel launches (summed over the workload's
    layers) from the committed ncu summaries, with the per-layer figures; None when
    the kernel's code has changed since those captures or a layer is missing."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "lora_adapter_application_b200", "csrc", "bgmv.cu")
    try:
        with open(p) as f:
            rec = json.load(f)["bgmv_kernel"]
        if code_digest(src) != rec["code_sha256"]:
            return None, None
        per = rec[workload]["dram_bytes_per_launch"]
        per = per if isinstance(per, list) else [per]
        if len(per) != n_layers:
            return None, None
        return float(sum(per)), per
    except (OSError, KeyError, ValueError):
        return None, None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


class Dist:
    def __init__(self):
        self.rank = int(os.environ.get("RANK", 0))
        self.world = int(os.environ.get("WORLD_SIZE", 1))
        self.local = int(os.environ.get("LOCAL_RANK", 0))
        self.pg = None
        self.device = "cuda"

    def init(self, backend="nccl"):
        if self.world > 1:
            import datetime
            kw = {"device_id": torch.device("cuda", self.local)} if backend == "nccl" else {}
            torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
            self.pg = torch.distributed.group.WORLD
        self.device = "cuda" if backend == "nccl" else "cpu"

    def barrier(self):
        if self.world > 1:
            torch.distributed.barrier()

    def max(self, x):
        if self.world == 1:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    def sum(self, x):
        if self.world == 1:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.world > 1:
            torch.distributed.destroy_process_group()


class ClockSampler(threading.Thread):
    """NVML clock / clock-event-reason samples of this process's GPU (read only)."""

    def __init__(self, cuda_index, period=0.02):
        super().__init__(daemon=True)
        self.samples = []
        self.period = period
        self.ok = False
        self.stop_flag = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = None
            try:
                props = torch.cuda.get_device_properties(cuda_index)
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = int(vis.split(",")[cuda_index]) if vis else cuda_index
                handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv, self.h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that instead of clocks
            self.err = str(e)

    def reasons(self):
        try:
            return self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def run(self):
        while self.ok and not self.stop_flag.is_set():
            try:
                self.samples.append((time.perf_counter(),
                                     self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self.reasons(),
                                     self.nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self.stop_flag.set()

    def summary(self, t0, t1):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if len(win) < 3:   # a short timed region: widen to the neighbouring samples
            mid = 0.5 * (t0 + t1)
            win = sorted(self.samples, key=lambda s: abs(s[0] - mid))[:5]
            window = "nearest to timed region"
        if not win:
            return {"error": "no samples"}
        bits = 0
        for s in win:
            bits |= int(s[2])
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in REASON_BITS.items() if bits & b and n != "gpu_idle"],
                "power_w_max": max(s[3] for s in win), "samples": len(win), "window": window}


# ----------------------------------------------------------------------------- device data
class DeviceSet:
    """One copy of a batch's inputs on the device: ids, and per layer x, y (base
    output, updated in place), A, B; plus the batch metadata buffers."""

    def __init__(self, w, device, rows_per_tile, min_run):
        import lora_adapter_application_b200 as lora
        self.ids = w.ids.to(device)
        self.ranks = w.ranks.to(device)
        self.alphas = lora.alphas_full(w.alpha, w.N, device)
        self.layers = []
        for l in w.layers:
            self.layers.append({"x": l.x.to(device), "y": l.y0.to(device),
                                "A": [a.to(device) for a in l.A], "B": [b.to(device) for b in l.B],
                                "col_off": list(l.col_off)})
        self.meta = lora.Meta(w.T, w.N, rows_per_tile, min_run, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def nbytes(self):
        n = self.ids.numel() * 4
        for l in self.layers:
            n += l["x"].numel() * l["x"].element_size() + 2 * l["y"].numel() * l["y"].element_size()
            n += sum(t.numel() * t.element_size() for t in l["A"] + l["B"])
        return n


def step(ds):
    import lora_adapter_application_b200 as lora
    lora.lora_build_segments(ds.ids, ds.meta, ds.status)
    for l in ds.layers:
        lora.lora_add_linear(l["y"], l["x"], l["A"], l["B"], l["col_off"], ds.ranks, ds.alphas,
                             ds.meta, ds.status)


def device_sms(sms=None):
    if sms is not None:
        return sms
    return torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148


def segment_plan(w, sms=None):
    """(rows per gathered tile, shortest contiguous run, per-layer all-gathered
    flags) for one batch's segment build, from the library's lora_segment_plan:
    when lora_add_linear will run every row of every layer on the gathered-tile
    kernel, the build makes no contiguous runs and 32-row tiles (the mixed 70B
    batch on B200: 363 us with 16-row tiles and 64-row runs, 347 us so)."""
    import lora_adapter_application_b200 as lora
    return lora.lora_segment_plan(w.T, [sum(l.d_out) for l in w.layers], ROWS_PER_TILE,
                                  MIN_RUN.get(w.name, 64), sms=device_sms(sms))


def segment_params(w, sms=None):
    rows_per_tile, min_run, _ = segment_plan(w, sms)
    return rows_per_tile, min_run


def launches_per_step(w, sms=None):
    """Kernels one step launches: the grouping (one block when T <= 2048, or
    T <= 8192 with N <= 1023; else seven passes), then per layer the gathered-tile kernel, plus the tensor-core
    SGMV kernel when contiguous tiles are enabled and the layer qualifies (bf16,
    r_max a multiple of 16, n_slices * r_max <= 128) and pays: not when the batch
    has fewer 128-row tiles than SMs and the layer is 8192 or more columns wide
    (then the gathered-tile kernel takes every row; LORA_TC_ROUTE overrides), and
    not when the batch was built without contiguous runs (segment_plan)."""
    _, min_run, all_gathered = segment_plan(w, sms)
    builder = 1 if (w.T <= 2048 or (w.T <= 8192 and w.N <= 1023)) else 7
    n = builder
    for l, gathered in zip(w.layers, all_gathered):
        n += 1
        qualifies = (min_run > 0 and w.dtype == torch.bfloat16 and w.r_max % 16 == 0 and
                     len(l.d_out) * w.r_max <= 128)
        if qualifies and not gathered:
            n += 1
    return n


def make_sets(w, device, l2_bytes, rows_per_tile, min_run, max_sets=32):
    first = DeviceSet(w, device, rows_per_tile, min_run)
    per = first.nbytes()
    n = max(1, min(max_sets, math.ceil(2 * l2_bytes / per)))
    sets = [first] + [DeviceSet(w, device, rows_per_tile, min_run) for _ in range(n - 1)]
    return sets, per


def _event(external):
    try:
        return torch.cuda.Event(enable_timing=True, external=external)
    except TypeError:
        return torch.cuda.Event(enable_timing=True)


def time_device(sets, K, W, dist, graph=True):
    """Time exactly K whole steps on the device.  The K steps are captured into one
    CUDA graph and replayed once, so host launch overhead does not enter the
    timed region; without a graph the steps are launched one by one."""
    for i in range(W):
        step(sets[i % len(sets)])
    torch.cuda.synchronize()
    g = None
    if graph:
        try:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for i in range(K):
                    step(sets[i % len(sets)])
            torch.cuda.synchronize()
        except Exception as e:  # capture not available: launch eagerly
            print(f"graph capture failed ({e}); timing eager launches", file=sys.stderr)
            g = None
            torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    start.record()
    if g is not None:
        g.replay()
    else:
        for i in range(K):
            step(sets[i % len(sets)])
    end.record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    dist.barrier()
    step_ms = start.elapsed_time(end) / K
    for st in sets:
        code = int(st.status.item())
        if code:
            raise RuntimeError(f"device status {code}")
    graphed = g is not None
    del g
    return step_ms, t0, t1, graphed


KERNEL_STEPS = 40   # steps of the kernel-time pass (at least 20, whatever --steps is)


def time_layers(sets, K=KERNEL_STEPS):
    """Kernel time of the layer calls alone: every input set is grouped once, then
    K steps of only the lora_add_linear calls are captured into one graph and timed
    with one event pair around the whole replay (no event node between kernels, so
    nothing lengthens a step).  The same kernels, shapes and rotating input sets as
    the step; gaps between dependent kernels are included, so the figure is an upper
    bound on the kernels' own time and never exceeds the step time."""
    import lora_adapter_application_b200 as lora
    for ds in sets:
        lora.lora_build_segments(ds.ids, ds.meta, ds.status)
    torch.cuda.synchronize()

    def layers(ds):
        for l in ds.layers:
            lora.lora_add_linear(l["y"], l["x"], l["A"], l["B"], l["col_off"], ds.ranks, ds.alphas,
                                 ds.meta, ds.status)

    for i in range(len(sets)):
        layers(sets[i])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(K):
            layers(sets[i % len(sets)])
    g.replay()   # warm
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    g.replay()
    end.record()
    torch.cuda.synchronize()
    del g
    return start.elapsed_time(end) / K


def kernel_time(sets, step_ms, K=KERNEL_STEPS):
    """time_layers, taken again once if it came out above the step time (it cannot
    exceed it: the step is the same work plus the grouping); None if it still does."""
    for _ in range(2):
        k = time_layers(sets, K)
        if k <= step_ms:
            return k
    return None


def time_e2e(w, device, K, dist, n_streams=2):
    """Same step through host buffers: pinned host -> device copies of the step's
    inputs (ids, x and base output y of every layer), the path, and the updated y
    back to pinned host memory, all inside the timed region.  Consecutive steps
    alternate between n_streams streams, each with its own device buffers and
    pinned output, so that one step's copies overlap another's kernels as in a
    serving loop; every step still copies its own inputs in and its result out."""
    import lora_adapter_application_b200 as lora
    n_streams = max(1, int(n_streams))
    sets = [DeviceSet(w, device, *segment_params(w)) for _ in range(n_streams)]
    streams = [torch.cuda.Stream(device) for _ in range(n_streams)]
    host = {"ids": w.ids.pin_memory(),
            "layers": [{"x": l.x.pin_memory(), "y": l.y0.pin_memory()} for l in w.layers]}
    outs = [[torch.empty_like(l.y0).pin_memory() for l in w.layers] for _ in range(n_streams)]
    h2d = host["ids"].numel() * 4 + sum(h["x"].numel() * h["x"].element_size() +
                                        h["y"].numel() * h["y"].element_size() for h in host["layers"])
    d2h = sum(o.numel() * o.element_size() for o in outs[0])

    def one(i):
        ds, st, out = sets[i % n_streams], streams[i % n_streams], outs[i % n_streams]
        with torch.cuda.stream(st):
            ds.ids.copy_(host["ids"], non_blocking=True)
            for l, h in zip(ds.layers, host["layers"]):
                l["x"].copy_(h["x"], non_blocking=True)
                l["y"].copy_(h["y"], non_blocking=True)
            lora.lora_build_segments(ds.ids, ds.meta, ds.status, stream=st)
            for l in ds.layers:
                lora.lora_add_linear(l["y"], l["x"], l["A"], l["B"], l["col_off"], ds.ranks,
                                     ds.alphas, ds.meta, ds.status, stream=st)
            for l, o in zip(ds.layers, out):
                o.copy_(l["y"], non_blocking=True)

    for i in range(3 * n_streams):
        one(i)
    torch.cuda.synchronize()
    dist.barrier()
    cur = torch.cuda.current_stream()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(cur)
    for st in streams:
        st.wait_event(s)
    for i in range(K):
        one(i)
    for st in streams:
        cur.wait_stream(st)
    e.record(cur)
    torch.cuda.synchronize()
    ms = dist.max(s.elapsed_time(e) / K)
    for ds in sets:
        code = int(ds.status.item())
        if code:
            raise RuntimeError(f"device status {code}")
    del sets
    return ms, h2d, d2h


def cpu_oracle_rate(w, budget_s, threads=None):
    """Rows per second of the fp64 C oracle on a bounded sample of the workload."""
    import oracle
    oracle.build()
    if threads:
        oracle.set_threads(threads)
    cores = oracle.max_threads()
    active = np.nonzero(w.ids.numpy() >= 0)[0]
    probe = active[: min(8, len(active))]

    def run(rows):
        t = time.perf_counter()
        for l in w.layers:
            oracle.lora_apply(l.x, l.A, l.B, l.col_off, w.ranks, w.alpha, w.ids, l.y0, rows=rows)
        return time.perf_counter() - t

    t_probe = max(run(probe), 1e-6) / max(len(probe), 1)
    n = int(min(w.T, max(len(probe), budget_s / t_probe)))
    rows = np.arange(n, dtype=np.int32)          # the first n rows, -1 rows included as in the batch
    dt, reps = run(rows), 1
    while n == w.T and dt < budget_s:            # a batch cheaper than the budget: repeat it
        dt += run(rows)
        reps += 1
    return n * reps / dt, cores, n, reps, dt


# ----------------------------------------------------------------------------- arms
def bench_ours(args, dist):
    import lora_adapter_application_b200 as lora
    from lora_adapter_application_b200 import roofline
    lora.load()
    device = torch.device("cuda", dist.local)
    torch.cuda.set_device(device)
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    pk = peaks()

    sampler = ClockSampler(dist.local)
    sampler.start()

    w = workloads.make(args.workload, seed=args.seed + 1000 * dist.rank)
    sets, per_set = make_sets(w, device, l2, *segment_params(w))
    step_ms_local, t0, t1, graphed = time_device(sets, args.steps, args.warmup, dist,
                                                 not args.no_graph)
    step_ms = dist.max(step_ms_local)
    tokens_total = dist.sum(w.T)
    value = tokens_total / (step_ms * 1e-3)
    clocks = sampler.summary(t0, t1)
    kern_ms_local = kernel_time(sets, step_ms_local)
    n_sets = len(sets)
    del sets
    torch.cuda.empty_cache()
    rl = roofline_entry(w, kern_ms_local, pk)

    e2e_ms, h2d, d2h = time_e2e(w, device, min(args.steps, args.e2e_steps), dist, args.e2e_streams)

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.info.get('desc', '')}", "T": w.T, "N": w.N,
                   "r_max": w.r_max, "layers": [l.name for l in w.layers],
                   "active_rows": int((w.ids >= 0).sum()),
                   "l2": f"{n_sets} rotating input sets of {per_set / 1e6:.1f} MB "
                         f"(inputs {n_sets * per_set / 1e6:.0f} MB > L2 {l2 / 1e6:.0f} MB)",
                   "parallelism": f"dp{dist.world} (independent batch per GPU)",
                   "launch": ("CUDA graph of the K timed steps" if graphed else "eager") +
                             f"; kernel time from a separate graph of {KERNEL_STEPS} steps of "
                             "the layer calls alone",
                   "rows_per_tile": segment_params(w)[0], "min_run": segment_params(w)[1],
                   "seed": args.seed},
        "roofline": rl,
        "e2e": {"value": tokens_total / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "steps": min(args.steps, args.e2e_steps), "streams": args.e2e_streams},
        "gpu_launches": args.steps * launches_per_step(w),
        "clocks": clocks,
    }

    if dist.world == 1 and not args.no_cpu:
        rate, cores, n, reps, dt = cpu_oracle_rate(w, args.cpu_budget)
        result["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                                  "sample": f"first {n} of {w.T} rows of {w.name}, all layers, "
                                            f"{reps} pass(es), {dt:.1f} s"}

    if dist.world == 1 and not args.no_sweep:
        sweep = {}
        for name in SWEEP:
            sweep[name] = sweep_one(name, args, device, l2, pk, dist)
        result["sweep"] = sweep
    sampler.stop()
    return result


def roofline_entry(w, kern_ms, pk):
    """Roofline of the fused kernel's launches in one step: algorithmic bytes (x, y
    read and written, the live ranks of every adapter touched) over the kernel time,
    against the measured copy bandwidth; the DRAM bytes ncu counted for the same
    launches when a capture of the current kernel code exists."""
    from lora_adapter_application_b200 import roofline
    alg = roofline.workload_bytes(w)
    traffic, per_layer = measured_traffic(w.name, len(w.layers))
    peak = float(pk["hbm_gbs"])
    out = {"bound": "hbm", "achieved": None, "peak": peak, "unit": "GB/s", "frac": None,
           "traffic": traffic, "traffic_per_layer": per_layer,
           "kernel": "bgmv_kernel<MODE_FUSED>" + (" + sgmv_tc_kernel<MODE_FUSED>"
                                                  if segment_params(w)[1] > 0 else ""),
           "kernel_ms": kern_ms, "algorithmic_bytes": alg,
           "algorithmic_flops": roofline.workload_flops(w),
           "peak_source": f"{pk.get('source')} hbm_gbs"}
    if kern_ms:
        out["achieved"] = alg / (kern_ms * 1e-3) / 1e9
        out["frac"] = out["achieved"] / peak
    return out


def sweep_one(name, args, device, l2, pk, dist):
    w = workloads.make(name, seed=args.seed)
    sets, per_set = make_sets(w, device, l2, *segment_params(w), max_sets=4)
    probe_ms, _, _, _ = time_device(sets, 3, 3, dist, graph=False)
    K = int(min(500, max(20, args.sweep_seconds * 1e3 / probe_ms)))
    step_ms, _, _, _ = time_device(sets, K, 3, dist, graph=not args.no_graph)
    kern_ms = kernel_time(sets, step_ms)
    del sets
    torch.cuda.empty_cache()
    rl = roofline_entry(w, kern_ms, pk)
    return {"desc": w.info.get("desc", ""), "T": w.T, "steps": K, "ms_per_step": step_ms,
            "tokens_per_s": w.T / (step_ms * 1e-3), "roofline": rl,
            "frac_hbm_by_step": rl["algorithmic_bytes"] / (step_ms * 1e-3) / 1e9 / rl["peak"],
            "launches_per_step": launches_per_step(w)}


def bench_reference(args, dist):
    """The fp64 CPU oracle as the reference arm, on the host cores."""
    if dist.rank != 0:
        return None
    w = workloads.make(args.workload, seed=args.seed)
    per_step_budget = max(0.2, args.ref_seconds / max(1, args.steps + args.warmup))
    rate, cores, n, _, dt = cpu_oracle_rate(w, per_step_budget)
    import oracle
    rows = np.arange(n, dtype=np.int32)

    def one():
        for l in w.layers:
            oracle.lora_apply(l.x, l.A, l.B, l.col_off, w.ranks, w.alpha, w.ids, l.y0, rows=rows)

    for _ in range(args.warmup):
        one()
    t = time.perf_counter()
    for _ in range(args.steps):
        one()
    total = time.perf_counter() - t
    ms = total / args.steps * 1e3
    value = n / (ms * 1e-3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.info.get('desc', '')}", "T": w.T, "N": w.N,
                   "r_max": w.r_max, "parallelism": "host cores (OpenMP over rows)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: first {n} of {w.T} rows of {w.name}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(workloads.NAMES))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--e2e-streams", type=int, default=2,
                    help="streams the end-to-end steps alternate between (1 = one step at a time)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    ap.add_argument("--sweep-seconds", type=float, default=0.5)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch timed steps one by one")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")

    dist = Dist()
    if args.impl == "reference":
        res = bench_reference(args, dist)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    dist.init()
    try:
        res = bench_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
