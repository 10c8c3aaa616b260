#!/usr/bin/env python
"""Benchmark of the heterogeneous-batch LoRA branch (segmented shrink/expand) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

A step applies the LoRA delta of one batch to every projection the workload names
(inputs resident in HBM).  Each timed region replays a CUDA graph holding exactly K
steps that cycle through enough independent buffer sets (pools, X, Y) to exceed
twice the L2 cache, bracketed by CUDA events on the launching stream; the region is
taken R times (R >= 5) and the line reports the median, with the spread.  Metric:
LoRA delta tokens/s (adapter rows per second), plus achieved HBM GB/s of the step
against the measured copy peak.

Default workload: the 70B-shaped decoder block (d 8192, 2048 decode rows over 128
rank-16 adapters, all seven projections), the largest single-GPU configuration,
with the projections that read the same input rows (q/k/v, gate/up) applied by one
mlora_apply_multi call each.  --config selects another workload for the headline:
1 tiny, 2 qproj_decode, 3 qkv_prefill, 4 mixed_mlp, 5 block70b; --no-fused applies
every projection with its own mlora_apply.  With the default headline the line
also carries ``per_config``: the same measurement for workloads 2, 3 and 4 (and a
parity-only entry for 1), so one run covers every workload.

Next to the steady-state step (consecutive steps overlap only as far as programmatic
dependent launch lets the next step's kernels start early) the line reports the
isolated step (one step after an L2 flush, nothing to overlap with) and the first
step of the process.

The default line also carries ``base_gemm``: the base projection fused with the LoRA
branch (mlora_base_gemm_apply) against torch.matmul followed by mlora_apply, on the
prefill workload (--base-gemm runs that leg alone).

With --gpus N > 1 outside torchrun the script relaunches itself under
torch.distributed.run with N ranks.  Each rank runs its own batch of the same shape
(independent problems, no collective on the data path); value = all ranks' tokens /
the slowest rank's time.  --impl reference times the fp64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

METRIC = "LoRA delta tokens/s and achieved HBM GB/s (% roofline), decode & prefill"
UNIT = "delta tokens/s"
DEFAULT_CONFIG = 5
PER_CONFIG = (1, 2, 3, 4)
L2_FALLBACK = 126 * 2**20

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}
BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


# --------------------------------------------------------------------------- workload facts

# Projections of one layer that read the same input rows.
FUSION_SETS = ({"q_proj", "k_proj", "v_proj"}, {"gate_proj", "up_proj"})


def fusion_groups(W, fused: bool):
    """Projection indices applied together: with ``fused``, the members of each fusion
    set with a common d_in form one group (at its first member's place); otherwise
    every projection alone."""
    n = len(W.proj_shapes)
    if not fused:
        return [[j] for j in range(n)]
    groups, taken = [], set()
    for j, (name, d_in, _) in enumerate(W.proj_shapes):
        if j in taken:
            continue
        fam = next((f for f in FUSION_SETS if name in f), None)
        g = [j] if fam is None else [i for i, (nm, di, _) in enumerate(W.proj_shapes)
                                     if i not in taken and nm in fam and di == d_in]
        taken.update(g)
        groups.append(g)
    return groups


def group_leaders(groups):
    """Projection -> the projection whose X it reads (the first of its group)."""
    return {j: g[0] for g in groups for j in g}


def workload_facts(W, groups=None) -> dict:
    """Algorithmic bytes and flops of one step (every projection once; X once per group)."""
    leader = group_leaders(groups or [[j] for j in range(len(W.proj_shapes))])
    adapter = W.row_slot >= 0
    n_l = int(adapter.sum())
    distinct = W.referenced_slots
    r_rows = W.slot_rank[W.row_slot[adapter]].astype(np.int64)
    total_bytes = 0
    flops = 0
    per_proj = []
    for j, (name, d_in, d_out) in enumerate(W.proj_shapes):
        w_bytes = int(sum(int(W.slot_rank[s]) * (d_in + d_out) * 2 for s in distinct))
        x_bytes = n_l * d_in * 2 if leader[j] == j else 0
        y_bytes = n_l * d_out * 2 * 2
        b = w_bytes + x_bytes + y_bytes
        per_proj.append({"name": name, "d_in": d_in, "d_out": d_out, "bytes": b,
                         "weight_bytes": w_bytes})
        total_bytes += b
        flops += int(2 * r_rows.sum() * (d_in + d_out))
    return {"adapter_rows": n_l, "distinct_adapters": int(distinct.size),
            "bytes": total_bytes, "flops": flops, "per_projection": per_proj}


def workload_config(W, facts, groups, world: int) -> dict:
    """The ``config`` object of a bench line: the workload and how it is applied."""
    tokens = facts["adapter_rows"]
    return {
        "workload": W.name, "projections": [p[0] for p in W.proj_shapes],
        "shapes": [[p[1], p[2]] for p in W.proj_shapes], "rows": W.n_rows,
        "adapter_rows": tokens, "slots": W.n_slots,
        "distinct_adapters": facts["distinct_adapters"],
        "ranks": sorted(set(int(r) for r in W.slot_rank[W.referenced_slots])),
        "global_batch": tokens * world,
        "parallelism": f"replicas x{world} (independent batches)",
        "fused": [[W.proj_shapes[j][0] for j in g] for g in groups if len(g) > 1],
    }


def max_over_ranks(x: float, device=None) -> float:
    """Largest ``x`` over all ranks of the process group (``x`` itself without one).
    Every rank must call it the same number of times."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, steps: int, world: int, seconds: float) -> float:
    """Units that all ranks processed (each rank its own batch) per second of the
    slowest rank's time."""
    return units_per_rank * steps * world / seconds


def graph_kernel_count(graph):
    """Kernel nodes in a captured torch CUDA graph (the launches one replay makes), or
    None if the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as cudart
        g = cudart.cudaGraph_t(init_value=int(graph.raw_cuda_graph()))
        err, _, n = cudart.cudaGraphGetNodes(g, numNodes=0)
        if err != cudart.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = cudart.cudaGraphGetNodes(g, numNodes=n)
        if err != cudart.cudaError_t.cudaSuccess:
            return None
        count = 0
        for node in nodes[:n]:
            err, t = cudart.cudaGraphNodeGetType(node)
            if err != cudart.cudaError_t.cudaSuccess:
                return None
            count += int(t == cudart.cudaGraphNodeType.cudaGraphNodeTypeKernel)
        return count
    except Exception:
        return None


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "segmented_rank_gemm_02_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on these sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("src_hash") == kernel_source_hash():
            return e.get("dram_bytes_per_step")
    except Exception:
        pass
    return None


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML on a background thread."""

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        p = self.nvml
        while not self._stop.is_set():
            try:
                mhz = p.nvmlDeviceGetClockInfo(self.h, p.NVML_CLOCK_SM)
                try:
                    reasons = p.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    reasons = p.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, int(reasons)))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self._t.join(timeout=2)

    def summary(self, t0: float, t1: float) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:   # very short region: nearest samples around it
            inside = sorted(self.samples, key=lambda s: abs(s[0] - 0.5 * (t0 + t1)))[:3]
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= s[2]
        names = sorted(n for b, n in REASON_BITS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(inside)}


# --------------------------------------------------------------------------- CPU oracle

def cpu_oracle_rate(W, seconds: float, steps: int = 0, n_threads: int = 0):
    """Time the fp64 oracle on a bounded sample of the workload (tokens/s).
    ``n_threads`` 0 = every host core (OpenMP's default)."""
    import oracle
    threads = n_threads or oracle.max_threads()
    projs = [W.projection(j) for j in range(len(W.proj_shapes))]
    adapter_rows = np.nonzero(W.row_slot >= 0)[0]
    # per-row cost estimate on a small sample
    probe = adapter_rows[: min(16, adapter_rows.size)]
    t = time.perf_counter()
    for p in projs:
        oracle.reference(W, p, rows=probe, n_threads=threads)
    per_row = (time.perf_counter() - t) / max(1, probe.size)
    budget = seconds / max(1, steps) if steps else seconds
    n_rows = int(max(1, min(adapter_rows.size, budget / max(per_row, 1e-9))))
    rows = adapter_rows[:n_rows]
    done = 0
    t0 = time.perf_counter()
    reps = 0
    while True:
        for p in projs:
            oracle.reference(W, p, rows=rows, n_threads=threads)
        done += rows.size
        reps += 1
        el = time.perf_counter() - t0
        if steps:
            if reps >= steps:
                break
        elif el >= seconds * 0.5:
            break
    el = time.perf_counter() - t0
    sample = (f"first {rows.size} of {adapter_rows.size} adapter rows of {W.name}, all "
              f"{len(projs)} projection(s), {reps} pass(es)")
    return done / el, el, sample, threads


# --------------------------------------------------------------------------- GPU arm

class Repeated:
    """Median and spread of R timings of the same region (milliseconds)."""

    def __init__(self, ms):
        self.ms = sorted(float(m) for m in ms)

    @property
    def median(self) -> float:
        return statistics.median(self.ms)

    def summary(self, per: int = 1) -> dict:
        return {"median": self.median / per, "min": self.ms[0] / per, "max": self.ms[-1] / per,
                "n": len(self.ms)}


def flush_l2(buf) -> None:
    """Overwrite a buffer larger than L2 on the current stream (evicts cached lines)."""
    buf.add_(1)


def measure(args, cfg: int, fused: bool, rank: int, world: int, device_index: int,
            e2e_seconds: float, repeats: int, cpu: bool) -> dict:
    """One workload: parity on sampled rows, then the steady-state K-step graph R
    times, the isolated step, the first step, and the end-to-end leg."""
    import torch
    import oracle
    import segmented_rank_gemm_02_b200 as mlora
    import workloads as wl

    dev = torch.device("cuda", device_index)
    W = wl.make(cfg)
    groups = fusion_groups(W, fused)
    leader = group_leaders(groups)
    facts = workload_facts(W, groups)
    projs = [W.projection(j) for j in range(len(W.proj_shapes))]
    # the members of a fused group read their leader's X
    projs = [p if leader[j] == j else dataclasses.replace(p, X=projs[leader[j]].X)
             for j, p in enumerate(projs)]
    meta = mlora.build_segments(W.row_slot)

    # device copies of the adapters, used to fill every pool of the ring
    dA = [{s: mlora.as_bf16_tensor(p.A[s], dev) for s in p.A} for p in projs]
    dB = [{s: mlora.as_bf16_tensor(p.B[s], dev) for s in p.B} for p in projs]
    X0 = [mlora.as_bf16_tensor(p.X, dev) for p in projs]
    Y0 = [mlora.as_bf16_tensor(p.Y0, dev) for p in projs]

    def new_set():
        out = []
        for j, p in enumerate(projs):
            pool = mlora.Pool(p.d_in, p.d_out, W.n_slots, W.r_max)
            for s in sorted(p.A):
                pool.load_slot(s, int(W.slot_rank[s]), float(W.slot_alpha[s]), dA[j][s], dB[j][s])
            m = dict(meta)
            m["ranks"] = np.array([0 if s < 0 else W.slot_rank[s] for s in meta["slots"]], np.int32)
            segs = mlora.DeviceSegments(m, W.n_rows, dev)
            X = X0[j].clone() if leader[j] == j else out[leader[j]]["X"]
            out.append({"pool": pool, "segs": segs, "X": X, "Y": Y0[j].clone()})
        return out

    rb = next(b for b in (8, 16, 32, 64) if b >= W.r_max)
    pool_bytes = sum(W.n_slots * 2 * (((rb * (p.d_in + p.d_out) + 127) // 128) * 128)
                     for p in projs)
    act_bytes = sum(W.n_rows * ((p.d_in if leader[j] == j else 0) + p.d_out) * 2
                    for j, p in enumerate(projs))
    set_bytes = pool_bytes + act_bytes
    try:
        l2 = int(torch.cuda.get_device_properties(dev).L2_cache_size)
    except Exception:
        l2 = L2_FALLBACK
    n_sets = max(1, math.ceil(2 * l2 / set_bytes))
    sets = [new_set() for _ in range(n_sets)]
    flush_buf = torch.zeros(2 * l2 // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)

    def apply_group(entries, g, stream=None, segs=None):
        if len(g) == 1:
            e = entries[g[0]]
            mlora.apply(e["pool"], segs or e["segs"], e["X"], e["Y"], stream=stream)
        else:
            e0 = entries[g[0]]
            mlora.apply_multi([entries[j]["pool"] for j in g], segs or e0["segs"], e0["X"],
                              [entries[j]["Y"] for j in g], stream=stream)

    def step(k):
        for g in groups:
            apply_group(sets[k % n_sets], g, stream=stream)

    # the first step of the process on this workload (cold caches, first launches)
    with torch.cuda.stream(stream):
        flush_l2(flush_buf)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step(0)
        e1.record(stream)
    stream.synchronize()
    first_ms = e0.elapsed_time(e1)
    for j in range(len(projs)):
        sets[0][j]["Y"].copy_(Y0[j])
    torch.cuda.synchronize()

    # parity on sampled rows of a fresh set (outside any timed region)
    rows = np.unique(np.concatenate([meta["token_indices"][meta["offsets"][:-1]],
                                     np.nonzero(W.row_slot >= 0)[0][:8],
                                     meta["token_indices"][np.maximum(meta["offsets"][1:] - 1, 0)]]))
    rows = rows[W.row_slot[rows] >= 0][:96]
    worst = 0.0
    for g in groups:
        apply_group(sets[0], g)
        for j in g:
            e, p = sets[0][j], projs[j]
            assert e["pool"].check() == 0
            got = oracle.bf16_to_f64(mlora.bf16_bits(e["Y"][torch.as_tensor(rows, device=dev)]))
            ref = oracle.reference(W, p, rows=rows)
            worst = max(worst, float(np.max(np.abs(got - ref) / (1e-2 * (1 + np.abs(ref))))))
            e["Y"].copy_(Y0[j])
    torch.cuda.synchronize()

    # warm-up steps (eager; at least one per buffer set, which sizes every pool's
    # workspace before capture), then capture exactly K steps into one graph
    with torch.cuda.stream(stream):
        for k in range(max(args.warmup, n_sets)):
            step(k)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph(keep_graph=True)   # kept so its kernel nodes can be counted
    with torch.cuda.graph(graph, stream=stream):
        for k in range(args.steps):
            step(k)
    launches = graph_kernel_count(graph)
    graph.instantiate()
    with torch.cuda.stream(stream):
        graph.replay()   # first replay uploads the graph; not timed
    stream.synchronize()
    per_apply = (launches / (args.steps * len(groups))) if launches else None
    call = "mlora_apply_multi / mlora_apply" if fused and any(len(g) > 1 for g in groups) \
        else "mlora_apply"
    kernel_desc = (f"{call}: lora_decode_kernel" if per_apply == 1 else
                   f"{call}: lora_decode_kernel + long_shrink_kernel + long_expand_kernel"
                   if per_apply and per_apply >= 3 else call)

    dist = None
    if world > 1:
        import torch.distributed as dist

    def timed_once():
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            start.record(stream)
            graph.replay()
            end.record(stream)
        stream.synchronize()
        return start.elapsed_time(end)

    def timed_region():
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        ms = [timed_once() for _ in range(repeats)]
        t1 = time.perf_counter()
        if dist:
            dist.barrier()
        return Repeated(ms), t0, t1

    with ClockSampler(device_index) as clk:
        rep, t0, t1 = timed_region()
    clocks = clk.summary(t0, t1)
    if set(clocks.get("reasons", [])) & BAD_REASONS:
        with ClockSampler(device_index) as clk:
            rep, t0, t1 = timed_region()
        clocks = clk.summary(t0, t1)
        clocks["remeasured"] = True
    ms_med = max_over_ranks(rep.median, dev)
    del graph

    # the isolated step: one step after an L2 flush (no earlier step to overlap with);
    # the flush kernel in front keeps the host's launch time out of the interval
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        step(0)
    iso = []
    for _ in range(max(5, repeats)):
        with torch.cuda.stream(stream):
            flush_l2(flush_buf)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g1.replay()
            b.record(stream)
        stream.synchronize()
        iso.append(a.elapsed_time(b))
    del g1
    iso = Repeated(iso)
    iso_med = max_over_ranks(iso.median, dev)

    e2e = run_e2e(args, W, projs, meta, sets[0], dev, stream, world, groups, apply_group,
                  e2e_seconds) if e2e_seconds > 0 else None

    tokens = facts["adapter_rows"]
    steps = args.steps
    sec = ms_med / 1e3
    value = whole_job_rate(tokens, steps, world, sec)
    per_step_s = (rep.median / 1e3) / steps
    peaks = measured_peaks()
    achieved = facts["bytes"] / per_step_s / 1e9
    traffic = recorded_traffic(W.name + ("_fused" if fused and any(len(g) > 1 for g in groups)
                                         else ""))
    out = {
        "workload": W.name, "value": value, "unit": UNIT, "ms_per_step": ms_med / steps,
        "us_per_step": rep.summary(steps / 1e3),
        "isolated_us_per_step": iso_med * 1e3,
        "isolated_spread_us": iso.summary(1 / 1e3),
        "first_step_us": first_ms * 1e3,
        "config": dict(workload_config(W, facts, groups, world), **{
            "l2": f"rotating {n_sets} buffer set(s) of {set_bytes / 2**20:.0f} MiB "
                  f"({n_sets * set_bytes / 2**20:.0f} MiB > 2x {l2 / 2**20:.0f} MiB L2)",
            "timing": f"one CUDA graph of exactly K steps, CUDA events on its stream, "
                      f"taken {repeats} times: median (spread in us_per_step)"}),
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
            "peak_source": peaks["source"], "algorithmic_bytes_per_step": facts["bytes"],
            "flops_per_step": facts["flops"],
            "tensor_frac": facts["flops"] / per_step_s / 1e12 / peaks["bf16_tflops"],
            "isolated_frac": facts["bytes"] / (iso.median / 1e3) / 1e9 / peaks["hbm_gbs"],
            "kernel": kernel_desc,
        },
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "parity": {"rows_checked": int(rows.size), "max_err_over_tolerance": worst},
    }
    if cpu:
        rate, el, sample, cores = cpu_oracle_rate(W, args.cpu_seconds)
        out["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample, "seconds": el}
    for s in sets:
        for e in s:
            e["pool"].close()
    del sets, flush_buf
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def parity_only(cfg: int, device_index: int) -> dict:
    """Every row of a small workload against the oracle, plus the oracle's one-thread
    rate on it (the workload is far too small to time the GPU meaningfully)."""
    import torch
    import oracle
    import segmented_rank_gemm_02_b200 as mlora
    import workloads as wl
    from segmented_rank_gemm_02_b200 import staging
    dev = torch.device("cuda", device_index)
    W = wl.make(cfg)
    worst = 0.0
    for j in range(len(W.proj_shapes)):
        p = W.projection(j)
        st = staging.upload(W, p, dev)
        mlora.apply(st["pool"], st["segs"], st["X"], st["Y"])
        assert st["pool"].check() == 0
        got = oracle.bf16_to_f64(mlora.bf16_bits(st["Y"]))
        ref = oracle.reference(W, p)
        worst = max(worst, float(np.max(np.abs(got - ref) / (1e-2 * (1 + np.abs(ref))))))
        base = W.row_slot < 0
        assert np.array_equal(mlora.bf16_bits(st["Y"])[base], p.Y0[base])
        st["pool"].close()
    return {"workload": W.name, "parity": {"rows_checked": W.n_rows, "max_err_over_tolerance": worst}}


def base_gemm_leg(args, device_index: int, cfg: int = 3) -> dict:
    """The base projection fused with the LoRA branch (mlora_base_gemm_apply: one
    shrink, then one tensor-core GEMM that adds s (X A^T) B^T into the accumulator of
    X W^T) against the two-kernel path a caller would otherwise run (torch.matmul for
    X W^T, then mlora_apply onto it), on the prefill workload.  Each arm is a CUDA
    graph of K steps over rotating buffer sets larger than twice L2, timed R times."""
    import torch
    import segmented_rank_gemm_02_b200 as mlora
    import workloads as wl

    dev = torch.device("cuda", device_index)
    W = wl.make(cfg)
    proj = W.projection(0)
    Wb = W.base_weight(0)
    meta = mlora.build_segments(W.row_slot)
    meta["ranks"] = np.array([0 if s < 0 else W.slot_rank[s] for s in meta["slots"]], np.int32)
    X0 = mlora.as_bf16_tensor(proj.X, dev)
    W0 = mlora.as_bf16_tensor(Wb, dev)
    set_bytes = (W.n_rows * (proj.d_in + 2 * proj.d_out) + proj.d_out * proj.d_in) * 2
    try:
        l2 = int(torch.cuda.get_device_properties(dev).L2_cache_size)
    except Exception:
        l2 = L2_FALLBACK
    n_sets = max(2, math.ceil(2 * l2 / set_bytes))
    sets = []
    for _ in range(n_sets):
        pool = mlora.Pool(proj.d_in, proj.d_out, W.n_slots, W.r_max)
        for s in sorted(proj.A):
            pool.load_slot(s, int(W.slot_rank[s]), float(W.slot_alpha[s]), proj.A[s], proj.B[s])
        sets.append({"pool": pool, "segs": mlora.DeviceSegments(meta, W.n_rows, dev), "X": X0.clone(),
                     "W": W0.clone(), "Y": torch.empty((W.n_rows, proj.d_out), dtype=torch.bfloat16, device=dev)})
    stream = torch.cuda.Stream(device=dev)

    def fused(e):
        mlora.base_gemm_apply(e["pool"], e["segs"], e["X"], e["W"], e["Y"], stream=stream)

    def two_kernel(e):
        torch.matmul(e["X"], e["W"].t(), out=e["Y"])
        mlora.apply(e["pool"], e["segs"], e["X"], e["Y"], stream=stream)

    def matmul(e):
        torch.matmul(e["X"], e["W"].t(), out=e["Y"])

    def time_arm(fn):
        with torch.cuda.stream(stream):
            for k in range(max(args.warmup, n_sets)):   # sizes every workspace before capture
                fn(sets[k % n_sets])
        stream.synchronize()
        graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(graph, stream=stream):
            for k in range(args.steps):
                fn(sets[k % n_sets])
        launches = graph_kernel_count(graph)
        graph.instantiate()
        with torch.cuda.stream(stream):
            graph.replay()
        stream.synchronize()
        ms = []
        for _ in range(args.repeats):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                a.record(stream)
                graph.replay()
                b.record(stream)
            stream.synchronize()
            ms.append(a.elapsed_time(b))
        del graph
        return Repeated(ms), launches

    with ClockSampler(device_index) as clk:
        t0 = time.perf_counter()
        r_fused, n_fused = time_arm(fused)
        r_two, n_two = time_arm(two_kernel)
        r_mm, _ = time_arm(matmul)
        t1 = time.perf_counter()
    clocks = clk.summary(t0, t1)
    # the two arms' outputs on the same inputs: both round once to bf16, the two-kernel
    # arm twice (X W^T, then the sum), so they agree to about one bf16 step
    e = sets[0]
    fused(e)
    Yf = e["Y"].float()
    two_kernel(e)
    Yt = e["Y"].float()
    torch.cuda.synchronize()
    agree = float(((Yf - Yt).abs() / (1e-2 * (1 + Yt.abs()))).max().item())
    assert e["pool"].check() == 0
    steps = args.steps
    us = {name: r.median * 1e3 / steps for name, r in (("fused", r_fused), ("two_kernel", r_two),
                                                          ("matmul", r_mm))}
    adapter_rows = int((W.row_slot >= 0).sum())
    base_flops = 2.0 * W.n_rows * proj.d_in * proj.d_out
    lora_flops = 2.0 * adapter_rows * int(W.slot_rank.max()) * (proj.d_in + proj.d_out)
    peaks = measured_peaks()
    achieved = (base_flops + lora_flops) / (us["fused"] * 1e-6) / 1e12
    for s in sets:
        s["pool"].close()
    del sets
    torch.cuda.empty_cache()
    return {
        "workload": W.name, "call": "mlora_base_gemm_apply",
        "shape": {"rows": W.n_rows, "d_in": proj.d_in, "d_out": proj.d_out, "adapter_rows": adapter_rows,
                  "rank": int(W.slot_rank.max())},
        "us_per_step": {"fused": us["fused"], "matmul_plus_apply": us["two_kernel"], "matmul_alone": us["matmul"]},
        "spread_us": {"fused": r_fused.summary(steps / 1e3), "matmul_plus_apply": r_two.summary(steps / 1e3)},
        "speedup_vs_matmul_plus_apply": us["two_kernel"] / us["fused"],
        "delta_tokens_per_s": adapter_rows / (us["fused"] * 1e-6),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops_sustained"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops_sustained"],
                     "peak_source": peaks["source"] + " (sustained bf16)",
                     "flops_per_step": base_flops + lora_flops},
        "gpu_launches_per_step": {"fused": n_fused / steps if n_fused else None,
                                  "matmul_plus_apply": n_two / steps if n_two else None},
        "agreement_with_two_kernel_over_tolerance": agree,
        "l2": f"rotating {n_sets} buffer sets of {set_bytes / 2**20:.0f} MiB (> 2x L2)",
        "clocks": clocks,
    }


def run_ours(args, rank: int, world: int, device_index: int):
    import torch
    torch.cuda.set_device(device_index)
    cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    head = measure(args, args.config, args.fused, rank, world, device_index, args.e2e_seconds,
                   args.repeats, cpu)
    result = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": head["config"], "roofline": head["roofline"],
        "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
        "parity": head["parity"], "us_per_step": head["us_per_step"],
        "isolated_us_per_step": head["isolated_us_per_step"],
        "isolated_spread_us": head["isolated_spread_us"], "first_step_us": head["first_step_us"],
    }
    if "cpu_baseline" in head:
        result["cpu_baseline"] = head["cpu_baseline"]
    if args.per_config and world == 1:
        per = {}
        for cfg in PER_CONFIG:
            if cfg == args.config:
                continue
            if cfg == 1:
                e = parity_only(cfg, device_index)
            else:
                e = measure(args, cfg, args.fused, rank, world, device_index,
                            args.per_config_e2e_seconds, args.repeats, False)
                for k in ("config", "clocks"):
                    e.pop(k)
            if cfg in (1, 2) and rank == 0 and not args.no_cpu_baseline:
                import workloads as wl
                rate, el, sample, cores = cpu_oracle_rate(wl.make(cfg), min(args.cpu_seconds, 3.0),
                                                          n_threads=1)
                e["cpu_one_thread"] = {"value": rate, "unit": UNIT, "cores": cores,
                                       "kind": "oracle", "sample": sample, "seconds": el}
            per[str(cfg)] = e
        result["per_config"] = per
        result["base_gemm"] = base_gemm_leg(args, device_index)
    return result


def run_e2e(args, W, projs, meta0, entries, dev, stream, world, groups, apply_group,
            e2e_seconds):
    """The same step through the public API with host buffers, pipelined the way a
    serving loop would run it: step k's host grouping and H2D copies (copy-in
    stream) overlap step k-1's apply (compute stream) and step k-2's D2H copy
    (copy-out stream), over two device buffer sets.  Every step still groups its
    rows on the host, copies its metadata, X and Y0 from pinned memory to the device,
    applies, and copies Y back."""
    import torch
    import segmented_rank_gemm_02_b200 as mlora

    row_slot = np.ascontiguousarray(W.row_slot, np.int32)
    S_max = W.n_rows
    n = W.n_rows
    # One pinned host arena and one device arena per buffer set, laid out as
    # [metadata: offsets S+1 | slots S | ranks S | token_indices n][Y0 / Y of every
    # projection][X of every projection] (16-byte aligned parts), so that a step's
    # inputs go over in one H2D copy and its results come back in one D2H copy.
    def al(nbytes):
        return (nbytes + 255) // 256 * 256
    meta_bytes = al(4 * (3 * S_max + 1 + n))
    y_off, x_off, off = [], [], meta_bytes
    for p in projs:
        y_off.append(off)
        off += al(p.Y0.nbytes)
    y_end = off
    leader = group_leaders(groups)
    for j, p in enumerate(projs):
        if leader[j] == j:   # a fused group's members read their leader's X
            x_off.append(off)
            off += al(p.X.nbytes)
        else:
            x_off.append(x_off[leader[j]])
    arena_bytes = off
    host = [torch.empty(arena_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
    devb = [torch.empty(arena_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    for h in host:
        hn = h.numpy()
        for j, p in enumerate(projs):
            hn[y_off[j]:y_off[j] + p.Y0.nbytes] = p.Y0.view(np.uint8).reshape(-1)
            hn[x_off[j]:x_off[j] + p.X.nbytes] = p.X.view(np.uint8).reshape(-1)
    out = [torch.empty(y_end - meta_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]

    def view_bf16(t, start, shape):
        nb = int(np.prod(shape)) * 2
        return t[start:start + nb].view(torch.bfloat16).view(*shape)
    Xd = [[view_bf16(devb[b], x_off[j], p.X.shape) for j, p in enumerate(projs)] for b in range(2)]
    Yd = [[view_bf16(devb[b], y_off[j], p.Y0.shape) for j, p in enumerate(projs)] for b in range(2)]
    meta_view = [h[:4 * (3 * S_max + 1 + n)].view(torch.int32).numpy() for h in host]
    pool0 = entries[0]["pool"]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    s_comp = stream
    in_done = [None, None]    # H2D of the set finished (its pinned arena may be refilled)
    out_done = [None, None]   # D2H of the set finished (its device arena may be reused)
    counter = [0]

    def one_step():
        b = counter[0] & 1
        counter[0] += 1
        if in_done[b] is not None:
            in_done[b].synchronize()                     # the DMA has read host[b]
        m = mlora.build_segments(row_slot, pool0)        # host grouping (C, via the ABI)
        S = int(m["slots"].size)
        mh = meta_view[b]
        mh[:S + 1] = m["offsets"]
        mh[S_max + 1:S_max + 1 + S] = m["slots"]
        mh[2 * S_max + 1:2 * S_max + 1 + S] = m["ranks"]
        mh[3 * S_max + 1:] = m["token_indices"]
        with torch.cuda.stream(s_in):
            if out_done[b] is not None:
                s_in.wait_event(out_done[b])
            devb[b].copy_(host[b], non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
        in_done[b] = ev_in
        base = devb[b].data_ptr()
        segs = mlora.SegmentsStruct(S, n, n, int(m["max_segment_rows"]),
                                    base, base + 4 * (S_max + 1), base + 4 * (2 * S_max + 1), None,
                                    base + 4 * (3 * S_max + 1))
        holder = type("S", (), {})()
        holder.struct = segs
        s_comp.wait_event(ev_in)
        views = [{"pool": e["pool"], "X": Xd[b][j], "Y": Yd[b][j]} for j, e in enumerate(entries)]
        for g in groups:
            apply_group(views, g, stream=s_comp, segs=holder)
        ev_comp = torch.cuda.Event()
        ev_comp.record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp)
            out[b].copy_(devb[b][meta_bytes:y_end], non_blocking=True)
            ev_out = torch.cuda.Event()
            ev_out.record(s_out)
        out_done[b] = ev_out

    for _ in range(max(3, min(args.warmup, 10))):
        one_step()
    torch.cuda.synchronize()
    t = time.perf_counter()
    for _ in range(4):
        one_step()
    torch.cuda.synchronize()
    est = (time.perf_counter() - t) / 4
    steps = int(max(3, min(args.steps, e2e_seconds / max(est, 1e-6))))
    steps = int(max_over_ranks(steps, dev))   # the same count on every rank
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(s_in)
    for _ in range(steps):
        one_step()
    end.record(s_out)   # after the last step's D2H, which follows all of its work
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    # the result read back to the host is the device's result of the last step
    lb = (counter[0] - 1) & 1
    assert torch.equal(out[lb].to(dev), devb[lb][meta_bytes:y_end]), "e2e read-back mismatch"
    tokens = int((W.row_slot >= 0).sum())
    ms = max_over_ranks(ms, dev)
    h2d = arena_bytes
    d2h = y_end - meta_bytes
    return {"value": whole_job_rate(tokens, steps, world, ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps, "ms_per_step": ms / steps,
            "includes": "host grouping (mlora_build_segments), one H2D copy of metadata+X+Y0 "
                        "from pinned memory, the apply calls, one D2H copy of Y; steps pipelined "
                        "over copy-in, compute and copy-out streams with two buffer sets"}


# --------------------------------------------------------------------------- slot loads

def run_slot_load(args):
    """Adapter loads (mlora_pool_load_slot from page-locked host memory: H2D copy and
    repack) for every adapter the workload references, and how much they slow down
    applies running meanwhile on another stream (loads go to slots the batch does not
    use)."""
    import torch
    import segmented_rank_gemm_02_b200 as mlora
    import workloads as wl
    from segmented_rank_gemm_02_b200 import staging

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    W = wl.make(args.config)
    proj = W.projection(0)
    slots = sorted(proj.A)
    host = {s: (torch.from_numpy(proj.A[s].view(np.int16)).pin_memory(),
                torch.from_numpy(proj.B[s].view(np.int16)).pin_memory()) for s in slots}
    nbytes = sum(proj.A[s].nbytes + proj.B[s].nbytes for s in slots)
    spare = [s for s in range(W.n_slots) if s not in proj.A]
    pool = mlora.Pool(proj.d_in, proj.d_out, W.n_slots, W.r_max)
    s_load, s_apply = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def load_all(targets):
        for s, t in zip(slots, targets):
            pool.load_slot(t, int(W.slot_rank[s]), float(W.slot_alpha[s]), host[s][0], host[s][1],
                           stream=s_load)

    load_all(slots)
    torch.cuda.synchronize()
    reps = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_load)
    for _ in range(reps):
        load_all(slots)
    e1.record(s_load)
    torch.cuda.synchronize()
    load_ms = e0.elapsed_time(e1) / reps

    st = staging.upload(W, proj, dev, pool=pool)
    k = 200

    def applies():
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(s_apply)
        for _ in range(k):
            mlora.apply(pool, st["segs"], st["X"], st["Y"], stream=s_apply)
        a1.record(s_apply)
        return a0, a1

    a0, a1 = applies()
    torch.cuda.synchronize()
    a0, a1 = applies()
    torch.cuda.synchronize()
    alone_us = a0.elapsed_time(a1) * 1e3 / k
    # the same applies while adapters stream into the spare slots on the other stream
    targets = [spare[i % len(spare)] for i in range(len(slots))] if spare else None
    with_us = None
    if targets:
        a0, a1 = applies()
        for _ in range(reps):
            load_all(targets)
        torch.cuda.synchronize()
        with_us = a0.elapsed_time(a1) * 1e3 / k
    assert pool.check() == 0
    return {"metric": "adapter slot loads from page-locked host memory (H2D + repack)",
            "value": nbytes / (load_ms / 1e3) / 1e9, "unit": "GB/s", "higher_is_better": True,
            "config": {"workload": W.name, "adapters": len(slots), "bytes_per_round": nbytes,
                       "rank": sorted(set(int(W.slot_rank[s]) for s in slots))},
            "us_per_adapter": load_ms * 1e3 / len(slots),
            "apply_us_alone": alone_us, "apply_us_with_concurrent_loads": with_us,
            "note": "applies (eager launches) on one stream, loads into spare slots on another"}


# --------------------------------------------------------------------------- reference arm

def run_reference(args, rank: int, world: int):
    import workloads as wl
    W = wl.make(args.config)
    groups = fusion_groups(W, args.fused)
    facts = workload_facts(W, groups)
    budget = float(args.cpu_seconds) if args.cpu_seconds else 60.0
    # warm-up passes are bounded samples too (not timed)
    if args.warmup:
        cpu_oracle_rate(W, budget * 0.05, steps=1)
    rate, el, sample, cores = cpu_oracle_rate(W, budget, steps=max(1, args.steps))
    return {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(W, facts, groups, world),
        "cpu_baseline": {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def relaunch(argv, gpus: int) -> int:
    """Run this script under torch.distributed.run with ``gpus`` ranks on this node."""
    import socket
    import subprocess
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main(argv=None) -> int:
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--repeats", type=int, default=7,
                    help="timed K-step regions per measurement (median reported); at least 5")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--e2e-seconds", type=float, default=3.0)
    ap.add_argument("--per-config-e2e-seconds", type=float, default=1.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fused", action=argparse.BooleanOptionalAction, default=True,
                    help="one mlora_apply_multi per group of projections reading the same X "
                         "(default); --no-fused: one mlora_apply per projection")
    ap.add_argument("--per-config", action=argparse.BooleanOptionalAction, default=None,
                    help="also measure the other workloads (default: with the default headline)")
    ap.add_argument("--base-gemm", action="store_true",
                    help="only the fused base GEMM + LoRA leg (mlora_base_gemm_apply against "
                         "torch.matmul + mlora_apply) on the prefill workload (one GPU)")
    ap.add_argument("--slot-load", action="store_true",
                    help="measure adapter slot loads instead of the apply step (one GPU)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.repeats < 5:
        ap.error("--repeats must be at least 5")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if args.per_config is None:
        args.per_config = "--config" not in " ".join(argv)

    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        return relaunch(argv, args.gpus)
    world = int(env_world or "1")
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        return 2
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.slot_load:
        print(json.dumps(run_slot_load(args)), flush=True)
        return 0
    if args.base_gemm:
        import torch
        torch.cuda.set_device(0)
        leg = base_gemm_leg(args, 0)
        print(json.dumps(dict({"metric": "fused base GEMM + LoRA delta vs torch.matmul + mlora_apply",
                               "value": leg["us_per_step"]["fused"], "unit": "us per step",
                               "higher_is_better": False}, **leg)), flush=True)
        return 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0

    pg = False
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
        pg = True
    try:
        result = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
