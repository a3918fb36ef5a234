"""Benchmark: MoE dispatch + combine on one B200, on seeded synthetic inputs
resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen3|dsv3|dsv3_skew|mixtral|tiny|page_k4|page_k8|
                                page_k4_32k|page_k8_32k]
                    [--workloads dsv3,dsv3_skew,mixtral|none]

One step = one pass of the path over one batch.  What is timed (``value``) is
dispatch + combine, the steps of the metric:
  forward-only workloads:   dispatch (layout + permute, one call) | combine
  fwd+bwd workloads:        dispatch | combine + combine backward |
                            dispatch backward (a unit-weight combine)
The seeded stand-in expert (y = x * s_e, and its backward) runs between the
timed segments -- the combine needs its output -- but outside the CUDA
events: it stands where the grouped expert GEMMs would and is not part of
dispatch or combine.

Each segment is captured once in its own CUDA graph and replayed every step.
Before every timed segment L2 is flushed outside the events (a 256 MiB device
write, then a 256 MiB read of another buffer, so the segment starts with
neither useful nor dirty lines in L2); CUDA events on the launching stream
bracket each timed segment; the step time is the sum of its timed segments;
``value`` = tokens/s over all ranks (every rank's tokens / the slowest rank's
total time).

Default workload: Qwen3-MoE-shaped fwd+bwd (T=16384 tokens, H=2048, E=128 in
8 logical ranks, top_k=8, fp32 router weights, mild skew, align 16), the one
configuration that runs every step of the path.  ``workloads`` adds, in the
same run and the same JSON line, the DeepSeek-V3-shaped (balanced and severe
skew) and Mixtral-shaped configurations, each with its tokens/s, step GB/s,
fraction of the measured HBM peak and its dominant kernel's fraction.

Other keys of the JSON line (rank 0 prints ONE line):
  kernels      per dispatch/combine kernel (the layout and the permute as
               separate calls): mean time of an eager launch
               (flushed L2 before it, CUDA events around it), share of the
               timed work, algorithmic bytes and GB/s, fraction of the
               measured peak, ncu DRAM traffic per launch while the kernel's
               source is unchanged since the committed capture;
  roofline     the dominant dispatch/combine kernel (largest share; the
               stand-in is never a candidate): algorithmic bytes per launch /
               mean event-timed duration against the measured HBM copy
               bandwidth;
  full_step    the whole path including the stand-in (8 launches for fwd+bwd)
               captured in one graph, one flush per step;
  e2e          the full step through pinned host buffers with the
               host<->device copies inside the timed region;
  cpu_baseline the CPU oracle on a bounded token sample of the same workload,
               the same dispatch/combine steps: the plain single-threaded
               build and the OpenMP build on all host cores (rank 0, N=1).
With --impl reference the OpenMP oracle itself is timed as the reference arm.
N>1 runs independent replicas (the path has no exchange step on one device):
weak scaling.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "dispatch+combine tokens/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0

# The dispatch/combine kernels the metric times, and the stand-in expert
# launches that run between them untimed.
METHOD = ("layout", "permute", "combine", "combine_backward", "dispatch_backward")
STAND_IN = ("expert_scale", "expert_scale_bwd")

# Kernels one call of a step launches (the layout: a tile kernel and a row
# kernel; the dispatch: those and the permute; every other call: one).
KERNELS_PER_CALL = {"layout": 2, "dispatch": 3}

# Step names -> the kernel function each launches at top_k = K: the permute
# streams rows through its shared-memory ring at K <= 2; above K = 8 the
# combines use their any-K kernels.
def kernel_function(name: str, K: int) -> str:
    if name == "permute":
        return "permute_ring_kernel" if K <= 2 else "permute_kernel"
    if name in ("combine", "dispatch_backward"):
        return "combine_slots_kernel" if K <= 8 else "combine_kernel"
    if name == "combine_backward":
        return "combine_bwd_slots_kernel" if K <= 8 else "combine_bwd_kernel"
    if name == "layout":
        return "layout_tiles_kernel + layout_rows_kernel"
    return "expert_scale_kernel"

KERNEL_SOURCES = {
    "layout": "layout.cu", "permute": "permute.cu", "expert_scale": "expert_scale.cu",
    "expert_scale_bwd": "expert_scale.cu", "combine": "combine.cu", "combine_backward": "combine.cu",
    "dispatch_backward": "combine.cu",
}


# ------------------------------------------------------------------ setup ---

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(ws, backend="nccl"):
    if ws > 1:
        import torch.distributed as dist
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=180))
        return dist
    return None


def max_over_ranks(dist, value: float, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(dist, tokens_per_rank: int, steps: int, total_ms: float, device):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    ws = dist.get_world_size() if dist is not None else 1
    slowest = max_over_ranks(dist, total_ms, device)
    return tokens_per_rank * ws * steps / (slowest / 1e3), slowest


def barrier(dist, device):
    if dist is not None:
        dist.barrier(device_ids=[device.index] if device.type == "cuda" else None)


# ------------------------------------------------------ algorithmic bytes ---

def algorithmic_bytes(T, H, K, E, R, N_cap, N_pad):
    """Bytes each launch must move (read + write) -- what the method needs,
    not what the kernel happens to do.  P = pad rows = N_pad - A."""
    A = T * K
    P = N_pad - A
    row = 2 * H
    return {
        "layout": 8 * A + T * R,
        "permute": T * row + A * row + P * row + 8 * A + 4 * A + 4 * N_cap,
        "expert_scale": A * row + N_pad * row,
        "combine": A * row + T * row + 4 * A + 4 * A,
        "combine_backward": T * row + A * row + A * row + P * row + 12 * A + 4 * N_pad,
        "expert_scale_bwd": A * row + N_pad * row,
        "dispatch_backward": A * row + T * row + 4 * A,
    }


# ----------------------------------------------------------------- clocks ---

class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = [v.strip() for v in vis.split(",")] if vis else []
        self.gpu = ids[gpu_index] if gpu_index < len(ids) and ids[gpu_index] else str(gpu_index)
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        try:
            rows = [ln.split(",") for ln in open(self.path).read().strip().splitlines() if ln]
            os.unlink(self.path)
        except Exception:
            return None
        sm, mx, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1])); mx.append(float(r[2])); power.append(float(r[3]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


# ------------------------------------------------------------------- ours ---

class Path:
    """Preallocated buffers and the launches of one step, grouped into the
    segments the bench times (dispatch / combine) and the stand-in expert
    launches between them (run, not timed)."""

    def __init__(self, inp, cfg, device):
        from combine_moe_dispatch_03_b200 import api
        self.api = api
        self.cfg = cfg
        self.dev = device
        T, H, E, K, R = cfg.T, cfg.H, cfg.E, cfg.K, cfg.R
        self.backward = bool(cfg.backward)
        self.x = inp["x"].to(device)
        self.topk = inp["topk_idx"].to(device)
        self.w = inp["weights"].to(device)
        self.s = inp["scales"].to(device)
        self.N = api.worst_case_rows(T, K, E, cfg.align)
        bf = dict(dtype=torch.bfloat16, device=device)
        self.status = api.new_status(device)
        self.lay = api.alloc_layout(T, K, E, R, cfg.align, device)
        self.xp = torch.zeros(self.N, H, **bf)
        self.r2f = torch.empty(self.N, dtype=torch.int32, device=device)
        self.f2r = torch.empty(T, K, dtype=torch.int32, device=device)
        self.y = torch.zeros(self.N, H, **bf)
        self.out = torch.empty(T, H, **bf)
        if self.backward:
            self.g = inp["grad_out"].to(device)
            self.grad_rows = torch.zeros(self.N, H, **bf)
            self.grad_w = torch.empty(T, K, dtype=torch.float32, device=device)
            self.grad_xp = torch.zeros(self.N, H, **bf)
            self.grad_x = torch.empty(T, H, **bf)

    def segments(self):
        """(segment name, calls, timed) in step order.  The dispatch segment
        is one call (moe_dispatch: the layout, then the permute)."""
        seg = [("dispatch", ("dispatch",), True),
               ("expert", ("expert_scale",), False)]
        if self.backward:
            seg += [("combine", ("combine", "combine_backward"), True),
                    ("expert_bwd", ("expert_scale_bwd",), False),
                    ("dispatch_backward", ("dispatch_backward",), True)]
        else:
            seg += [("combine", ("combine",), True)]
        return seg

    def launches(self):
        return [n for _, calls, _ in self.segments() for n in calls]

    def kernel_calls(self):
        """The step's calls with the dispatch as its two separate calls (layout,
        permute), so that each method kernel is timed on its own."""
        out = []
        for n in self.launches():
            out += ["layout", "permute"] if n == "dispatch" else [n]
        return out

    def method_launches(self):
        return [n for n in self.kernel_calls() if n in METHOD]

    def call(self, name):
        api, c, st = self.api, self.cfg, self.status
        if name == "dispatch":
            api.dispatch(self.x, self.topk, c.E, c.R, c.align, capacity=self.N, status=st,
                         layout_out=self.lay, out=(self.xp, self.r2f, self.f2r))
        elif name == "layout":
            api.dispatch_layout(self.topk, c.E, c.R, c.align, status=st, out=self.lay)
        elif name == "permute":
            api.permute(self.x, self.topk, self.lay, capacity=self.N, status=st,
                        out=(self.xp, self.r2f, self.f2r))
        elif name == "expert_scale":
            api.expert_scale(self.xp, self.lay, self.s, status=st, out=self.y)
        elif name == "combine":
            api.combine_weighted(self.y, self.f2r, self.w, status=st, out=self.out)
        elif name == "combine_backward":
            api.combine_backward(self.g, self.y, self.r2f, self.f2r, self.w, self.lay, status=st,
                                 out=(self.grad_rows, self.grad_w))
        elif name == "expert_scale_bwd":
            api.expert_scale(self.grad_rows, self.lay, self.s, status=st, out=self.grad_xp)
        elif name == "dispatch_backward":
            api.combine_weighted(self.grad_xp, self.f2r, None, status=st, out=self.grad_x)
        else:
            raise KeyError(name)

    def step(self):
        for n in self.launches():
            self.call(n)


class Flush:
    """Evicts L2 outside the timed events: a 256 MiB write, then a 256 MiB
    read of a second buffer, so the next timed launch finds neither its own
    data nor dirty lines (whose write-back it would pay for) in L2."""

    def __init__(self, device):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.acc = torch.zeros((), dtype=torch.float32, device=device)

    def __call__(self, i=1):
        self.w.fill_(i & 0xFF)
        torch.sum(self.r, dim=0, out=self.acc)


def kernel_source_sha(name: str) -> str:
    p = os.path.join(ROOT, "combine_moe_dispatch_03_b200", "csrc", KERNEL_SOURCES[name])
    h = hashlib.sha256()
    for f in (p, os.path.join(ROOT, "combine_moe_dispatch_03_b200", "csrc", "common.cuh")):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(name: str, cfg_name: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel source as it is now; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        d = json.load(open(p))
        e = d[cfg_name][name]
        if e.get("source_sha") == kernel_source_sha(name):
            return e["bytes_per_launch"]
    except Exception:
        pass
    return None


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def capture(path, calls):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for n in calls:
            path.call(n)
    return g


def time_segments(path, steps, warmup, flush, dist, device):
    """Every segment captured once in its own CUDA graph; per step each timed
    segment is replayed between two CUDA events after an L2 flush, the
    stand-in segments are replayed without events.  Returns per-segment
    event times [steps] and the per-step sums."""
    segs = path.segments()
    graphs = [capture(path, calls) for _, calls, _ in segs]
    for _ in range(max(warmup, 0)):
        for (name, _, timed), g in zip(segs, graphs):
            if timed:
                flush()
            g.replay()
    torch.cuda.synchronize(device)
    path.api.check_status(path.status)
    timed_names = [name for name, _, timed in segs if timed]
    evs = {n: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)] for n in timed_names}
    barrier(dist, device)
    torch.cuda.synchronize(device)
    for i in range(steps):
        for (name, _, timed), g in zip(segs, graphs):
            if timed:
                flush(i)
                evs[name][i][0].record()
                g.replay()
                evs[name][i][1].record()
            else:
                g.replay()
    torch.cuda.synchronize(device)
    barrier(dist, device)
    path.api.check_status(path.status)
    per_seg = {n: [a.elapsed_time(b) for a, b in evs[n]] for n in timed_names}
    step_ms = [sum(per_seg[n][i] for n in timed_names) for i in range(steps)]
    del graphs
    return per_seg, step_ms


def time_kernels(path, steps, warmup, flush, dist, device):
    """Eager launches, one at a time: before each dispatch/combine launch an L2
    flush, then CUDA events around the launch alone (the stand-in launches
    run between them, untimed).  Returns {launch: [ms per step]}."""
    names = path.kernel_calls()
    for _ in range(max(warmup, 0)):
        for n in names:
            if n in METHOD:
                flush()
            path.call(n)
    torch.cuda.synchronize(device)
    evs = {n: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)] for n in names if n in METHOD}
    barrier(dist, device)
    torch.cuda.synchronize(device)
    for i in range(steps):
        for n in names:
            if n in METHOD:
                flush(i)
                evs[n][i][0].record()
                path.call(n)
                evs[n][i][1].record()
            else:
                path.call(n)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    path.api.check_status(path.status)
    return {n: [a.elapsed_time(b) for a, b in v] for n, v in evs.items()}


def time_full_step(path, steps, warmup, flush, dist, device):
    """The whole path, stand-in included, captured in one graph; one flush
    per step outside the events."""
    g = capture(path, path.launches())
    for _ in range(max(warmup, 0)):
        flush()
        g.replay()
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    barrier(dist, device)
    torch.cuda.synchronize(device)
    for i in range(steps):
        flush(i)
        evs[i][0].record()
        g.replay()
        evs[i][1].record()
    torch.cuda.synchronize(device)
    barrier(dist, device)
    path.api.check_status(path.status)
    del g
    return [a.elapsed_time(b) for a, b in evs]


def measure_workload(cfg, inp, steps, warmup, dist, device, flush, ws, peak):
    """Dispatch + combine of one workload: graph-timed segments (the value),
    eager per-kernel times (the roofline), algorithmic bytes."""
    path = Path(inp, cfg, device)
    path.step()                       # first calls: per-device launch caches, outside capture
    torch.cuda.synchronize(device)
    per_seg, step_ms = time_segments(path, steps, warmup, flush, dist, device)
    value, total_max = aggregate_throughput(dist, cfg.T, steps, sum(step_ms), device)
    ms_per_step = total_max / steps
    per_kernel = time_kernels(path, steps, warmup, flush, dist, device)
    N_pad = int(path.lay.expert_offsets[-1].item())
    nbytes = algorithmic_bytes(cfg.T, cfg.H, cfg.K, cfg.E, cfg.R, path.N, N_pad)
    method = path.method_launches()
    step_bytes = sum(nbytes[n] for n in method)
    mean_k = {n: statistics.fmean(per_kernel[n]) for n in method}
    total_k = sum(sum(per_kernel[n]) for n in method)
    kernels = {}
    for n in method:
        gbs = nbytes[n] / (mean_k[n] / 1e3) / 1e9
        kernels[n] = {"function": kernel_function(n, cfg.K), "mean_ms": mean_k[n],
                      "share": sum(per_kernel[n]) / total_k, "gbs": gbs, "frac": gbs / peak,
                      "bytes_per_launch": nbytes[n], "traffic": ncu_traffic(n, cfg.name)}
    dom = max(method, key=lambda n: sum(per_kernel[n]))
    gbs = step_bytes / (ms_per_step / 1e3) / 1e9
    res = {
        "value": value, "unit": "tokens/s", "ms_per_step": ms_per_step,
        "p50_ms_per_step": statistics.median(step_ms),
        "segments_ms": {n: statistics.fmean(v) for n, v in per_seg.items()},
        "hbm": {"achieved_gbs": gbs, "bytes_per_step": step_bytes, "peak_gbs": peak,
                "frac": gbs / peak},
        "dominant": {"kernel": dom, "function": kernel_function(dom, cfg.K),
                     "frac": kernels[dom]["frac"], "gbs": kernels[dom]["gbs"]},
        "kernels": kernels,
        "N_cap": path.N, "N_pad": N_pad,
        "launches_per_step": sum(KERNELS_PER_CALL.get(n, 1) for n in path.launches()),
        "timed_launches_per_step": sum(KERNELS_PER_CALL.get(n, 1) for n in method),
    }
    return path, res, nbytes


def run_ours(args, cfg, inp, dist, rank, ws, device):
    from combine_moe_dispatch_03_b200 import build as _b
    if rank == 0:
        _b.build()
    if dist is not None:
        dist.barrier()
    _b.build()
    flush = Flush(device)
    peak, peak_kind = measured_peak()
    sampler = ClockSampler(device.index)
    sampler.start()
    time.sleep(0.3)
    t_wall = time.perf_counter()
    path, main, nbytes = measure_workload(cfg, inp, args.steps, args.warmup, dist, device, flush,
                                          ws, peak)
    t_wall = time.perf_counter() - t_wall
    full = None
    if not args.no_full_step:
        fms = time_full_step(path, args.steps, args.warmup, flush, dist, device)
        fv, fmax = aggregate_throughput(dist, cfg.T, args.steps, sum(fms), device)
        full = {"value": fv, "unit": "tokens/s", "ms_per_step": fmax / args.steps,
                "launches_per_step": sum(KERNELS_PER_CALL.get(n, 1) for n in path.launches()),
                "how": "all launches of the step, stand-in included, in one CUDA graph; "
                       "one L2 flush per step outside the events"}
    e2e = None if args.no_e2e else run_e2e(args, path, inp, dist, device)
    del path
    torch.cuda.empty_cache()

    workloads = {}
    from combine_moe_dispatch_03_b200.inputs import CONFIGS, make_inputs
    extra = [] if args.workloads in ("", "none") else args.workloads.split(",")
    for name in extra:
        if name == cfg.name:
            continue
        wcfg = CONFIGS[name]
        winp = make_inputs(wcfg, seed=wcfg.seed + rank, with_grad=wcfg.backward)
        wpath, wres, _ = measure_workload(wcfg, winp, args.steps, args.warmup, dist, device,
                                          flush, ws, peak)
        wres["workload"] = wcfg.description
        wres["timed"] = ("layout+permute | combine + combine backward | dispatch backward"
                         if wcfg.backward else "layout+permute | combine")
        workloads[name] = wres
        del wpath, winp
        torch.cuda.empty_cache()
    clocks = sampler.stop()

    k = main["kernels"]
    dom = main["dominant"]["kernel"]
    result = {
        "metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
        "p50_ms_per_step": main["p50_ms_per_step"],
        "timing": "dispatch and combine segments, each captured in its own CUDA graph and "
                  "replayed per step between CUDA events; the stand-in expert runs between "
                  "them outside the events",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": cfg.description, "T": cfg.T, "H": cfg.H, "E": cfg.E, "K": cfg.K,
            "R": cfg.R, "align": cfg.align, "N_cap": main["N_cap"], "N_pad": main["N_pad"],
            "router_dtype": "fp32", "global_batch": cfg.T * ws, "parallelism": "replicas",
            "l2": "flushed before every timed segment and every timed kernel: 256 MiB device "
                  "write + 256 MiB read of another buffer, outside the events",
            "timed": ("layout+permute | combine + combine backward | dispatch backward"
                      if cfg.backward else "layout+permute | combine"),
            "untimed": "stand-in expert y = x*s_e (and its backward) between the segments",
        },
        "segments_ms": main["segments_ms"],
        "hbm": dict(main["hbm"], peak_kind=peak_kind),
        "roofline": {"bound": "hbm", "kernel": k[dom]["function"], "launch": dom,
                     "achieved": k[dom]["gbs"], "peak": peak, "unit": "GB/s",
                     "frac": k[dom]["frac"], "traffic": k[dom]["traffic"],
                     "bytes_per_launch": k[dom]["bytes_per_launch"], "mean_ms": k[dom]["mean_ms"],
                     "peak_kind": peak_kind},
        "kernels": k,
        "workloads": workloads,
        "full_step": full,
        "e2e": e2e,
        "gpu_launches": main["launches_per_step"] * args.steps,
        "gpu_launches_timed": main["timed_launches_per_step"] * args.steps,
        "clocks": clocks,
        "wall_s_headline": t_wall,
    }
    return result


def run_e2e(args, path, inp, dist, device):
    """The full step through pinned host buffers: every step copies its
    inputs host->device and its results (out, and for fwd+bwd grad_x and
    grad_w) device->host, inside the timed region.  The steps are pipelined
    the way a serving loop runs them: step i+1's inputs copy in on one stream
    and step i-1's results copy out on another while step i computes, with
    double-buffered device inputs and outputs (events order every reuse).
    L2 is not flushed here: every step's inputs alone exceed L2."""
    steps = max(3, min(args.steps, 50))
    names_in = ["x", "topk_idx", "weights", "scales"] + (["grad_out"] if path.backward else [])
    attr_in = {"x": "x", "topk_idx": "topk", "weights": "w", "scales": "s", "grad_out": "g"}
    attr_in = {n: attr_in[n] for n in names_in}
    attr_out = ("out", "grad_x", "grad_w") if path.backward else ("out",)
    host_in = {k: inp[k].pin_memory() for k in names_in}
    host_out = {a: torch.empty_like(getattr(path, a), device="cpu").pin_memory() for a in attr_out}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    slots = []
    for k in range(2):
        slot = {}
        for a in list(attr_in.values()) + list(attr_out):
            slot[a] = getattr(path, a) if k == 0 else torch.empty_like(getattr(path, a))
        slots.append(slot)
    s_in = torch.cuda.Stream(device)
    s_comp = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    ev = {name: [torch.cuda.Event(), torch.cuda.Event()] for name in ("in", "comp", "out")}

    def issue_in(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev["comp"][b])      # step i-2 has read these inputs
            for n, a in attr_in.items():
                slots[b][a].copy_(host_in[n], non_blocking=True)
            ev["in"][b].record(s_in)

    def issue_comp(i):
        b = i % 2
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev["in"][b])
            if i >= 2:
                s_comp.wait_event(ev["out"][b])     # step i-2's results have been copied out
            for a, t in slots[b].items():
                setattr(path, a, t)
            path.step()
            ev["comp"][b].record(s_comp)

    def issue_out(i):
        b = i % 2
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["comp"][b])
            for a in attr_out:
                host_out[a].copy_(slots[b][a], non_blocking=True)
            ev["out"][b].record(s_out)

    def run(n, t0=None, t1=None):
        if t0 is not None:
            t0.record(s_in)
            s_comp.wait_stream(s_in)
            s_out.wait_stream(s_in)
        for i in range(n + 2):
            if i < n:
                issue_in(i)
            if 1 <= i <= n:
                issue_comp(i - 1)
            if 2 <= i <= n + 1:
                issue_out(i - 2)
        if t1 is not None:
            s_out.wait_stream(s_in)
            s_out.wait_stream(s_comp)
            t1.record(s_out)

    run(3)
    torch.cuda.synchronize(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    run(steps, t0, t1)
    torch.cuda.synchronize(device)
    for a, t in slots[0].items():       # leave the path on its own buffers
        setattr(path, a, t)
    path.api.check_status(path.status)
    total = t0.elapsed_time(t1)
    value, total = aggregate_throughput(dist, path.cfg.T, steps, total, device)
    return {"value": value, "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": total / steps,
            "how": "full step (stand-in included) through the public API; inputs copied in "
                   "from pinned host memory and results copied out every step",
            "pipelined": "copy-in of step i+1 and copy-out of step i-1 overlap step i (3 streams)"}


# ------------------------------------------------------ CPU oracle timing ---

def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.lower().startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def oracle_prepare(orc, cfg, inp, tokens):
    """A token sample of the workload plus the stand-in's outputs, which the
    timed oracle pass takes as inputs (the stand-in is not timed)."""
    from combine_moe_dispatch_03_b200.inputs import bf16_bits
    T = min(tokens, cfg.T)
    T -= T % cfg.R
    T = max(T, cfg.R)
    s = dict(x=bf16_bits(inp["x"][:T]), topk=inp["topk_idx"][:T].numpy(),
             w=inp["weights"][:T].numpy(), sc=inp["scales"].numpy(), E=cfg.E, R=cfg.R,
             align=cfg.align, T=T, N=T * cfg.K + cfg.E * (cfg.align - 1), backward=cfg.backward)
    lay = orc.layout(s["topk"], s["E"], s["R"], s["align"])
    pm = orc.permute(s["x"], s["topk"], s["E"], lay["expert_offsets"], s["N"])
    s["y"] = orc.expert_scale(pm["x_perm"], lay["expert_offsets"], lay["tokens_per_expert"],
                              s["sc"])
    if cfg.backward:
        s["g"] = bf16_bits(inp["grad_out"][:T])
        bw = orc.combine_backward(s["g"], s["y"], pm["row_to_flat"], pm["flat_to_row"], s["w"],
                                  lay["expert_offsets"])
        s["gxp"] = orc.expert_scale(bw["grad_rows"], lay["expert_offsets"],
                                    lay["tokens_per_expert"], s["sc"])
    return s


def oracle_pass(orc, s):
    """One pass of the timed dispatch + combine steps through the oracle."""
    lay = orc.layout(s["topk"], s["E"], s["R"], s["align"])
    pm = orc.permute(s["x"], s["topk"], s["E"], lay["expert_offsets"], s["N"])
    orc.combine(s["y"], pm["flat_to_row"], s["w"], seq=False)
    if s["backward"]:
        orc.combine_backward(s["g"], s["y"], pm["row_to_flat"], pm["flat_to_row"], s["w"],
                             lay["expert_offsets"])
        orc.combine(s["gxp"], pm["flat_to_row"], None, seq=False)


def time_oracle_leg(orc, s, min_s):
    oracle_pass(orc, s)    # warm (page-in)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_pass(orc, s)
        n += 1
        el = time.perf_counter() - t0
        if el >= min_s:
            break
    return s["T"] * n / el, n, el


def time_oracle(cfg, inp, min_s=8.0, tokens=1024):
    import oracle as orc
    orc.build()
    orc.build(openmp=True)
    orc.use_openmp(False)
    s = oracle_prepare(orc, cfg, inp, tokens)
    v1, n1, e1 = time_oracle_leg(orc, s, min_s)
    orc.use_openmp(True)
    try:
        threads = orc.threads()
        vm, nm, em = time_oracle_leg(orc, s, min_s)
    finally:
        orc.use_openmp(False)
    steps = ("layout, permute, combine, combine backward, dispatch backward" if cfg.backward
             else "layout, permute, combine")
    sample = (f"first {s['T']} tokens of the workload (same H, E, K, R, align), the timed "
              f"dispatch/combine steps ({steps}); stand-in outputs precomputed, untimed")
    return {"value": vm, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": sample + f"; OpenMP build, {nm} passes in {em:.1f} s",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "single_core": {"value": v1, "unit": "tokens/s", "cores": 1,
                            "sample": sample + f"; plain build, {n1} passes in {e1:.1f} s"}}


def run_reference(args, cfg, inp, rank, ws):
    """The CPU oracle (OpenMP build, all host cores) timed as the reference
    arm, rank 0 only."""
    if rank != 0:
        return None
    import oracle as orc
    orc.build(openmp=True)
    orc.use_openmp(True)
    threads = orc.threads()
    # size the per-step sample so that warm-up + timed steps take ~2 minutes
    probe = oracle_prepare(orc, cfg, inp, 256)
    t0 = time.perf_counter()
    oracle_pass(orc, probe)
    per_token = (time.perf_counter() - t0) / probe["T"]
    budget = 120.0 / (args.steps + args.warmup)
    tokens = int(max(cfg.R, min(cfg.T, budget / max(per_token, 1e-9))))
    s = oracle_prepare(orc, cfg, inp, tokens)
    for _ in range(max(args.warmup, 0)):
        oracle_pass(orc, s)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_pass(orc, s)
        times.append(time.perf_counter() - t0)
    orc.use_openmp(False)
    total = sum(times)
    value = s["T"] * args.steps / total
    steps = ("layout, permute, combine, combine backward, dispatch backward" if cfg.backward
             else "layout, permute, combine")
    desc = (f"first {s['T']} tokens of the workload per step (same H, E, K, R, align), "
            f"the dispatch/combine steps ({steps}), C oracle built with OpenMP on "
            f"{threads} threads; stand-in outputs precomputed, untimed")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.description, "T": cfg.T, "H": cfg.H, "E": cfg.E, "K": cfg.K,
                   "R": cfg.R, "align": cfg.align, "parallelism": "replicas",
                   "sample_tokens": s["T"]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------- main ---

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen3")
    ap.add_argument("--workloads", default="dsv3,dsv3_skew,mixtral",
                    help="extra workloads timed in the same run ('none' to skip)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-full-step", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (profiling of smaller cases; must divide by R)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    sys.path.insert(0, ROOT)
    from combine_moe_dispatch_03_b200.inputs import CONFIGS, make_inputs
    cfg = CONFIGS[args.workload]
    if args.tokens is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, T=args.tokens,
                                  description=cfg.description + f" (T overridden to {args.tokens})")
    ws, rank, local = dist_env()

    if args.impl == "reference":
        inp = make_inputs(cfg, with_grad=cfg.backward)
        res = run_reference(args, cfg, inp, rank, ws)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(ws)
    try:
        inp = make_inputs(cfg, seed=cfg.seed + rank, with_grad=cfg.backward)
        res = run_ours(args, cfg, inp, dist, rank, ws, device)
        if rank == 0:
            if ws == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = time_oracle(cfg, inp)
            else:
                res["cpu_baseline"] = None
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
