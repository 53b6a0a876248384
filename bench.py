"""Benchmark of the MoE layer (route -> dispatch -> grouped SwiGLU FFN -> combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

One step = one pass of the whole layer over one batch of synthetic inputs that
are already resident in HBM (weights, x, logits), timed with CUDA events on the
launching stream. L2 is flushed (a 512 MiB write) between steps, outside the
step's events. Prints one JSON line (rank 0).

N > 1 runs one process per GPU: launched under torchrun (WORLD_SIZE set, which
must equal --gpus), or, when started directly with --gpus N, bench.py re-launches
itself under torch.distributed.run with N ranks on this node. Each rank runs an
independent replica of the layer on its own batch (the path has no cross-GPU
exchange on one node here; "replicas only"), value = all ranks' tokens / the max
over ranks of the timed region.

--impl reference times the CPU oracle (the plain fp64 definition of the layer)
on the host cores, on a bounded sample of tokens of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (route+dispatch+grouped GEMM+combine); % of roofline"
UNIT = "tokens/s"
DEFAULT_CONFIG = "mixtral_prefill"


# ---------------------------------------------------------------------------
# algorithmic work (bytes / flops) of one layer call, from the actual routing
# ---------------------------------------------------------------------------

def algorithmic(wl, counts):
    """Per-step algorithmic bytes and flops of each step (padding excluded). `counts` are the
    rows each expert actually processes (after any capacity drops)."""
    T, d, E, k, f = wl.T, wl.d, wl.E, wl.k, wl.f
    A = int(sum(counts))  # placed assignments
    n_act = int(sum(1 for c in counts if c > 0))
    sh = wl.n_shared
    w = {}
    w["route"] = dict(bytes=T * E * 4 + T * k * 8, flops=0)
    w["dispatch"] = dict(bytes=T * d * 2 + A * d * 2 + T * k * 8, flops=0)
    w["gate_up"] = dict(flops=4 * A * d * f + sh * 4 * T * d * f,
                        bytes=(n_act + sh) * 2 * d * f * 2 + A * d * 2 + sh * T * d * 2)
    w["down"] = dict(flops=2 * A * d * f + sh * 2 * T * d * f,
                     bytes=(n_act + sh) * d * f * 2 + A * d * 2 + sh * T * d * 2)
    w["combine"] = dict(bytes=A * d * 2 + T * k * 8 + T * d * 2 + sh * T * d * 2, flops=0)
    w["_n_act"] = n_act
    return w


NOMINAL_BF16_TFLOPS = 2250.0  # dense bf16 tensor peak of a B200 (data sheet, without sparsity)
NOMINAL_HBM_GBS = 8000.0      # HBM3e bandwidth of a B200 (data sheet)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dram_traffic.md")
KERNEL_SOURCES = ("combine_warp_top_expert_b200/csrc/expert_ffn.cu", "combine_warp_top_expert_b200/csrc/moe_device.cuh",
                  "combine_warp_top_expert_b200/csrc/moe_internal.h")


def strip_c_comments(text: str) -> str:
    """C/C++ source without comments and with runs of white space collapsed (string and
    character literals kept as they are), so that comment edits leave the hash unchanged."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
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
    """Hash of the grouped-GEMM sources' code (comments and layout ignored); a traffic
    figure is valid only for the code it was taken on."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(strip_c_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum) recorded in
    profiles/dram_traffic.md for this workload and kernel, or None if absent or taken on other sources."""
    if not os.path.exists(TRAFFIC_RECORD):
        return None
    text = open(TRAFFIC_RECORD).read()
    if "```json" not in text:
        return None
    try:
        rec = json.loads(text.split("```json", 1)[1].split("```", 1)[0])
    except ValueError:
        return None
    if rec.get("source_hash") != kernel_source_hash():
        return None
    e = rec.get("workloads", {}).get(workload, {}).get(kernel)
    return None if e is None else int(e["dram_bytes_per_launch"])


def replica_seed(base_seed: int, rank: int) -> int:
    """Each replica (rank) runs the workload on its own batch."""
    return base_seed + rank


def max_over_ranks(local_value: float, world: int, device=None) -> float:
    """The slowest rank's value (device-timed milliseconds or seconds); identity at world = 1."""
    if world <= 1:
        return float(local_value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(local_value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(local_value: int, world: int, device=None) -> int:
    """All ranks' counts added up (the whole job's); identity at world = 1."""
    if world <= 1:
        return int(local_value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([int(local_value)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())


def aggregate_throughput(tokens_per_rank: int, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's timed region (weak scaling)."""
    return world * tokens_per_rank * steps / max_seconds


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, pw, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            try:
                pw.append(float(parts[2]))
            except ValueError:
                pass
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "power_w_median": statistics.median(pw) if pw else None, "samples": len(sm)}


# ---------------------------------------------------------------------------
# reference arm / CPU baseline: the oracle on a bounded sample
# ---------------------------------------------------------------------------

def oracle_sample_run(wl, n_tokens: int, weights=None):
    """Time the oracle's whole layer on the first n_tokens tokens of the batch."""
    import numpy as np
    import moe_synth
    import oracle
    toks = np.arange(n_tokens)
    x = moe_synth.host_x(wl, toks)
    lg = moe_synth.host_logits(wl, toks)
    if weights is None:
        weights = (moe_synth.host_w13(wl), moe_synth.host_w2(wl),
                   moe_synth.host_w13s(wl) if wl.n_shared else None, moe_synth.host_w2s(wl) if wl.n_shared else None)
    w13, w2, w13s, w2s = weights
    t0 = time.perf_counter()
    oracle.layer(x, lg, w13, w2, wl.k, wl.R, w13s, w2s)
    return time.perf_counter() - t0, weights


def cpu_baseline(wl, min_s: float = 10.0, target_s: float = 15.0):
    """The oracle as it stands on a bounded token sample, grown until it takes 10-30 s of CPU time."""
    n = 4
    dt, weights = oracle_sample_run(wl, n)
    while dt < min_s and n < wl.T:
        n = int(min(wl.T, max(n + 1, n * min(8.0, max(1.5, target_s / max(dt, 1e-3))))))
        dt, _ = oracle_sample_run(wl, n, weights)
    return dict(value=n / dt, unit=UNIT, cores=os.cpu_count(), kind="oracle",
                sample=f"oracle layer (fp64, OpenMP over rows) on the first {n} of {wl.T} tokens of {wl.name}, "
                       f"all {wl.E} experts' weights resident; {dt:.1f} s")


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    steps = []
    weights = None
    n = 4
    dt, weights = oracle_sample_run(wl, n)
    # size one step to ~ (2 min) / (K + W)
    per_step = max(2.0, 120.0 / max(1, args.steps + args.warmup))
    n = int(min(wl.T, max(1, n * per_step / max(dt, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample_run(wl, n, weights)
    for _ in range(args.steps):
        dt, _ = oracle_sample_run(wl, n, weights)
        steps.append(dt)
    tot = sum(steps)
    value = n * len(steps) / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
        "config": {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "f": wl.f, "R": wl.R,
                   "n_shared": wl.n_shared, "sample_tokens_per_step": n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"oracle layer on the first {n} of {wl.T} tokens per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_gpu(args, wl, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import combine_warp_top_expert_b200 as moe
    import moe_synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    moe.set_gemm_policy({"auto": moe.GEMM_AUTO, "single": moe.GEMM_SINGLE, "pair": moe.GEMM_PAIR}[args.gemm_policy])
    moe.set_pdl(not args.no_pdl)
    moe.set_dispatch_path(DISPATCH_PATHS[args.dispatch_path])
    wl_r = wl.with_(seed=replica_seed(wl.seed, rank))
    cap = moe.capacity_for(args.capacity_factor, wl.T, wl.k, wl.E) if args.capacity_factor else 0
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared, capacity=cap)
    dv = moe_synth.device_inputs(wl_r, device=dev)
    layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"), device=dev, gather=args.gather)
    o = layer.outs
    ws = layer.ws
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def layer_step():
        """One step as a user calls it: the whole layer, one moe_layer call."""
        layer(dv["logits"], dv["x"], stream)

    def split_step(evs):
        """The same work as five separate entry points, with an event between them (the
        per-step split; each interval also holds its call's launch latency)."""
        evs[0].record(stream)
        moe.moe_route(shape, dv["logits"], o["topk_idx"], o["topk_gate"], ws, stream)
        evs[1].record(stream)
        moe.moe_dispatch(shape, dv["x"], o["topk_idx"], o["expert_counts"], o["expert_offsets"], o["rank_counts"],
                         o["rank_offsets"], o["row_src"], o["assign_row"], o["x_perm"], o["imbalance"], ws, stream)
        evs[2].record(stream)
        if args.gather:
            moe.moe_expert_gate_up_gather(shape, dv["x"], o["row_src"], o["expert_offsets"], dv["w13"],
                                          dv.get("w13s"), ws, stream)
        else:
            moe.moe_expert_gate_up(shape, o["x_perm"], o["expert_offsets"], dv["w13"], dv["x"], dv.get("w13s"), ws,
                                   stream)
        evs[3].record(stream)
        moe.moe_expert_down(shape, o["expert_offsets"], dv["w2"], dv.get("w2s"), o["y_perm"], o.get("y_shared"), ws,
                            stream)
        evs[4].record(stream)
        moe.moe_combine(shape, o["y_perm"], o["assign_row"], o["topk_gate"], o.get("y_shared"), o["out"], ws,
                        stream)
        evs[5].record(stream)

    names = ("route", "dispatch", "gate_up", "down", "combine")
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for _ in range(args.warmup):
        flush.zero_()
        layer_step()
    torch.cuda.synchronize(dev)
    status = moe.get_status(ws)
    counts = o["expert_counts"].cpu().numpy().tolist()
    imbalance = o["imbalance"].cpu().numpy().tolist()

    # timed region: K steps of one moe_layer call each; L2 flushed before every step,
    # outside that step's events
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    events = [(ev(), ev()) for _ in range(args.steps)]
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    smi_index = vis.split(",")[local_rank].strip() if vis else str(local_rank)
    launches0 = moe.kernel_launches()
    with ClockSampler(smi_index) as clocks:
        for i in range(args.steps):
            flush.zero_()
            events[i][0].record(stream)
            layer_step()
            events[i][1].record(stream)
        torch.cuda.synchronize(dev)
    # the library's own count of its kernel launches, over all ranks
    gpu_launches = sum_over_ranks(moe.kernel_launches() - launches0, world, dev)
    if world > 1:
        dist.barrier()
    per_step = [a.elapsed_time(b) for a, b in events]
    max_ms = max_over_ranks(sum(per_step), world, dev)
    value = aggregate_throughput(wl.T, args.steps, world, max_ms / 1e3)
    status |= moe.get_status(ws)

    # per-step split: the same K steps through the five entry points, events between calls
    for _ in range(2):
        flush.zero_()
        split_step([ev() for _ in range(6)])
    split_events = [[ev() for _ in range(6)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        split_step(split_events[i])
    torch.cuda.synchronize(dev)
    per_kernel = {n: [e[j].elapsed_time(e[j + 1]) for e in split_events] for j, n in enumerate(names)}
    split_ms = statistics.mean(e[0].elapsed_time(e[5]) for e in split_events)

    # e2e through the public API with host buffers (pinned): every step copies its inputs
    # host->device and its result device->host inside the timed region; successive steps
    # overlap their copies with their neighbours' compute (two staging slots).
    x_h = dv["x"].cpu().pin_memory()
    lg_h = dv["logits"].cpu().pin_memory()
    outs_h = [torch.empty((wl.T, wl.d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    for i in range(max(2, args.warmup)):
        layer.forward_host(lg_h, x_h, outs_h[i % 2], stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for i in range(args.steps):
        layer.forward_host(lg_h, x_h, outs_h[i % 2], stream)
    torch.cuda.synchronize(dev)
    e2e_total = time.perf_counter() - t0
    e2e_value = aggregate_throughput(wl.T, args.steps, world, max_over_ranks(e2e_total, world, dev))
    # one isolated call (copies not overlapped by anything), for reference
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    layer.forward_host(lg_h, x_h, outs_h[0], stream)
    torch.cuda.synchronize(dev)
    e2e_single_ms = (time.perf_counter() - t0) * 1e3

    if rank != 0:
        return
    peaks = load_peaks()
    work = algorithmic(wl, counts)
    kern_ms = {n: statistics.mean(v) for n, v in per_kernel.items()}
    # roofline of each step and of the layer
    roof = {}
    t_roof = 0.0
    t_roof_nominal = 0.0
    for n in names:
        b = work[n]["bytes"] / (peaks["hbm"] * 1e9)
        fl = work[n]["flops"] / (peaks["bf16"] * 1e12)
        t_roof += max(b, fl)
        t_roof_nominal += max(work[n]["bytes"] / (NOMINAL_HBM_GBS * 1e9), work[n]["flops"] / (NOMINAL_BF16_TFLOPS * 1e12))
        roof[n] = dict(ms=kern_ms[n], bound="tensor" if fl > b else "hbm",
                       achieved=(work[n]["flops"] / (kern_ms[n] * 1e-3) / 1e12) if fl > b
                       else (work[n]["bytes"] / (kern_ms[n] * 1e-3) / 1e9),
                       frac=max(b, fl) / (kern_ms[n] * 1e-3))
    dom = max(("gate_up", "down"), key=lambda n: kern_ms[n])
    d = roof[dom]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded generator; weights random-init, no checkpoints)",
        "config": {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "f": wl.f, "R": wl.R,
                   "n_shared": wl.n_shared, "seed": wl.seed, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "flushed between steps (512 MiB write, outside the step's events)",
                   "gemm_tiles": args.gemm_policy,
                   "launch_overlap": "off" if args.no_pdl else "programmatic dependent launch",
                   "dispatch_path": args.dispatch_path,
                   "x_perm": "not materialised (rows gathered in the gate/up GEMM)" if args.gather else "materialised",
                   "capacity_factor": args.capacity_factor, "capacity": cap,
                   "dropped_fraction": 1.0 - sum(counts) / float(wl.T * wl.k) if wl.T else 0.0,
                   "experts_active": work["_n_act"], "imbalance_rank_expert": imbalance,
                   "expert_counts": counts,
                   "ms_per_step_median": statistics.median(per_step),
                   "layer_roofline_frac": t_roof / (max_ms / args.steps / 1e3),
                   "layer_roofline_frac_nominal": t_roof_nominal / (max_ms / args.steps / 1e3),
                   "per_step_ms": {n: round(v, 4) for n, v in kern_ms.items()},
                   "per_step_split": "a second pass of K steps through the five entry points, CUDA events "
                                     f"between calls ({split_ms:.4f} ms per step in that pass)",
                   "per_step_roofline": {n: {"bound": r["bound"], "frac": round(r["frac"], 4)} for n, r in roof.items()},
                   "peaks": peaks, "device_status": status},
        "roofline": {"kernel": f"moe_expert_{dom}", "bound": d["bound"], "achieved": d["achieved"],
                     "peak": peaks["bf16"] if d["bound"] == "tensor" else peaks["hbm"],
                     "unit": "TFLOP/s" if d["bound"] == "tensor" else "GB/s",
                     "frac": d["achieved"] / (peaks["bf16"] if d["bound"] == "tensor" else peaks["hbm"]),
                     "peak_kind": f"{peaks['source']} burst",
                     # context: the same against the sustained (power-capped) GEMM figure, for a kernel
                     # timed inside long steps, and against the nominal data-sheet peaks
                     "frac_sustained": d["achieved"] / peaks["bf16_sustained"] if d["bound"] == "tensor" else None,
                     "frac_nominal": d["achieved"] / (NOMINAL_BF16_TFLOPS if d["bound"] == "tensor" else NOMINAL_HBM_GBS),
                     "traffic": recorded_traffic(wl.name, f"moe_expert_{dom}")
                     if args.tokens is None and args.seed is None else None},
        "clocks": clocks.summary(),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(x_h.numel() * 2 + lg_h.numel() * 4),
                "d2h_bytes_per_step": int(outs_h[0].numel() * 2),
                "timing": "wall clock over the K steps issued back to back (copies of each step overlap the "
                          "neighbouring steps' compute), one synchronize at the end",
                "isolated_call_ms": e2e_single_ms},
        "gpu_launches": gpu_launches,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the grouped GEMM against cuBLAS on the dense-equivalent problem (--dense-compare)
# ---------------------------------------------------------------------------

def run_dense_compare(args):
    """One expert holding every row (no padding: rows % 256 == 0), our two GEMMs against
    torch.matmul (cuBLAS) on the same bf16 operands, L2 flushed before every call, median of
    the timed calls; both tile shapes of ours."""
    import torch

    import combine_warp_top_expert_b200 as moe
    import moe_synth
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def timed(fn, reps=10, warm=3):
        ts = []
        for i in range(warm + reps):
            flush.zero_()
            a, b = ev(), ev()
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= warm:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    for rows, d, f in ((8192, 4096, 14336), (16384, 7168, 2048)):
        wl = moe_synth.Workload("dense", T=rows, d=d, E=1, k=1, f=f, R=1)
        dv = moe_synth.device_inputs(wl)
        shape = moe.Shape(T=rows, d=d, E=1, k=1, f=f, R=1)
        ws = moe.new_workspace(shape)
        offs = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
        y = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
        h = torch.empty((rows, f), dtype=torch.bfloat16, device="cuda")
        line = {"dense_compare": {"rows": rows, "d": d, "f": f}}
        for name, pol in (("single", moe.GEMM_SINGLE), ("pair", moe.GEMM_PAIR)):
            old = moe.set_gemm_policy(pol)
            try:
                gu = timed(lambda: moe.moe_expert_gate_up(shape, dv["x"], offs, dv["w13"], None, None, ws))
                dn = timed(lambda: moe.moe_expert_down(shape, offs, dv["w2"], None, y, None, ws))
            finally:
                moe.set_gemm_policy(old)
            line["dense_compare"][f"ours_{name}_gate_up_tflops"] = round(4.0 * rows * d * f / gu / 1e9, 1)
            line["dense_compare"][f"ours_{name}_down_tflops"] = round(2.0 * rows * d * f / dn / 1e9, 1)
        w13t, w2t = dv["w13"][0].t(), dv["w2"][0].t()
        gu = timed(lambda: torch.matmul(dv["x"], w13t))
        dn = timed(lambda: torch.matmul(h, w2t))
        line["dense_compare"]["cublas_gate_up_tflops"] = round(4.0 * rows * d * f / gu / 1e9, 1)
        line["dense_compare"]["cublas_down_tflops"] = round(2.0 * rows * d * f / dn / 1e9, 1)
        line["dense_compare"]["device_status"] = moe.get_status(ws)
        print(json.dumps(line), flush=True)
        del dv, ws, y, h
        torch.cuda.empty_cache()


def run_sustain(args, wl):
    """--sustain S: the workload's moe_layer back to back for about S seconds (L2 flushed
    before every call, as in the timed region), nvidia-smi sampling SM clock and board power
    every 100 ms. Prints per-window throughput with the clock and power seen in that window,
    and the steady state (second half): what the layer sustains under the board's power
    limit, against the short bursts of the timed region."""
    import torch

    import combine_warp_top_expert_b200 as moe
    import moe_synth
    dv = moe_synth.device_inputs(wl)
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared)
    layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for _ in range(args.warmup):
        flush.zero_()
        layer(dv["logits"], dv["x"])
    torch.cuda.synchronize()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    smi_index = vis.split(",")[0].strip() if vis else "0"
    windows = []  # (host time at the window's end, calls, summed layer ms)
    t_start = time.perf_counter()
    with ClockSampler(smi_index) as clocks:
        while time.perf_counter() - t_start < args.sustain:
            evs = [(ev(), ev()) for _ in range(25)]
            for a, b in evs:
                flush.zero_()
                a.record()
                layer(dv["logits"], dv["x"])
                b.record()
            torch.cuda.synchronize()
            windows.append((time.perf_counter() - t_start, len(evs), sum(a.elapsed_time(b) for a, b in evs)))
    t_samples = [i * 0.1 for i in range(len(clocks.lines))]  # sampler period
    samples = []
    for t, ln in zip(t_samples, clocks.lines):
        parts = [p.strip() for p in ln.split(",")]
        try:
            samples.append((t, float(parts[0]), float(parts[2])))
        except (ValueError, IndexError):
            continue
    half = [w for w in windows if w[0] >= args.sustain / 2] or windows
    ms_steady = sum(w[2] for w in half) / sum(w[1] for w in half)
    steady_s = [x for x in samples if x[0] >= args.sustain / 2 + 0.3] or samples
    out = {"sustain": {
        "workload": wl.name, "seconds": round(windows[-1][0], 2) if windows else 0.0, "calls": sum(w[1] for w in windows),
        "first_window_ms_per_call": round(windows[0][2] / windows[0][1], 4) if windows else None,
        "steady_ms_per_call": round(ms_steady, 4), "steady_tokens_per_s": round(wl.T / (ms_steady * 1e-3)),
        "steady_sm_mhz": statistics.median(x[1] for x in steady_s) if steady_s else None,
        "steady_power_w": statistics.median(x[2] for x in steady_s) if steady_s else None,
        "clocks": clocks.summary(), "device_status": moe.get_status(layer.ws),
        "note": "L2 flushed before every call; per-call CUDA events; nvidia-smi every 100 ms"}}
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# expert parallelism across GPUs (--ep)
# ---------------------------------------------------------------------------

def run_gpu_ep(args, wl, rank, world, local_rank):
    """The expert-parallel layer: `world` ranks (one per GPU), each with its own batch of the
    workload's T tokens and the weights of E / world experts; rows and results cross NVLink
    inside the dispatch and combine kernels (peer buffers in PyTorch symmetric memory).
    At world = 1 the one rank owns every expert and exchanges with itself. Timed per step
    with CUDA events (L2 flushed between steps), max over ranks."""
    import torch
    import torch.distributed as dist

    import combine_warp_top_expert_b200 as moe
    import moe_synth
    from combine_warp_top_expert_b200 import ep

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    moe.set_pdl(not args.no_pdl)
    if wl.E % world:
        raise SystemExit(f"--ep needs E % ranks == 0 (E={wl.E}, ranks={world})")
    Er = wl.E // world
    wl_r = wl.with_(seed=replica_seed(wl.seed, rank))
    cap = moe.capacity_for(args.capacity_factor, wl.T * world, wl.k, wl.E) if args.capacity_factor else 0
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=world, n_shared=wl.n_shared, capacity=cap)
    dv = moe_synth.device_inputs(wl_r, device=dev, weights=False)
    wts = moe_synth.device_expert_weights(wl, rank * Er, (rank + 1) * Er, device=dev)  # this rank's experts only
    w13, w2, w13s, w2s = wts["w13"], wts["w2"], wts.get("w13s"), wts.get("w2s")
    rows_cap = world * wl.T * wl.k
    peers = (ep.EPPeers.symmetric(dist.group.WORLD, wl.E, wl.d, rows_cap, dev) if world > 1
             else ep.EPPeers.emulated(1, wl.E, wl.d, rows_cap, dev))
    layer = ep.EPMoELayer(shape, rank, w13, w2, peers, w13s, w2s, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        layer(dv["logits"], dv["x"])
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches0 = moe.kernel_launches()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record()
        layer(dv["logits"], dv["x"])
        evs[i][1].record()
    torch.cuda.synchronize(dev)
    gpu_launches = sum_over_ranks(moe.kernel_launches() - launches0, world, dev)
    status = layer.status()
    local_ms = sum(a.elapsed_time(b) for a, b in evs)
    max_ms = max_over_ranks(local_ms, world, dev)
    value = aggregate_throughput(wl.T, args.steps, world, max_ms / 1e3)
    recv = int(layer.recv_offsets[-1].item())
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded generator; weights random-init)",
            "config": {"workload": wl.name, "T_per_rank": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "f": wl.f,
                       "n_shared": wl.n_shared, "parallelism": f"expert parallel x{world} (E/R = {Er} experts per GPU)",
                       "capacity": cap, "rows_received_rank0": recv, "device_status": status,
                       "l2": "flushed between steps (512 MiB write, outside the step's events)"},
            # route 1; counts 2 (histogram, exchange); dispatch 4 (wait, plan, rows, signal); expert FFN 2
            # (+2 shared) between a wait and a signal; combine 3 (wait, gather-sum, signal); final wait 1
            "gpu_launches": gpu_launches,
        }), flush=True)
    del layer, peers
    torch.cuda.synchronize(dev)


# ---------------------------------------------------------------------------
# regime sweep: per-expert cost against activated experts and tokens per expert
# ---------------------------------------------------------------------------

def fit_max_affine(G, N, t, iters=50):
    """Fit t = max(a + b*G, c + beta*N) by alternating least squares over the two
    regimes (weight streaming: cost per activated expert; compute: cost per token)."""
    import numpy as np
    G, N, t = (np.asarray(v, dtype=np.float64) for v in (G, N, t))
    n = N / np.maximum(G, 1)
    regime = n >= np.median(n)  # True: compute
    params = None
    for _ in range(iters):
        if regime.all() or (~regime).all():
            regime = n >= np.median(n)
        A1 = np.stack([np.ones((~regime).sum()), G[~regime]], 1)
        A2 = np.stack([np.ones(regime.sum()), N[regime]], 1)
        (a, b), *_ = np.linalg.lstsq(A1, t[~regime], rcond=None)
        (c, beta), *_ = np.linalg.lstsq(A2, t[regime], rcond=None)
        new = (c + beta * N) > (a + b * G)
        params = (a, b, c, beta)
        if (new == regime).all():
            break
        regime = new
    a, b, c, beta = params
    pred = np.maximum(a + b * G, c + beta * N)
    return dict(a=a, b=b, c=c, beta=beta, n_star=b / beta if beta > 0 else None,
                rel_rms=float(np.sqrt(np.mean(((pred - t) / t) ** 2))))


def run_regime_sweep(args):
    """Expert FFN time of G experts with n tokens each (d, f of a DeepSeek-V3 expert), through
    moe_expert_ffn; fits the max-affine model and reports the crossover n* = b / beta."""
    import statistics

    import torch

    import combine_warp_top_expert_b200 as moe
    import moe_synth
    d, f = args.regime_d, args.regime_f
    Gs = [1, 8, 32, 64, 148, 256]
    ns = [1, 8, 16, 32, 64, 96, 128, 160, 192, 224, 256, 320, 384, 512, 768, 1024]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    rows = []
    for G in Gs:
        wl = moe_synth.Workload("regime", T=1, d=d, E=G, k=1, f=f, R=1)
        dvw = moe_synth.device_inputs(wl)
        for n in ns:
            A = G * n
            shape = moe.Shape(T=A, d=d, E=G, k=1, f=f, R=1)
            xw = moe_synth.device_inputs(wl.with_(T=A, seed=1), weights=False)["x"]
            offs = (torch.arange(G + 1, dtype=torch.int32, device="cuda") * n).contiguous()
            y = torch.empty((A, d), dtype=torch.bfloat16, device="cuda")
            ws = moe.new_workspace(shape)
            ts = []
            for rep in range(3 + 5):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                moe.moe_expert_ffn(shape, xw, offs, dvw["w13"], dvw["w2"], None, None, None, y, None, ws)
                e1.record()
                torch.cuda.synchronize()
                if rep >= 3:
                    ts.append(e0.elapsed_time(e1))
            ms = statistics.median(ts)
            assert moe.get_status(ws) == 0
            rows.append(dict(G=G, n=n, N=A, ms=ms, tflops=6.0 * A * d * f / (ms * 1e-3) / 1e12,
                             weight_gbs=G * 3 * d * f * 2 / (ms * 1e-3) / 1e9))
            print(json.dumps(dict(regime_point=rows[-1])), flush=True)
            del xw, y, ws
        del dvw
        torch.cuda.empty_cache()
    full = [r for r in rows if r["G"] >= 32]  # enough experts to occupy every SM
    for name, key in (("tokens", lambda r: r["N"]), ("tile_rounded_tokens", lambda r: r["G"] * -(-r["n"] // 128) * 128)):
        fit = fit_max_affine([r["G"] for r in full], [key(r) for r in full], [r["ms"] for r in full])
        fit.update(d=d, f=f, unit="ms", N=name, model="t = max(a + b*G, c + beta*N), G >= 32",
                   b_gbs=3 * d * f * 2 / (fit["b"] * 1e-3) / 1e9,
                   beta_tflops=6.0 * d * f / (fit["beta"] * 1e-3) / 1e12)
        print(json.dumps(dict(regime_fit=fit)), flush=True)


DISPATCH_PATHS = {"auto": 0, "two_pass": 1, "one_pass": 2}


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def relaunch_command(gpus: int, argv, port: int):
    """The command that runs this benchmark as `gpus` ranks on this node (one process per GPU)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def rank_check(args, rank, world):
    """--rank-check: join the process group (gloo, no GPU), agree on the slowest rank's
    value, print one line per rank and leave; checks the multi-rank launch on any host."""
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        mx = max_over_ranks(100.0 * (rank + 1), world)
        launches = sum_over_ranks(5 * (rank + 1), world)
        mine = {"rank": rank, "world": world, "gpus": args.gpus, "max_ms": mx, "launches_all_ranks": launches,
                "seed": replica_seed(0, rank)}
        every = [None] * world
        dist.all_gather_object(every, mine)
        if rank == 0:  # one line for all ranks (the ranks share one output stream)
            print(json.dumps({"rank_check": every}), flush=True)
    finally:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gemm-policy", default="auto", choices=["auto", "single", "pair"],
                    help="grouped-GEMM tiles: chosen from the shape (auto), single-CTA 128-row, or CTA-pair 256x256 "
                         "(a group's last block of <= 128 rows as a half-height pair tile)")
    ap.add_argument("--dispatch-path", default="auto", choices=list(DISPATCH_PATHS),
                    help="dispatch: one kernel for small batches and two otherwise (auto), always the histogram "
                         "kernel + permute kernel (two_pass), or the one-pass kernel wherever it applies")
    ap.add_argument("--capacity-factor", type=float, default=None,
                    help="per-expert capacity ceil(C*T*k/E); excess assignments are dropped (default: none)")
    ap.add_argument("--regime-sweep", action="store_true",
                    help="sweep activated experts x tokens per expert and fit t = max(a + b*G, c + beta*N)")
    ap.add_argument("--regime-d", type=int, default=7168)
    ap.add_argument("--regime-f", type=int, default=2048)
    ap.add_argument("--gather", action="store_true",
                    help="no x_perm: dispatch writes indices only and the gate/up GEMM gathers rows of x itself")
    ap.add_argument("--seed", type=int, default=None,
                    help="seed of the synthetic inputs (default: the workload's; the router bias is calibrated "
                         "on the default seed)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's batch size T (smaller cases for profiling)")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch every kernel in plain stream order (no programmatic dependent launch)")
    ap.add_argument("--dense-compare", action="store_true",
                    help="our grouped GEMM on one expert holding every row against cuBLAS (torch.matmul) on the "
                         "same operands")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism across the --gpus ranks (E/R experts per GPU, rows exchanged over "
                         "NVLink inside dispatch and combine) instead of independent replicas")
    ap.add_argument("--sustain", type=float, default=0.0,
                    help="run the layer back to back for this many seconds, sampling SM clock and board power, "
                         "and report the steady-state throughput (one GPU)")
    ap.add_argument("--rank-check", action="store_true",
                    help="start the ranks, join a gloo process group, print one line per rank and exit (no GPU)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus < 1:
        sys.exit(f"--gpus must be >= 1, got {args.gpus}")
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        # one process per GPU: re-launch under torch.distributed.run with --gpus ranks
        r = subprocess.run(relaunch_command(args.gpus, sys.argv[1:], free_port()))
        sys.exit(r.returncode)
    if world_env is not None and int(world_env) != args.gpus:
        sys.exit(f"--gpus {args.gpus} does not match WORLD_SIZE={world_env}")

    if args.regime_sweep:
        run_regime_sweep(args)
        return
    if args.dense_compare:
        run_dense_compare(args)
        return
    import moe_synth
    wl = moe_synth.workload(args.config)
    if args.tokens is not None:
        wl = wl.with_(T=args.tokens)
    if args.seed is not None:
        wl = wl.with_(seed=args.seed)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.rank_check:
        rank_check(args, rank, world)
        return
    if args.sustain:
        run_sustain(args, wl)
        return
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.ep:
            run_gpu_ep(args, wl, rank, world, local_rank)
        else:
            run_gpu(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
