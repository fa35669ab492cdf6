"""Throughput of the QSA sparse-attention step on B200, one JSON line on rank 0.

Headline workload: decode at 64K cells -- every step runs qsa_decode for
n = 1, 2, ..., 8 draft tokens (36 tokens per step), each call appending its
n new cells itself, top_k 2048, on synthetic inputs shaped like the model the
pages describe.  The line's ``configs`` object holds the other workloads of
the metric, measured the same way: decode at 256K cells (64 splits) and the
two prompt chunks (cells scored per second).  ``--config`` picks another
headline workload (0-4), ``--configs`` the others.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--configs 2,3,4]
                    [--impl reference]

Timing: W untimed steps, then passes of exactly K steps, each between a
barrier and a device synchronize on both sides, CUDA events on the launching
stream, repeated until --min-seconds of device time (so the clock sampler sees
the GPU under load); the median pass counts, max over ranks.  Each step reads
a different one of 4 copies of the cache, so every step's cache (80 MB at 64K
cells) has left the 126 MB L2 since its last use.  Multi-GPU runs are
independent replicas (the step has no exchange): ``value`` is the sum over
ranks; ``--gpus N`` without torchrun around it starts the N ranks itself.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

ROTATE = 4
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = {
    "attn_kernel": "qsa_attn.cuh",
    "index_score_kernel": "qsa_index_score.cuh",
    "score_gemm_kernel": "qsa_score_gemm.cuh",
    "score_select_kernel": "qsa_prefill_select.cuh",
    "prefill_final_kernel": "qsa_prefill_select.cuh",
    "cluster_select_kernel+topk": "qsa_topk_cluster.cuh",
    "cluster_select_kernel": "qsa_topk_cluster.cuh",
    "merge_kernel": "qsa_merge.cuh",
}
CELL_BYTES = 2 * 2 * 256 + 2 * 2 * 8 * 2      # K + V codes and their scales, both KV heads
KEY_BYTES = 64 * 2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0 = per-workload default)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=1, choices=range(5))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--configs", default="2,3,4",
                    help="more workloads measured into the line's `configs` object ('none' for none)")
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="timed passes of --steps steps are repeated until this much device time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    a.configs = [] if a.configs in ("", "none") else [int(c) for c in a.configs.split(",")]
    return a


# ---------------------------------------------------------------- workloads

class Spec:
    """The per-step work of one workload."""

    def __init__(self, cfg: int):
        self.cfg = cfg
        c = synth.CONFIGS[cfg]
        self.kind = c["kind"]
        self.top_k = c["top_k"]
        self.L = c["L"]
        self.seed = 1000 + cfg
        if self.kind == "decode":
            self.ns = list(range(1, 9)) if cfg == 1 else [c["n"]]
            self.nsplit = c["nsplit"]
            self.units = sum(self.ns)                     # tokens per step
            self.metric, self.unit = "decode QSA tokens/s", "tokens/s"
        else:
            self.T, self.pos0 = c["T"], c["pos0"]
            self.ns = [self.T]
            self.nsplit = 0                               # the library's choice for T rows
            self.units = sum(self.pos0 + t + 1 for t in range(self.T))   # cells scored per step
            self.metric, self.unit = "prefill QSA cells-scored/s", "cells/s"
        self.name = synth.CONFIG_NAMES[cfg]


def host_inputs(spec: Spec):
    wl = synth.make_workload(spec.cfg)
    nmax = max(spec.ns)
    k, v, key = synth.make_new_cells(spec.seed + 7, nmax)
    return wl, k, v, key


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        mhz, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(mhz)}


# ---------------------------------------------------------------- peaks and traffic

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def source_hash(kernel: str) -> str:
    """Hash of the kernel's source without comments and blank space: edits to comments
    alone keep the recorded traffic, any change to the code drops it."""
    src = os.path.join(ROOT, "top_sparse_attention_score_b200", "csrc", KERNEL_SOURCES[kernel])
    code = re.sub(r"/\*.*?\*/", "", open(src).read(), flags=re.S)
    code = re.sub(r"//[^\n]*", "", code)
    code = "\n".join(line.strip() for line in code.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None if the
    kernel source changed since the counters were taken."""
    if not os.path.exists(TRAFFIC_FILE) or kernel not in KERNEL_SOURCES:
        return None
    t = json.load(open(TRAFFIC_FILE)).get(workload, {}).get(kernel)
    if not t or t.get("source_sha") != source_hash(kernel):
        return None
    return t["bytes_per_launch"]


# ---------------------------------------------------------------- distributed plumbing

def dist_init(n, backend: str = "nccl"):
    """Join the job's process group (one process per GPU; rendezvous from the
    torchrun environment).  Returns (rank, world, local rank); (0, 1, 0) alone."""
    if n <= 1 or "RANK" not in os.environ:
        return 0, 1, 0
    import datetime

    import torch
    import torch.distributed as dist
    local = int(os.environ.get("LOCAL_RANK", 0))
    if backend == "nccl":
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist.get_rank(), dist.get_world_size(), local


def dist_max(x: float, world: int) -> float:
    """The largest x over ranks (every rank calls it, in the same order)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def job_rate(units_per_step: float, steps: int, ms_local: float, world: int):
    """Whole-job throughput of `world` replicas that each ran `steps` steps of
    `units_per_step` units: all ranks' units over the slowest rank's time.
    Returns (units per second, the slowest rank's milliseconds)."""
    ms_max = dist_max(ms_local, world)
    return world * units_per_step * steps / (ms_max / 1000.0), ms_max


# ---------------------------------------------------------------- CPU oracle leg

def oracle_sample(spec: Spec, wl, k, v, key, budget_s: float):
    """Run the oracle on whole steps' rows until about budget_s seconds pass;
    return (units per second, cores, description)."""
    import oracle
    cores = os.cpu_count() or 1
    units = 0
    t0 = time.perf_counter()
    done_rows = 0
    while True:
        for n in spec.ns:
            if spec.kind == "decode":
                oracle.cache_write(wl.cache, spec.L - n, k[:n], v[:n], key[:n])
                w = synth.Workload(spec.name, "decode", wl.cache, spec.L, n, spec.L - n, spec.top_k,
                                   spec.nsplit, wl.scale, wl.q[:n], wl.iq[:n], wl.iw[:n])
                oracle.rows(w, threads=cores)
                units += n
                done_rows += n
            else:
                # prefill: a slice of the chunk's rows, counted in cells scored
                rows = np.arange(0, spec.T, max(1, spec.T // 16), dtype=np.int32)
                oracle.rows(wl, rows, threads=cores)
                units += int(sum(spec.pos0 + int(t) + 1 for t in rows))
                done_rows += rows.size
            if time.perf_counter() - t0 >= budget_s:
                dt = time.perf_counter() - t0
                what = (f"{done_rows} query rows of the workload (float64 oracle, OpenMP over rows)")
                return units / dt, cores, what, dt


def run_reference(args, spec: Spec):
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return
    wl, k, v, key = host_inputs(spec)
    for _ in range(args.warmup):
        oracle_sample(spec, wl, k, v, key, 0.0)
    steps = args.steps or 3
    vals = []
    t0 = time.perf_counter()
    for _ in range(steps):
        val, cores, what, _ = oracle_sample(spec, wl, k, v, key, 0.0)
        vals.append(val)
    total = time.perf_counter() - t0
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": spec.metric, "value": value, "unit": spec.unit,
            "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
            "ms_per_step": 1000 * total / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec.name, "cells": spec.L, "top_k": spec.top_k},
            "cpu_baseline": {"value": value, "unit": spec.unit, "cores": cores, "kind": "oracle",
                             "sample": f"each step: {what}"},
            "e2e": {"value": value, "unit": spec.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- CUDA leg

def _packed(torch, arrays, device=None, pin=False):
    """One contiguous byte buffer holding `arrays` (numpy), each piece 256-byte aligned;
    returns (buffer, views in the arrays' dtypes and shapes)."""
    offs, at = [], 0
    for a in arrays:
        offs.append(at)
        at = (at + a.nbytes + 255) // 256 * 256
    buf = torch.empty(max(at, 16), dtype=torch.uint8, device=device or "cpu")
    if pin:
        buf = buf.pin_memory()
    views = []
    for a, o in zip(arrays, offs):
        v = buf[o:o + a.nbytes].view(getattr(torch, str(a.dtype))).view(*a.shape)
        views.append(v)
    return buf, views


class Workload:
    """Device state of one workload: rotating cache copies, packed step inputs, outputs."""

    def __init__(self, torch, qsa, spec, dev):
        self.spec = spec
        wl, k_h, v_h, key_h = host_inputs(spec)
        self.wl, self.k_h, self.v_h, self.key_h = wl, k_h, v_h, key_h
        self.caches = [qsa.DeviceCache.from_host(wl.cache, dev) for _ in range(ROTATE)]
        rows = max(spec.ns)
        host = [np.ascontiguousarray(x) for x in (wl.q[:rows], wl.iq[:rows], wl.iw[:rows], k_h[:rows],
                                                   v_h[:rows], key_h[:rows])]
        self.h_buf, hv = _packed(torch, host, pin=True)
        for view, a in zip(hv, host):
            view.copy_(torch.from_numpy(a))
        # two device sets of inputs and outputs (and two pinned output buffers), so the
        # end-to-end run copies one step's data while the neighbouring step computes
        self.out_rows = sum(spec.ns)
        self.d_bufs, self.call_sets, self.outs, self.outs_h = [], [], [], []
        for _ in range(2):
            d_buf, (q, iq, iw, kn, vn, keyn) = _packed(torch, host, dev)
            d_buf.copy_(self.h_buf)
            out = torch.empty(self.out_rows, 24, 256, dtype=torch.float32, device=dev)
            calls, at = [], 0
            for n in spec.ns:  # each call's views, made once (a caller with fixed buffers holds them)
                calls.append((n, q[:n], iq[:n], iw[:n], (kn[:n], vn[:n], keyn[:n]), out[at:at + n]))
                at += n
            self.d_bufs.append(d_buf)
            self.call_sets.append(calls)
            self.outs.append(out)
            self.outs_h.append(torch.empty(out.shape, dtype=torch.float32).pin_memory())
        self.calls, self.out = self.call_sets[0], self.outs[0]
        if spec.kind == "decode":
            nbytes = max(qsa.workspace_bytes(qsa.MODE_DECODE, n, spec.L, spec.top_k, spec.nsplit) for n in spec.ns)
        else:
            nbytes = qsa.workspace_bytes(qsa.MODE_PREFILL, spec.T, spec.pos0 + spec.T, spec.top_k)
        self.ws = qsa.workspace(nbytes, dev)
        self.h2d_bytes = int(self.h_buf.numel())
        self.d2h_bytes = int(self.out.numel() * 4)

    def step(self, qsa, i, b=0):
        """One step: every call of the workload through the public API, each appending
        its rows' own cells in the same call (cache copy i % ROTATE, input and output set b)."""
        spec, c = self.spec, self.caches[i % ROTATE]
        for n, q, iq, iw, app, out in self.call_sets[b]:
            if spec.kind == "decode":
                qsa.decode(c, spec.L, q, iq, iw, spec.top_k, spec.nsplit, self.wl.scale, ws=self.ws, out=out,
                           append=app)
            else:
                qsa.prefill_chunk(c, spec.pos0, q, iq, iw, spec.top_k, self.wl.scale, ws=self.ws, out=out,
                                  append=app)


def measure(torch, qsa, spec, args, dev, stream, world, local, with_cpu):
    """Device-resident rate (CUDA graphs of whole steps), end-to-end rate from pinned host
    buffers, per-kernel times and the roofline of one workload."""
    w = Workload(torch, qsa, spec, dev)
    for i in range(args.warmup):
        w.step(qsa, i)
    torch.cuda.synchronize()

    # ---- device-resident: each step captured once per cache copy in a CUDA graph
    graphs, per_graph = [], 0
    for r in range(ROTATE):
        g = torch.cuda.CUDAGraph()
        before = qsa.launch_count()
        with torch.cuda.graph(g):
            w.step(qsa, r)
        per_graph = qsa.launch_count() - before
        graphs.append(g)
    for i in range(max(args.warmup, ROTATE)):
        graphs[i % ROTATE].replay()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed_pass(k, fn):
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        for i in range(k):
            fn(i)
        ev1.record(stream)
        torch.cuda.synchronize()
        return ev0.elapsed_time(ev1)

    replay = lambda i: graphs[i % ROTATE].replay()  # noqa: E731
    if args.steps:
        steps = args.steps
    else:  # about a quarter second per pass
        per_step = timed_pass(2 * ROTATE, replay) / (2 * ROTATE)
        steps = int(dist_max(float(max(20, min(100000, 250.0 / max(per_step, 1e-3)))), world))
    # Passes of exactly `steps` steps until at least min_seconds of timed work, so the clock
    # sampler sees the GPU under load; the median pass is reported.
    first = timed_pass(steps, replay)
    passes = int(dist_max(float(max(3, min(10000, -(-args.min_seconds * 1000.0 // max(first, 1e-3))))), world))
    with ClockSampler(local) as clk:
        times = [timed_pass(steps, replay) for _ in range(passes)]
    ms_pass = statistics.median(times)
    value, ms_max = job_rate(spec.units, steps, ms_pass, world)
    for g in graphs:
        g.reset()
    del graphs

    # ---- end to end through the public API: per step one copy of the packed inputs from
    # pinned host memory, the calls (each appending its rows' cells), one copy of all outputs
    # back into pinned host memory.  The copies run on two copy streams (in and out) with two
    # input / output sets, so step i + 1's inputs arrive and step i - 1's outputs leave while
    # step i computes; every copy of every step is inside the timed region.
    cs_in, cs_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_h2d, ev_comp, ev_d2h = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_pass(k):
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        cs_in.wait_event(ev0)
        cs_out.wait_event(ev0)
        for i in range(k):
            b = i & 1
            with torch.cuda.stream(cs_in):
                if i >= 2:
                    cs_in.wait_event(ev_comp[b])  # step i - 2 has read this input set
                w.d_bufs[b].copy_(w.h_buf, non_blocking=True)
                ev_h2d[b].record(cs_in)
            stream.wait_event(ev_h2d[b])
            if i >= 2:
                stream.wait_event(ev_d2h[b])  # step i - 2's outputs have left this output set
            w.step(qsa, i, b)
            ev_comp[b].record(stream)
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(ev_comp[b])
                w.outs_h[b].copy_(w.outs[b], non_blocking=True)
                ev_d2h[b].record(cs_out)
        for b in range(min(k, 2)):
            stream.wait_event(ev_d2h[b])
        ev1.record(stream)
        torch.cuda.synchronize()
        return ev0.elapsed_time(ev1)

    e2e_pass(4)
    e2e_times = [e2e_pass(steps) for _ in range(3)]
    e2e_value, _ = job_rate(spec.units, steps, statistics.median(e2e_times), world)

    # the same with each step's copies and calls back to back on one stream (no overlap)
    def serial_step(i):
        w.d_bufs[0].copy_(w.h_buf, non_blocking=True)
        w.step(qsa, i, 0)
        w.outs_h[0].copy_(w.outs[0], non_blocking=True)

    timed_pass(2, serial_step)
    serial_times = [timed_pass(steps, serial_step) for _ in range(3)]
    serial_value, _ = job_rate(spec.units, steps, statistics.median(serial_times), world)

    # ---- per-kernel durations, step-level calls with events on the same stream
    kern = kernel_times(qsa, torch, w, spec, stream, 20)
    roof = roofline(spec, kern, peaks())
    res = {"metric": spec.metric, "value": value, "unit": spec.unit, "ms_per_step": ms_max / steps,
           "steps": steps, "passes": passes,
           "config": {"workload": spec.name, "cells": spec.L, "top_k": spec.top_k,
                      "rows_per_call": spec.ns if spec.kind == "decode" else spec.T,
                      "nsplit": spec.nsplit if spec.kind == "decode" else "auto",
                      "l2": f"{ROTATE} rotating cache copies "
                            f"({ROTATE * spec.L * (CELL_BYTES + KEY_BYTES) / 1e6:.0f} MB > 126 MB L2)",
                      "timing": f"median of {passes} passes of {steps} graph-replayed steps"},
           "e2e": {"value": e2e_value, "unit": spec.unit, "h2d_bytes_per_step": w.h2d_bytes,
                   "d2h_bytes_per_step": w.d2h_bytes, "serial_value": serial_value,
                   "api": "per step one H2D copy of the packed inputs from pinned memory, one call per row "
                          "group appending its cells (qsa_decode / qsa_prefill_chunk with append), one D2H "
                          "copy of the outputs to pinned memory; copies on an input and an output copy stream, "
                          "double-buffered, overlapping the neighbouring steps' calls (serial_value: copies and "
                          "calls of each step back to back on one stream)"},
           "gpu_launches": per_graph * steps,
           "roofline": roof["main"], "kernels": roof["kernels"], "clocks": clk.summary()}
    if "score_attn" in roof:
        res["roofline_score_attn"] = roof["score_attn"]
    if "score_gemm" in roof:
        res["roofline_score_gemm"] = roof["score_gemm"]
    if with_cpu:
        val, cores, what, dt = oracle_sample(spec, w.wl, w.k_h, w.v_h, w.key_h, 15.0)
        res["cpu_baseline"] = {"value": val, "unit": spec.unit, "cores": cores, "kind": "oracle",
                               "sample": f"{what}, {dt:.1f} s"}
    del w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_cuda(args, spec: Spec):
    import torch

    from top_sparse_attention_score_b200 import build as pkg_build
    from top_sparse_attention_score_b200 import qsa

    rank, world, local = dist_init(args.gpus)
    if rank == 0:
        pkg_build.build()
    barrier(world)
    qsa.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    head = measure(torch, qsa, spec, args, dev, stream, world, local,
                   with_cpu=rank == 0 and world == 1 and not args.no_cpu_baseline)
    extra = {}
    for cfg in args.configs:
        if cfg == spec.cfg:
            continue
        sub = measure(torch, qsa, Spec(cfg), args, dev, stream, world, local, with_cpu=False)
        extra[sub["config"]["workload"]] = sub

    line = {"metric": head["metric"], "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": head["steps"], "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic", "config": dict(head["config"],
                                                parallelism="replicas" if world > 1 else "single GPU"),
            "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "roofline": head["roofline"],
            "kernels": head["kernels"], "clocks": head["clocks"]}
    for key in ("roofline_score_attn", "roofline_score_gemm", "cpu_baseline"):
        if key in head:
            line[key] = head[key]
    if extra:
        line["configs"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def kernel_times(qsa, torch, w, spec, stream, reps):
    """Average device time of every kernel the step's calls launch, per launch, from the
    library's own trace events (qsa_trace_begin / qsa_trace_end) around the real calls."""
    acc, count = {}, {}
    info = {"union_cells": 0, "gathered_cells": 0, "rows": 0, "cells_scored": 0, "ncells": 0, "nsplit": {},
            "calls": 0}
    ids = torch.empty(max(spec.ns), spec.top_k, dtype=torch.int32, device=w.out.device)
    # Each call sits behind a ~1.5 ms torch sleep kernel so the host has queued all of its
    # launches before the first starts: the events bracket kernels, not launch gaps.
    for rep in range(reps + 2):
        c = w.caches[rep % ROTATE]
        for n, q, iq, iw, app, out in w.calls:
            torch.cuda._sleep(3_000_000)
            with qsa.trace(stream=torch.cuda.current_stream()) as tr:
                if spec.kind == "decode":
                    qsa.decode(c, spec.L, q, iq, iw, spec.top_k, spec.nsplit, w.wl.scale, ws=w.ws, out=out,
                               ids_out=ids[:n], append=app)
                else:
                    qsa.prefill_chunk(c, spec.pos0, q, iq, iw, spec.top_k, w.wl.scale, ws=w.ws, out=out,
                                      ids_out=ids[:n], append=app)
            if rep < 2:
                continue
            for name, ms in tr.kernels:
                acc[name] = acc.get(name, 0.0) + ms
                count[name] = count.get(name, 0) + 1
            if rep == 2:
                vis0 = spec.L - n + 1 if spec.kind == "decode" else spec.pos0 + 1
                ncells = spec.L if spec.kind == "decode" else spec.pos0 + spec.T
                idn = ids[:n].cpu().numpy()
                info["union_cells"] += int(np.unique(idn[idn >= 0]).size)
                info["gathered_cells"] += int((idn >= 0).sum())
                info["rows"] += n
                info["cells_scored"] += int(sum(vis0 + r for r in range(n)))
                info["ncells"] += ncells * n
                info["nsplit"][n] = spec.nsplit or auto_nsplit(n, spec.top_k)
                info["calls"] += 1
    avg = {k: acc[k] / count[k] for k in acc}
    per_call = {k: count[k] / (reps * len(spec.ns)) for k in acc}  # launches of each kernel per call
    return {"avg_ms": avg, "launches_per_call": per_call, "info": info, "reps": reps}


def auto_nsplit(rows, top_k):
    """The library's automatic split count (qsa_api.cu): 32 pieces for up to 8 rows,
    about 256 CTAs in all beyond."""
    want = 32 if rows <= 8 else 128 // rows
    return max(1, min(64, max(1, top_k // 32), want))


SELECTION_KERNELS = ("cluster_select_kernel", "topk_zero_kernel", "topk_hist_kernel", "topk_filter_kernel",
                     "topk_final_kernel")


def roofline(spec, kern, pk):
    """Algorithmic bytes (or flops) per launch over measured launch time, for every step
    kernel; the dominant one (most time per call) is `main`."""
    info, avg, per_call = kern["info"], kern["avg_ms"], kern["launches_per_call"]
    calls = max(1, info["calls"])
    hbm, tensor = pk["hbm_gbs"], pk["bf16_tflops"]
    rows = info["rows"] / calls
    ncells = info["ncells"] / calls                      # (row, cell) scores per call
    cells_scored = info["cells_scored"] / calls          # visible (row, cell) pairs per call
    kernels = {}

    def hbm_entry(name, nbytes, note):
        ms = avg.get(name)
        if not ms:
            return
        ach = nbytes / (ms / 1e3) / 1e9
        kernels[name] = {"kernel": name, "bound": "hbm", "ms": ms, "bytes_per_launch": nbytes, "achieved": ach,
                         "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "note": note}

    key_bytes = spec.L * KEY_BYTES
    attn_bytes = (info["union_cells"] * CELL_BYTES + info["rows"] * (24 * 256 * 4 * 2 + spec.top_k * 4)) / calls
    hbm_entry("index_score_kernel", key_bytes + 4 * ncells,
              "keys read once + fp32 scores written (the call's new cells quantized in the same launch)")
    sel = [k for k in SELECTION_KERNELS if k in avg]
    if sel:  # the decode selection: one cluster kernel, or the multi-kernel path for long rows
        ms = sum(avg[k] * per_call[k] for k in sel)
        nbytes = 4 * cells_scored + 4 * rows * spec.top_k
        ach = nbytes / (ms / 1e3) / 1e9
        kernels["selection"] = {"kernel": "+".join(sel), "bound": "hbm", "ms": ms, "bytes_per_launch": nbytes,
                                "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                                "note": "visible scores read + ids written"}
    if "score_select_kernel" in avg:
        ms = avg["score_select_kernel"]
        flops = 512.0 * cells_scored
        ach = flops / (ms / 1e3) / 1e12
        kernels["score_select_kernel"] = {
            "kernel": "score_select_kernel (tcgen05)", "bound": "tensor", "ms": ms, "flops_per_launch": flops,
            "achieved": ach, "peak": tensor, "unit": "TFLOP/s", "frac": ach / tensor,
            "note": "512 flops per visible (row, cell); fp16 has bf16's nominal rate; candidates only written"}
    hbm_entry("prefill_threshold_kernel", key_bytes / 16 + 16 * rows,
              "every 16th key (the sample) + thresholds; the sampled keys are re-read from L2 per 8 rows")
    hbm_entry("prefill_final_kernel", 4 * rows * spec.top_k,
              "ids written (the candidate lists are read from L2)")
    hbm_entry("cache_write_kernel", rows * (2 * 2 * 256 * 4 + 128 + CELL_BYTES + KEY_BYTES),
              "new cells: fp32 K/V and fp16 keys read, int8 codes, fp16 scales and keys written")
    hbm_entry("attn_kernel", attn_bytes, "union of the rows' selected cells x 1088 B + q, ids, out"
              + (" (prefill: gathered from L2 mostly)" if spec.kind == "prefill" else ""))
    if "attn_kernel" in kernels and spec.kind == "prefill":
        # every (row, selected cell) gathers 1088 B (both KV heads' codes and scales), most of it
        # from L2: the rate the prompt-chunk attention sustains on its gathers
        gathered = info["gathered_cells"] / calls * CELL_BYTES
        kernels["attn_kernel"]["gathered_bytes_per_launch"] = gathered
        kernels["attn_kernel"]["gather_gbs"] = gathered / (kernels["attn_kernel"]["ms"] / 1e3) / 1e9
    if "merge_kernel" in avg:
        ns = info["nsplit"]
        part_bytes = sum(n * 24 * ns[n] * 258 * 4 + n * 24 * 256 * 4 for n in ns) / calls
        hbm_entry("merge_kernel", part_bytes, "partials read + output written")
    # per call: a kernel's time times its launches per call
    for k, v in kernels.items():
        v["ms_per_call"] = v["ms"] * (1 if k == "selection" else per_call.get(k, 1))
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_call"])
    main = dict(kernels[dom])
    main["peak_source"] = pk["source"]
    main["traffic"] = traffic_for(main["kernel"].split(" ")[0], spec.name)
    out = {"kernels": kernels, "main": main}
    if spec.kind == "decode" and "index_score_kernel" in avg and "attn_kernel" in avg:
        both_b = key_bytes + attn_bytes
        both_t = (avg["index_score_kernel"] + avg["attn_kernel"]) / 1e3
        out["score_attn"] = {"bound": "hbm", "achieved": both_b / both_t / 1e9, "peak": hbm, "unit": "GB/s",
                             "frac": both_b / both_t / 1e9 / hbm,
                             "note": "keys + union of selected cells over the two kernels' summed time"}
    if "score_select_kernel" in kernels:
        out["score_gemm"] = dict(kernels["score_select_kernel"], peak_source=pk["source"])
    return out


def main():
    args = parse()
    if args.gpus > 1 and "RANK" not in os.environ:
        sys.exit(relaunch(args))
    spec = Spec(args.config)
    if args.impl == "reference":
        run_reference(args, spec)
    else:
        run_cuda(args, spec)


if __name__ == "__main__":
    main()
