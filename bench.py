"""Throughput of the QSA sparse-attention step on B200, one JSON line on rank 0.

Default workload: decode at 64K cells -- every step appends n new cells
(qsa_cache_write) and runs qsa_decode for n = 1, 2, ..., 8 draft tokens
(36 tokens per step), top_k 2048, on synthetic inputs shaped like the model
the pages describe.  ``--config`` picks another workload (0-4); prefill
workloads report cells scored per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl reference]

Timing: W untimed steps, then K steps between a barrier and a device
synchronize on both sides, CUDA events on the launching stream, max over
ranks.  Each step reads a different one of 4 copies of the cache, so every
step's cache (80 MB at 64K cells) has left the 126 MB L2 since its last use.
Multi-GPU runs are independent replicas (the step has no exchange):
``value`` is the sum over ranks.
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
    "topk": "qsa_topk_cluster.cuh",
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
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


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

    wl, k_h, v_h, key_h = host_inputs(spec)
    caches = [qsa.DeviceCache.from_host(wl.cache, dev) for _ in range(ROTATE)]
    q = torch.from_numpy(wl.q).to(dev)
    iq = torch.from_numpy(wl.iq).to(dev)
    iw = torch.from_numpy(wl.iw).to(dev)
    kn = torch.from_numpy(k_h).to(dev)
    vn = torch.from_numpy(v_h).to(dev)
    keyn = torch.from_numpy(key_h).to(dev)
    nmax = max(spec.ns)
    if spec.kind == "decode":
        ws_bytes = max(qsa.workspace_bytes(qsa.MODE_DECODE, n, spec.L, spec.top_k, spec.nsplit)
                       for n in spec.ns)
    else:
        ws_bytes = qsa.workspace_bytes(qsa.MODE_PREFILL, spec.T, spec.pos0 + spec.T, spec.top_k)
    ws = qsa.workspace(ws_bytes, dev)
    out = torch.empty(nmax, 24, 256, dtype=torch.float32, device=dev)
    ids = torch.empty(nmax, spec.top_k, dtype=torch.int32, device=dev)

    def step(i, qq=q, iqq=iq, iww=iw, kk=kn, vv=vn, key=keyn, o=out):
        c = caches[i % ROTATE]
        for n in spec.ns:
            if spec.kind == "decode":
                qsa.cache_write(c, spec.L - n, kk[:n], vv[:n], key[:n])
                qsa.decode(c, spec.L, qq[:n], iqq[:n], iww[:n], spec.top_k, spec.nsplit, wl.scale,
                           ws=ws, out=o[:n], ids_out=ids[:n])
            else:
                qsa.cache_write(c, spec.pos0, kk, vv, key)
                qsa.prefill_chunk(c, spec.pos0, qq, iqq, iww, spec.top_k, wl.scale, ws=ws, out=o,
                                  ids_out=ids)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # ---- device-resident throughput: each step (all its calls) captured once per cache copy
    # in a CUDA graph, so the timed loop measures the kernels, not Python's launch overhead
    graphs, per_graph = [], 0
    for r in range(ROTATE):
        g = torch.cuda.CUDAGraph()
        before = qsa.launch_count()
        with torch.cuda.graph(g):
            step(r)
        per_graph = qsa.launch_count() - before
        graphs.append(g)
    for i in range(args.warmup):
        graphs[i % ROTATE].replay()
    torch.cuda.synchronize()
    if args.steps:
        steps = args.steps
    else:  # about two seconds of timed work, so the clock sampler sees the GPU under load
        probe0, probe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        probe0.record(stream)
        for i in range(2 * ROTATE):
            graphs[i % ROTATE].replay()
        probe1.record(stream)
        torch.cuda.synchronize()
        per_step = probe0.elapsed_time(probe1) / (2 * ROTATE)
        steps = int(max(20, min(100000, 2000.0 / max(per_step, 1e-3))))
        steps = int(dist_max(float(steps), world))
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for i in range(steps):
            graphs[i % ROTATE].replay()
        ev1.record(stream)
        torch.cuda.synchronize()
    launches = per_graph * steps
    ms = ev0.elapsed_time(ev1)
    barrier(world)
    value, ms_max = job_rate(spec.units, steps, ms, world)

    # ---- end to end through the public API from pinned host buffers
    q_h = torch.from_numpy(wl.q).pin_memory()
    iq_h = torch.from_numpy(wl.iq).pin_memory()
    iw_h = torch.from_numpy(wl.iw).pin_memory()
    kk_h = torch.from_numpy(k_h).pin_memory()
    vv_h = torch.from_numpy(v_h).pin_memory()
    key_hh = torch.from_numpy(key_h).pin_memory()
    out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    qd, iqd, iwd = torch.empty_like(q), torch.empty_like(iq), torch.empty_like(iw)
    kd, vd, keyd = torch.empty_like(kn), torch.empty_like(vn), torch.empty_like(keyn)
    h2d = sum(t.numel() * t.element_size() for t in (q_h, iq_h, iw_h, kk_h, vv_h, key_hh))
    d2h = 0
    for n in spec.ns:
        d2h += n * 24 * 256 * 4

    # each call's row views, made once (a caller with fixed buffers holds them)
    views = {n: (kd[:n], vd[:n], keyd[:n], qd[:n], iqd[:n], iwd[:n], out[:n], out_h[:n]) for n in spec.ns}

    def e2e_step(i):
        for dst, src in ((qd, q_h), (iqd, iq_h), (iwd, iw_h), (kd, kk_h), (vd, vv_h), (keyd, key_hh)):
            dst.copy_(src, non_blocking=True)
        c = caches[i % ROTATE]
        for n in spec.ns:
            if spec.kind == "decode":
                kn_, vn_, keyn_, qn_, iqn_, iwn_, outn_, outhn_ = views[n]
                qsa.cache_write(c, spec.L - n, kn_, vn_, keyn_)
                qsa.decode(c, spec.L, qn_, iqn_, iwn_, spec.top_k, spec.nsplit, wl.scale, ws=ws, out=outn_)
                outhn_.copy_(outn_, non_blocking=True)
            else:
                qsa.cache_write(c, spec.pos0, kd, vd, keyd)
                qsa.prefill_chunk(c, spec.pos0, qd, iqd, iwd, spec.top_k, wl.scale, ws=ws, out=out)
                out_h.copy_(out, non_blocking=True)

    for i in range(2):
        e2e_step(i)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(steps):
        e2e_step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    e2e_value, _ = job_rate(spec.units, steps, ev0.elapsed_time(ev1), world)

    # ---- per-kernel durations, step-level calls with events on the same stream
    kern = kernel_times(qsa, torch, spec, caches, wl, q, iq, iw, ws, dev, stream, 20)
    pk = peaks()
    roof = roofline(spec, kern, pk)

    line = {"metric": spec.metric, "value": value, "unit": spec.unit, "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_max / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": spec.name, "cells": spec.L, "top_k": spec.top_k,
                       "rows_per_call": spec.ns if spec.kind == "decode" else spec.T,
                       "nsplit": spec.nsplit if spec.kind == "decode" else "auto",
                       "l2": f"{ROTATE} rotating cache copies "
                             f"({ROTATE * spec.L * (CELL_BYTES + KEY_BYTES) / 1e6:.0f} MB > 126 MB L2)",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "e2e": {"value": e2e_value, "unit": spec.unit, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "roofline": roof["main"],
            "kernels": roof["kernels"],
            "clocks": clk.summary()}
    if spec.kind == "decode" and "score_attn" in roof:
        line["roofline_score_attn"] = roof["score_attn"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, cores, what, dt = oracle_sample(spec, wl, k_h, v_h, key_h, 15.0)
        line["cpu_baseline"] = {"value": val, "unit": spec.unit, "cores": cores, "kind": "oracle",
                                "sample": f"{what}, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def kernel_times(qsa, torch, spec, caches, wl, q, iq, iw, ws, dev, stream, reps):
    """Average duration of each step kernel, from CUDA events around the
    step-level calls (the same kernels qsa_decode / qsa_prefill_chunk launch)."""
    acc = {"index_score_kernel": 0.0, "topk": 0.0, "attn_kernel": 0.0, "merge_kernel": 0.0}
    count = {k: 0 for k in acc}
    info = {"union_cells": 0, "rows": 0, "cells_scored": 0, "ncells": 0, "nsplit": {}}
    ld_max = (spec.L + 3) // 4 * 4
    nmax = max(spec.ns)
    scores = torch.empty(nmax, ld_max, dtype=torch.float32, device=dev)
    tk_ws = qsa.workspace(qsa.topk_workspace_bytes(nmax, spec.L, spec.top_k), dev)
    ids = torch.empty(nmax, spec.top_k, dtype=torch.int32, device=dev)
    out = torch.empty(nmax, 24, 256, dtype=torch.float32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    parts = {}
    # Each call sits behind a ~1.5 ms torch sleep kernel so the host has queued all of
    # its launches before the first starts: the events bracket kernels, not launch gaps.
    for rep in range(reps + 2):
        c = caches[rep % ROTATE]
        for n in spec.ns:
            if spec.kind == "decode":
                vis0, ncells = spec.L - n + 1, spec.L
                ns = spec.nsplit or auto_nsplit(n, spec.top_k)
            else:
                vis0, ncells = spec.pos0 + 1, spec.pos0 + spec.T
                ns = auto_nsplit(n, spec.top_k)
            part = parts.setdefault((n, ns), torch.empty(n, 24, ns, 258, dtype=torch.float32, device=dev)
                                  if ns > 1 else None)
            torch.cuda._sleep(3_000_000)
            ev[0].record(stream)
            qsa.index_score(c, iq[:n], iw[:n], ncells, scores=scores[:n])
            ev[1].record(stream)
            qsa.topk(scores[:n], vis0, spec.top_k, ws=tk_ws, ids=ids[:n])
            ev[2].record(stream)
            res = qsa.attn(c, q[:n], ids[:n], ns, wl.scale, part=part, out=out[:n] if ns == 1 else None)
            ev[3].record(stream)
            if ns > 1:
                qsa.merge(res, out=out[:n])
            ev[4].record(stream)
            torch.cuda.synchronize()
            if rep < 2:
                continue
            names = list(acc)
            for j in range(4):
                if j == 3 and ns == 1:
                    continue
                acc[names[j]] += ev[j].elapsed_time(ev[j + 1])
                count[names[j]] += 1
            if rep == 2:
                idn = ids[:n].cpu().numpy()
                info["union_cells"] += int(np.unique(idn[idn >= 0]).size)
                info["rows"] += n
                info["cells_scored"] += int(sum(vis0 + r for r in range(n)))
                info["ncells"] += ncells * n
                info["nsplit"][n] = ns
    avg = {k: (acc[k] / count[k] if count[k] else None) for k in acc}
    return {"avg_ms": avg, "launches": count, "info": info, "reps": reps}


def auto_nsplit(rows, top_k):
    """The library's automatic split count (qsa_api.cu): 32 pieces for up to 8 rows,
    about 256 CTAs in all beyond."""
    want = 32 if rows <= 8 else 128 // rows
    return max(1, min(64, max(1, top_k // 32), want))


def roofline(spec, kern, pk):
    """Algorithmic bytes (or flops) per launch over measured launch time, for
    every step kernel; the dominant one (most time per call) is `main`."""
    info, avg = kern["info"], kern["avg_ms"]
    calls = len(spec.ns)
    hbm, tensor = pk["hbm_gbs"], pk["bf16_tflops"]
    rows = info["rows"] / calls
    ncells = info["ncells"] / calls                      # (row, cell) scores per call
    kernels = {}

    def hbm_entry(name, nbytes, note):
        ms = avg[name]
        if not ms:
            return None
        ach = nbytes / (ms / 1e3) / 1e9
        return {"kernel": name, "bound": "hbm", "ms": ms, "bytes_per_launch": nbytes, "achieved": ach,
                "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "note": note}

    # index score: keys once, scores written once (decode); prefill: 512 flops per visible cell
    key_bytes = spec.L * KEY_BYTES
    if spec.kind == "decode":
        kernels["index_score_kernel"] = hbm_entry("index_score_kernel", key_bytes + 4 * ncells,
                                                  "keys read once + fp32 scores written")
    else:
        ms = avg["index_score_kernel"]
        flops = 512.0 * info["cells_scored"] / calls
        ach = flops / (ms / 1e3) / 1e12
        kernels["index_score_kernel"] = {"kernel": "score_gemm_kernel (tcgen05)", "bound": "tensor", "ms": ms,
                                         "flops_per_launch": flops, "achieved": ach, "peak": tensor,
                                         "unit": "TFLOP/s", "frac": ach / tensor,
                                         "note": "512 flops per visible (row, cell); fp16 has bf16's nominal rate"}
    # selection: every visible score read, ids written
    kernels["topk"] = hbm_entry("topk", 4 * info["cells_scored"] / calls + 4 * rows * spec.top_k,
                                "visible scores read + ids written (decode: one cluster kernel; "
                                "prefill: histogram, filter and final kernels together)")
    # attention: the union of the rows' selected cells (K, V, scales) + queries, ids, outputs
    attn_bytes = (info["union_cells"] * CELL_BYTES + info["rows"] * (24 * 256 * 4 * 2 + spec.top_k * 4)) / calls
    kernels["attn_kernel"] = hbm_entry("attn_kernel", attn_bytes,
                                       "union of the rows' selected cells x 1088 B + q, ids, out"
                                       + (" (prefill: gathered from L2 mostly)" if spec.kind == "prefill" else ""))
    if avg["merge_kernel"]:
        ns = info["nsplit"]
        part_bytes = sum(n * 24 * ns[n] * 258 * 4 + n * 24 * 256 * 4 for n in ns) / calls
        kernels["merge_kernel"] = hbm_entry("merge_kernel", part_bytes, "partials read + output written")
    kernels = {k: v for k, v in kernels.items() if v}
    dom = max(kernels, key=lambda k: kernels[k]["ms"] or 0)
    main = dict(kernels[dom])
    main["peak_source"] = pk["source"]
    main["traffic"] = traffic_for(dom, spec.name)
    out = {"kernels": kernels, "main": main}
    if spec.kind == "decode":
        both_b = key_bytes + attn_bytes
        both_t = (avg["index_score_kernel"] + avg["attn_kernel"]) / 1e3
        out["score_attn"] = {"bound": "hbm", "achieved": both_b / both_t / 1e9, "peak": hbm, "unit": "GB/s",
                             "frac": both_b / both_t / 1e9 / hbm,
                             "note": "keys + union of selected cells over the two kernels' summed time"}
    return out


def main():
    args = parse()
    spec = Spec(args.config)
    if args.impl == "reference":
        run_reference(args, spec)
    else:
        run_cuda(args, spec)


if __name__ == "__main__":
    main()
