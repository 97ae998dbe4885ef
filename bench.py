#!/usr/bin/env python
"""Benchmark of paged MLA latent-attention decode on B200.

One step = one decode step of a model's MLA stack: ``--layers`` (default 24)
calls of ``mla_decode``, each over its own layer's paged KV cache, for the
same batch of query rows.  24 layers x 142,000 positions x 576 FP8 bytes is
the per-GPU MLA payload the Kimi K3 page quotes ("Inside Kimi K3 optimisation
work", section 1, DCP), so the default workload, ``long_ctx_142k`` (B=1, T=1,
H=96, 142,000 cached positions, FP8 e4m3 with per-token scale), reads 1.98 GB
of KV per step; that is larger than the 126 MB L2, so every layer's cache
comes from HBM.

Prints one JSON line (rank 0).  ``value`` is KV-read GB/s of the whole job:
the bytes of all cached positions each query row sees (read once per layer),
over the device time of the timed steps.  ``--impl reference`` times the fp64
CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import shutil
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mla_workloads as W  # noqa: E402

METRIC = "MLA decode KV-read GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_ctx_142k", choices=W.CONFIG_ORDER)
    ap.add_argument("--kv", choices=[W.KV_BF16, W.KV_FP8], default=None)
    ap.add_argument("--T", type=int, default=None, help="query tokens per sequence (1 + drafts), 1..8")
    ap.add_argument("--static-scale", action="store_true",
                    help="FP8 cache with one per-tensor scale instead of one per position")
    ap.add_argument("--layers", type=int, default=24)
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tcgen05"])
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-append", dest="append", action="store_false",
                    help="skip timing the cache writer (mla_append_kv) on the workload's new tokens")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# bookkeeping shared by both arms
# ----------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = ("mla_latent_attention_b200/csrc/mla_tc.cu", "mla_latent_attention_b200/csrc/mla_common.cuh",
                  "mla_latent_attention_b200/csrc/tc_ptx.cuh")


def kernel_source_hash() -> str:
    """Hash of the attention kernel's sources with comments and blank space
    removed, so that editing a comment does not orphan a recorded capture."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kv: str):
    """DRAM bytes per launch of the attention kernel from an ncu capture,
    recorded in profiles/ncu_traffic.txt as
    ``<workload> <kv> <kernel source hash> <dram read+write bytes per launch>``.
    None when there is no capture for the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    try:
        with open(path) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    want = kernel_source_hash()
    for ln in lines:
        parts = ln.split()
        if len(parts) == 4 and not ln.startswith("#") and parts[0] == workload and parts[1] == kv \
                and parts[2] == want:
            return float(parts[3])
    return None


def make_bench_workload(args, device="cpu"):
    w = W.make_workload(args.workload, device=device, kv=args.kv, T=args.T)
    if args.static_scale:
        w = W.static_scale_workload(w)
    return w


def visible_positions(w) -> int:
    """Sum over query rows' distinct sequences of cached positions read once
    per layer (each sequence's pages are read once for all its rows)."""
    return int(w.ctx_lens.to(torch.int64).sum())


def step_units(w, layers):
    pos = visible_positions(w)
    kv_bytes = pos * w.kv_bytes_per_position() * layers
    R = w.T * w.H
    q_bytes = w.B * R * (512 + 64) * 2 * layers
    out_bytes = w.B * R * (512 * 2 + 4) * layers
    # flops: 2*576 (scores) + 2*512 (values) per (row, visible position)
    if w.vis_lens is not None:
        vis = int(w.vis_lens.to(torch.int64).sum()) * w.H
    else:
        ctx = w.ctx_lens.to(torch.int64)
        vis = int(sum(int(c) - w.T + t + 1 for c in ctx for t in range(w.T))) * w.H
    flops = 2176 * vis * layers
    return dict(kv_bytes=kv_bytes, total_bytes=kv_bytes + q_bytes + out_bytes, flops=flops,
                seqs=w.B)


def max_over_ranks(seconds: float, world: int, device) -> float:
    """The largest of every rank's time (each rank passes its own); the
    value itself with one rank.  Every rank must call it at the same point."""
    if world <= 1:
        return float(seconds)
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def workload_config(args, w, units, kernel, parallelism):
    """The bench line's ``config``: the same keys for both arms."""
    return {"workload": args.workload, "B": w.B, "T": w.T, "H": w.H, "ctx": int(w.ctx_lens.max()),
            "kv": w.kv_label(), "layers": args.layers, "kernel": kernel, "num_splits": args.num_splits,
            "parallelism": parallelism,
            "l2": f"inputs larger than L2: {args.layers} layer caches, "
                  f"{units['kv_bytes'] / 1e9:.2f} GB of KV per step"}


_LIBCUDA = None


def event_ms(a, b) -> float:
    """Elapsed ms between two recorded CUDA events, through the driver API
    (works for event-record nodes of a replayed CUDA graph, which torch's
    Event.elapsed_time refuses)."""
    import ctypes
    global _LIBCUDA
    if _LIBCUDA is None:
        _LIBCUDA = ctypes.CDLL("libcuda.so.1")
        _LIBCUDA.cuEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p,
                                                ctypes.c_void_p]
    ms = ctypes.c_float(0.0)
    rc = _LIBCUDA.cuEventElapsedTime(ctypes.byref(ms), ctypes.c_void_p(a.cuda_event),
                                     ctypes.c_void_p(b.cuda_event))
    if rc != 0:
        raise RuntimeError(f"cuEventElapsedTime failed with CUresult {rc}")
    return float(ms.value)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        exe = shutil.which("nvidia-smi")
        if exe is None:
            return
        self.proc = subprocess.Popen(
            [exe, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
             "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, flag in zip(names, parts[4:8]):
                if flag.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * max(sm)]
        busy.sort()
        return {"sm_mhz": busy[len(busy) // 2], "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(w, layers, seconds):
    """Time the fp64 oracle on a bounded sample of rows of one layer.

    Rows are taken whole (every visible position of each sampled row), in
    batches of one row per core, until about ``seconds`` of wall time; the
    time per full step is extrapolated by rows: layers * B*T*H / rows done."""
    import oracle
    lib = oracle.load()
    wc = w.to("cpu")
    total_rows = wc.B * wc.T * wc.H
    threads = cpu_threads()
    rows_done, t_spent, start = 0, 0.0, 0
    gen = torch.Generator().manual_seed(5)
    order = torch.randperm(total_rows, generator=gen)
    while t_spent < seconds and rows_done < total_rows:
        batch = order[start:start + threads]
        start += threads
        t0 = time.perf_counter()
        oracle.decode_workload(wc, rows=batch, threads=threads, lib=lib)
        t_spent += time.perf_counter() - t0
        rows_done += int(batch.numel())
    step_time = t_spent * layers * total_rows / rows_done
    return step_time, rows_done, t_spent, threads


# ----------------------------------------------------------------------------
# reference arm: the oracle on host cores
# ----------------------------------------------------------------------------
def run_reference(args, rank, world):
    if rank != 0:
        return
    w = make_bench_workload(args)
    units = step_units(w, args.layers)
    steps = args.steps if args.steps is not None else 3
    budget = max(0.5, 120.0 / (steps + args.warmup))   # whole run within ~2 minutes
    times = []
    info = None
    for i in range(args.warmup + steps):
        st, rows, spent, threads = oracle_sample(w, args.layers, budget)
        if i >= args.warmup:
            times.append(st)
            info = (rows, spent, threads)
    step_time = sum(times) / len(times)
    value = units["kv_bytes"] / step_time / 1e9
    rows, spent, threads = info
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 1,
        "steps": steps, "warmup": args.warmup, "ms_per_step": step_time * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(args, w, units, "oracle", "oracle on host cores"),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} whole query rows of one layer per step "
                                   f"({spent:.1f} s), extrapolated to {args.layers} layers x "
                                   f"{w.B * w.T * w.H} rows"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def time_append(mla, w, kv, sc, L, stream, reps=50):
    """The cache writer on its own: each layer's T new tokens per sequence
    written (and, for an FP8 cache, quantised) by one mla_append_kv, the L
    launches captured as a graph and replayed ``reps`` times."""
    dev = w.q_lat.device
    gen = torch.Generator(device=dev)
    gen.manual_seed(31)
    c_new = torch.randn((w.B, w.T, W.D_LATENT), generator=gen, device=dev).to(torch.bfloat16)
    k_new = torch.randn((w.B, w.T, W.D_ROPE), generator=gen, device=dev).to(torch.bfloat16)

    def step():
        for i in range(L):
            mla.append_kv(c_new, k_new, kv[i], None if sc is None else sc[i], w.page_table, w.ctx_lens)

    step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / (reps * L)
    tokens = w.B * w.T
    # bf16 values in; the stored form out (FP8 codes and, per position, the scale; or bf16)
    out_bytes = w.kv_bytes_per_position()
    nbytes = tokens * (2 * W.D_QK + out_bytes)
    return {"us_per_launch": us, "tokens_per_launch": tokens, "bytes_per_launch": nbytes,
            "achieved_gbs": nbytes / us / 1e3, "launches": reps * L,
            "note": "one launch per layer, timed apart from the decode step"}


def run_ours(args, rank, world, local_rank):
    import mla_latent_attention_b200 as mla
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = make_bench_workload(args, device=dev)
    L = args.layers
    units = step_units(w, L)
    # each layer: its own copy of the paged cache (same contents, own memory)
    kv = [w.kv_pages] + [w.kv_pages.clone() for _ in range(L - 1)]
    sc = None if w.kv_scale is None else [w.kv_scale] + [w.kv_scale.clone() for _ in range(L - 1)]
    B, T, H = w.B, w.T, w.H
    q_lat = torch.stack([w.q_lat] * L)          # [L,B,T,H,512]
    q_pe = torch.stack([w.q_pe] * L)
    outs = torch.empty((L, B, T, H, 512), dtype=torch.bfloat16, device=dev)
    lses = torch.empty((L, B, T, H), dtype=torch.float32, device=dev)
    dims = mla.make_dims(w.q_lat, w.kv_pages, w.page_table, kernel=args.kernel,
                         num_splits=args.num_splits)
    ws_bytes = mla.workspace_size(dims)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    launches_per_call = 2 if ws_bytes > 256 else 1
    ev_a = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(L)]
    ev_m = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(L)]
    ev_b = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(L)]

    def one_step(timed_events):
        for i in range(L):
            if timed_events:
                ev_a[i].record()
            mla.decode(q_lat[i], q_pe[i], kv[i], None if sc is None else sc[i], w.page_table,
                       w.ctx_lens, w.sm_scale, out=outs[i], lse=lses[i], kernel=args.kernel,
                       num_splits=args.num_splits, workspace=ws,
                       stage_event=ev_m[i] if timed_events else None)
            if timed_events:
                ev_b[i].record()

    # torch creates CUDA events lazily: record each once so its handle exists
    # before it is handed to the library or captured
    for e in ev_a + ev_m + ev_b:
        e.record()
    # eager warm-up (sets kernel attributes), then capture one step as a graph;
    # a second graph of the same step carries per-layer event nodes, for the
    # per-kernel durations only (event nodes are kept out of the timed graph)
    one_step(False)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    graph = torch.cuda.CUDAGraph()
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            one_step(False)
        with torch.cuda.graph(graph_ev, stream=stream):
            one_step(True)
    torch.cuda.synchronize()
    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    graph.replay()
    torch.cuda.synchronize()
    est = time.perf_counter() - t0
    steps = args.steps if args.steps is not None else max(10, min(20000, int(3.0 / max(est, 1e-6))))

    sampler = ClockSampler(local_rank)
    sampler.start()
    # keep the GPU busy ~0.5 s so clock samples reflect load, untimed
    t_end = time.perf_counter() + 0.5
    while time.perf_counter() < t_end:
        graph.replay()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        graph.replay()
    stop.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    elapsed = start.elapsed_time(stop) / 1e3
    # per-kernel durations: steps of the graph with event nodes, read one by one
    dec, mer = [], []
    for _ in range(12):
        graph_ev.replay()
        torch.cuda.synchronize()
        dec += [event_ms(ev_a[i], ev_m[i]) / 1e3 for i in range(L)]
        mer += [event_ms(ev_m[i], ev_b[i]) / 1e3 for i in range(L)]
    clocks = sampler.stop()

    max_elapsed = max_over_ranks(elapsed, world, dev)

    # end to end through the public API with host buffers: per step the query
    # rows of every layer go host->device and the outputs come back.
    h_qlat = torch.empty(q_lat.shape, dtype=q_lat.dtype, pin_memory=True).copy_(q_lat)
    h_qpe = torch.empty(q_pe.shape, dtype=q_pe.dtype, pin_memory=True).copy_(q_pe)
    h_out = torch.empty(outs.shape, dtype=outs.dtype, pin_memory=True)
    h_lse = torch.empty(lses.shape, dtype=lses.dtype, pin_memory=True)
    e2e_steps = max(3, min(steps, 200))
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        q_lat.copy_(h_qlat, non_blocking=True)
        q_pe.copy_(h_qpe, non_blocking=True)
        one_step(False)
        h_out.copy_(outs, non_blocking=True)
        h_lse.copy_(lses, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_time = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    e2e_value = world * e2e_steps * units["kv_bytes"] / e2e_time / 1e9
    h2d = (h_qlat.numel() * h_qlat.element_size() + h_qpe.numel() * h_qpe.element_size())
    d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()

    # after every decode measurement: the writer changes the caches' last T slots
    append = time_append(mla, w, kv, sc, L, stream) if args.append else None

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    value = world * steps * units["kv_bytes"] / max_elapsed / 1e9
    dec_avg = sum(dec) / len(dec)
    per_launch_bytes = units["total_bytes"] / L
    per_launch_flops = units["flops"] / L
    achieved_gbs = per_launch_bytes / dec_avg / 1e9
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved_gbs / hbm_peak, "traffic": recorded_traffic(args.workload, w.kv_label()),
                "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                "kernel": "mla decode attention kernel", "peak_source": f"{peak_src} hbm_gbs",
                "avg_launch_us": dec_avg * 1e6, "merge_avg_launch_us": sum(mer) / len(mer) * 1e6}
    tflops = per_launch_flops / dec_avg / 1e12
    kernel_dtype = {"simt": "f32"}.get(args.kernel, "e4m3" if w.kv_dtype == W.KV_FP8 else "bf16")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": max_elapsed / steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": kernel_dtype, "data": "synthetic",
        "config": workload_config(args, w, units, args.kernel, f"replicas x{world}"),
        "hbm_fraction_of_8TBs": value / world / NOMINAL_HBM_GBS,
        "seq_steps_per_s": world * steps * units["seqs"] / max_elapsed,
        "tensor_tflops": tflops,
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": steps * L * launches_per_call,
        "clocks": clocks,
    }
    if append is not None:
        line["append"] = append
    if world == 1 and not args.no_cpu_baseline:
        st, rows, spent, threads = oracle_sample(w, L, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": units["kv_bytes"] / st / 1e9, "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{rows} whole query rows of one layer ({spent:.1f} s), extrapolated to "
                      f"{L} layers x {B * T * H} rows"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if args.impl == "ours":
            torch.cuda.set_device(local_rank)
        backend = "nccl" if args.impl == "ours" else "gloo"
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=300))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
