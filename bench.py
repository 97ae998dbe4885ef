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
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip timing every workload of the problem statement after the headline one")
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


class LayerStack:
    """One decode step of an L-layer MLA stack: L calls of the library over L
    separate copies of a workload's paged cache (same contents, own memory),
    for the same query rows.  A context-partitioned workload decodes its
    partitions to fp32 partials and merges them with mla_merge_partials."""

    def __init__(self, mla, w, L, dev, args, parts=None):
        self.mla, self.w, self.L, self.args = mla, w, L, args
        self.units = [parts] if parts else [[w]]
        srcs = parts if parts else [w]
        self.kv = [[s.kv_pages if i == 0 else s.kv_pages.clone() for s in srcs] for i in range(L)]
        self.sc = [[None if s.kv_scale is None else (s.kv_scale if i == 0 else s.kv_scale.clone())
                    for s in srcs] for i in range(L)]
        self.srcs = srcs
        B, T, H = w.B, w.T, w.H
        self.q_lat = torch.stack([w.q_lat] * L)
        self.q_pe = torch.stack([w.q_pe] * L)
        self.outs = torch.empty((L, B, T, H, 512), dtype=torch.bfloat16, device=dev)
        self.lses = torch.empty((L, B, T, H), dtype=torch.float32, device=dev)
        self.part_out = self.part_lse = None
        if parts:
            self.part_out = torch.empty((L, len(parts), B, T, H, 512), dtype=torch.float32, device=dev)
            self.part_lse = torch.empty((L, len(parts), B, T, H), dtype=torch.float32, device=dev)
        need = 0
        self.calls_per_layer = 0
        for s in srcs:
            d = mla.make_dims(w.q_lat, s.kv_pages, s.page_table, kernel=args.kernel,
                              num_splits=args.num_splits, vis_lens=s.vis_lens,
                              out_dtype=torch.float32 if parts else torch.bfloat16, kv_scale=s.kv_scale)
            n = mla.workspace_size(d)
            need = max(need, n)
            self.calls_per_layer += 2 if n > 256 else 1
        if parts:
            self.calls_per_layer += 1
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        n_dec = len(srcs)
        self.ev = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
                    for _ in range(n_dec + (1 if parts else 0))] for _ in range(L)]
        for e in (x for a in self.ev for b in a for x in b):
            e.record()      # torch creates CUDA events lazily: make the handles exist

    def layer(self, i, events=False):
        mla, parts = self.mla, self.part_out is not None
        for k, s in enumerate(self.srcs):
            e = self.ev[i][k]
            if events:
                e[0].record()
            out = self.part_out[i, k] if parts else self.outs[i]
            lse = self.part_lse[i, k] if parts else self.lses[i]
            mla.decode(self.q_lat[i], self.q_pe[i], self.kv[i][k], self.sc[i][k], s.page_table, s.ctx_lens,
                       s.sm_scale, out=out, lse=lse, vis_lens=s.vis_lens, kernel=self.args.kernel,
                       num_splits=self.args.num_splits, workspace=self.ws,
                       stage_event=e[1] if events else None)
            if events:
                e[2].record()
        if parts:
            e = self.ev[i][-1]
            if events:
                e[0].record()
                e[1].record()
            mla.merge_partials(self.part_out[i], self.part_lse[i], out=self.outs[i], lse=self.lses[i])
            if events:
                e[2].record()

    def step(self, events=False):
        for i in range(self.L):
            self.layer(i, events)

    def split_us(self):
        """(attention, merge) device microseconds of the last replay, per layer."""
        att = mer = 0.0
        for i in range(self.L):
            for e in self.ev[i]:
                att += event_ms(e[0], e[1]) * 1e3
                mer += event_ms(e[1], e[2]) * 1e3
        return att / self.L, mer / self.L


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            fn()
    return g


def time_replays(graph, steps):
    """Device seconds of ``steps`` back-to-back replays (CUDA events on the
    stream the replays are launched on)."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(steps):
        graph.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / 1e3


def kernel_split(stack, graph_ev, rounds=6, burst=4):
    """Attention and merge microseconds per layer from the event-instrumented
    graph, replayed ``burst`` times back to back (no host synchronisation in
    between, so the GPU stays busy as in the timed loop) and read after the
    last replay of each round.  Each event node adds its own latency between
    the kernels, so these durations overstate both kernels; ``split_step``
    scales their shares to the timed step."""
    att, mer = [], []
    for _ in range(rounds):
        for _ in range(burst):
            graph_ev.replay()
        torch.cuda.synchronize()
        a, m = stack.split_us()
        att.append(a)
        mer.append(m)
    att.sort()
    mer.sort()
    return att[len(att) // 2], mer[len(mer) // 2]


def split_step(layer_us, att_ev, mer_ev):
    """(attention, merge) microseconds of one layer of the timed step.  Each
    kernel of the event-instrumented copy sits between two event nodes, which
    add the same latency to each: that latency is half the amount by which
    the two event-measured times exceed the timed layer, and it is taken off
    both.  (On the 142K layer this puts the merge at 4.4 us of the layer; the
    step timed with and without the merge on one GPU differs by 4.1 us, where
    a split in proportion to the event times gave the merge 8.4 us.)"""
    if att_ev + mer_ev <= 0:
        return layer_us, 0.0
    extra = max(0.0, (att_ev + mer_ev - layer_us) / 2.0)
    mer = min(max(mer_ev - extra, 0.0), layer_us)
    return layer_us - mer, mer


def roof_fraction(units_layer, us, peaks, bound):
    """Achieved rate of one layer against the roofline that binds it."""
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    e4m3 = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    gbs = units_layer["total_bytes"] / us / 1e3
    tfs = units_layer["flops"] / us / 1e6
    if bound == "hbm":
        return {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm}
    return {"bound": "tensor (e4m3)", "achieved": tfs, "peak": e4m3, "unit": "TFLOP/s", "frac": tfs / e4m3,
            "note": "algorithmic flop; the exact hi/lo operand split issues twice as many e4m3 MMAs"}


# Binding roofline per workload (flop per cached byte against the B200 ridge):
# one or a few query rows per sequence are HBM-bound, 288 rows per sequence
# (B x 3 drafts x 96 heads) are tensor-bound.
BINDING = {"single_query_256": "hbm", "spec_verify_small": "hbm", "batched_verify_fp8_32k": "tensor",
           "long_ctx_142k": "hbm", "ragged_dcp8": "tensor"}
PER_CONFIG = [("single_query_256", None), ("spec_verify_small", None), ("batched_verify_fp8_32k", None),
              ("long_ctx_142k", None), ("long_ctx_142k", W.KV_BF16), ("ragged_dcp8", None)]


def measure_config(mla, name, kv, dev, args, peaks, stream, seconds=0.4):
    """Every workload of the problem statement at full size, timed like the
    headline: a graph of L layers over L cache copies (L chosen so one step
    reads at least 1 GB of KV, above the 126 MB L2); a workload too small for
    that (the 256-position sanity case) flushes L2 before each step and is
    timed step by step."""
    w = W.make_workload(name, device=dev, kv=kv)
    parts = W.partition_round_robin(w, W.CONFIGS[name].partitions) if W.CONFIGS[name].partitions > 1 else None
    u1 = step_units(w, 1)
    L = max(1, min(24, -(-int(1e9) // max(1, u1["kv_bytes"]))))
    flush = L * u1["kv_bytes"] < 4 * 126e6
    stack = LayerStack(mla, w, L, dev, args, parts)
    stack.step()
    torch.cuda.synchronize()
    g = capture(stack.step, stream)
    g_ev = capture(lambda: stack.step(True), stream)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    if flush:
        scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        times = []
        for _ in range(20):
            scratch.fill_(1)
            times.append(time_replays(g, 1))
        times.sort()
        step_s = times[len(times) // 2]
        steps = 20
        del scratch
    else:
        t1 = time_replays(g, 1)
        steps = max(3, min(2000, int(seconds / max(t1, 1e-6))))
        step_s = time_replays(g, steps) / steps
    att_ev, mer_ev = kernel_split(stack, g_ev)
    layer_us = step_s / L * 1e6
    att, mer = split_step(layer_us, att_ev, mer_ev)
    res = {"kv": w.kv_label(), "B": w.B, "T": w.T, "H": w.H, "layers": L, "steps": steps,
           "l2": "flushed before each step" if flush else f"{L * u1['kv_bytes'] / 1e9:.2f} GB of KV per step",
           "layer_us": layer_us, "attention_us": att, "merge_us": mer,
           "event_node_us": {"attention": att_ev, "merge": mer_ev},
           "kv_read_gbs": u1["kv_bytes"] / layer_us / 1e3,
           "seq_steps_per_s": w.B / (layer_us * 1e-6),
           "hbm_fraction_of_8TBs": u1["kv_bytes"] / layer_us / 1e3 / NOMINAL_HBM_GBS}
    if parts:
        res["partitions"] = len(parts)
    res["roof"] = roof_fraction(u1, layer_us, peaks, BINDING[name])
    res["roof_attention_kernel"] = roof_fraction(u1, att, peaks, BINDING[name]) if not parts else None
    del g, g_ev, stack
    torch.cuda.empty_cache()
    return res


def e2e_overlapped(stack, steps, world, dev, group=4):
    """The same step through the public API with the query rows coming from
    pinned host memory and the outputs going back to it every step.  The two
    copy directions run on streams of their own, ordered with the kernels by
    events, in groups of `group` consecutive layers (one copy per tensor and
    group): a group's inputs for the next step are copied once its decodes
    have read them, its outputs once they have been written."""
    L = stack.L
    h_qlat = torch.empty(stack.q_lat.shape, dtype=stack.q_lat.dtype, pin_memory=True).copy_(stack.q_lat)
    h_qpe = torch.empty(stack.q_pe.shape, dtype=stack.q_pe.dtype, pin_memory=True).copy_(stack.q_pe)
    h_out = torch.empty(stack.outs.shape, dtype=stack.outs.dtype, pin_memory=True)
    h_lse = torch.empty(stack.lses.shape, dtype=stack.lses.dtype, pin_memory=True)
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    groups = [(g0, min(g0 + group, L)) for g0 in range(0, L, group)]
    ev_in = [torch.cuda.Event() for _ in groups]
    ev_done = [torch.cuda.Event() for _ in groups]
    ev_saved = [torch.cuda.Event() for _ in groups]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for s in range(steps):
        with torch.cuda.stream(up):
            for j, (a, b) in enumerate(groups):
                if s > 0:
                    up.wait_event(ev_done[j])       # the previous step's decodes of the group have read q
                stack.q_lat[a:b].copy_(h_qlat[a:b], non_blocking=True)
                stack.q_pe[a:b].copy_(h_qpe[a:b], non_blocking=True)
                ev_in[j].record(up)
        for j, (a, b) in enumerate(groups):
            comp.wait_event(ev_in[j])
            if s > 0:
                comp.wait_event(ev_saved[j])        # the previous step's outputs of the group are on the host
            for i in range(a, b):
                stack.layer(i)
            ev_done[j].record(comp)
        with torch.cuda.stream(down):
            for j, (a, b) in enumerate(groups):
                down.wait_event(ev_done[j])
                h_out[a:b].copy_(stack.outs[a:b], non_blocking=True)
                h_lse[a:b].copy_(stack.lses[a:b], non_blocking=True)
                ev_saved[j].record(down)
    comp.wait_stream(down)
    comp.wait_stream(up)
    e1.record(comp)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3
    h2d = h_qlat.numel() * h_qlat.element_size() + h_qpe.numel() * h_qpe.element_size()
    d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()
    return t, h2d, d2h


def run_ours(args, rank, world, local_rank):
    import mla_latent_attention_b200 as mla
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = make_bench_workload(args, device=dev)
    L = args.layers
    units = step_units(w, L)
    stack = LayerStack(mla, w, L, dev, args)
    launches_per_call = stack.calls_per_layer
    # eager warm-up (sets kernel attributes), then one step captured as a graph;
    # a second graph of the same step carries per-layer event nodes, for the
    # per-kernel durations only (event nodes are kept out of the timed graph)
    stack.step()
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    graph = capture(stack.step, stream)
    graph_ev = capture(lambda: stack.step(True), stream)
    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize()
    est = time_replays(graph, 1)
    steps = args.steps if args.steps is not None else max(10, min(20000, int(3.0 / max(est, 1e-6))))

    sampler = ClockSampler(local_rank)
    sampler.start()
    # keep the GPU busy ~0.5 s so clock samples reflect load, untimed
    t_end = time.perf_counter() + 0.5
    while time.perf_counter() < t_end:
        graph.replay()
    if world > 1:
        torch.distributed.barrier()
    elapsed = time_replays(graph, steps)
    if world > 1:
        torch.distributed.barrier()
    dec_ev, mer_ev = kernel_split(stack, graph_ev)
    max_elapsed = max_over_ranks(elapsed, world, dev)

    e2e_steps = max(3, min(steps, 200))
    e2e_time, h2d, d2h = e2e_overlapped(stack, e2e_steps, world, dev)
    e2e_time = max_over_ranks(e2e_time, world, dev)
    e2e_value = world * e2e_steps * units["kv_bytes"] / e2e_time / 1e9

    # after every decode measurement: the writer changes the caches' last T slots
    kv0 = [k[0] for k in stack.kv]
    sc0 = [c[0] for c in stack.sc]
    append = time_append(mla, w, kv0, None if sc0[0] is None else sc0, L, stream) if args.append else None

    peaks, peak_src = load_peaks()
    per_config = None
    if args.per_config and world == 1:
        del graph, graph_ev
        per_config = {}
        for name, kv in PER_CONFIG:
            key = name if kv is None else f"{name}:{kv}"
            per_config[key] = measure_config(mla, name, kv, dev, args, peaks, stream)
    clocks = sampler.stop()

    if rank != 0:
        return
    value = world * steps * units["kv_bytes"] / max_elapsed / 1e9
    layer_us = max_elapsed / steps / L * 1e6
    dec_us, mer_us = split_step(layer_us, dec_ev, mer_ev)
    per_launch_bytes = units["total_bytes"] / L
    per_launch_flops = units["flops"] / L
    achieved_gbs = per_launch_bytes / dec_us / 1e3
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved_gbs / hbm_peak, "traffic": recorded_traffic(args.workload, w.kv_label()),
                "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                "kernel": "mla decode attention kernel", "peak_source": f"{peak_src} hbm_gbs",
                "avg_launch_us": dec_us, "merge_avg_launch_us": mer_us, "layer_us": layer_us,
                "split": "CUDA events around each kernel in a copy of the step graph; the latency "
                         "the event nodes add (half the amount by which the two event-measured times "
                         "exceed the timed layer) is taken off each, so the two add up to the timed layer",
                "event_node_us": {"attention": dec_ev, "merge": mer_ev}}
    tflops = per_launch_flops / dec_us / 1e6
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
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "note": "host copies on two side streams, one per tensor and group of four layers, overlapped with other layers' kernels"},
        "gpu_launches": steps * L * launches_per_call,
        "clocks": clocks,
    }
    if append is not None:
        line["append"] = append
    if per_config is not None:
        line["per_config"] = per_config
    if world == 1 and not args.no_cpu_baseline:
        st, rows, spent, threads = oracle_sample(w, L, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": units["kv_bytes"] / st / 1e9, "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{rows} whole query rows of one layer ({spent:.1f} s), extrapolated to "
                      f"{L} layers x {w.B * w.T * w.H} rows"}
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
