"""Host-side bookkeeping of bench.py (CPU only): the algorithmic units a step
is credited with, the comment-blind kernel hash that gates the recorded DRAM
traffic, the reference arm's JSON line, and the multi-rank path (max over
ranks on two gloo ranks; the reference arm under torchrun with two ranks)."""
import json
import os
import shutil
import subprocess
import sys


import bench
import mla_workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_step_units_single_token():
    """One token, 96 heads, 1,000 FP8 positions: 580 B per position (576 codes
    + fp32 scale) read once per layer; 2*576 + 2*512 flop per (row, position)."""
    w = W.make_workload("long_ctx_142k", ctx_override=("fixed", 1000))
    L = 3
    u = bench.step_units(w, L)
    assert u["kv_bytes"] == 1000 * 580 * L
    q = 96 * 576 * 2
    out = 96 * (512 * 2 + 4)
    assert u["total_bytes"] == u["kv_bytes"] + (q + out) * L
    assert u["flops"] == 2176 * 1000 * 96 * L


def test_step_units_draft_tokens():
    """T = 3 drafts: token t sees ctx - 3 + t + 1 positions; bf16 is 1,152 B per position."""
    w = W.make_workload("spec_verify_small", B=2, ctx_override=("uniform", 100, 200))
    u = bench.step_units(w, 1)
    ctx = [int(c) for c in w.ctx_lens]
    assert u["kv_bytes"] == sum(ctx) * 1152
    assert u["flops"] == 2176 * w.H * sum(c - 3 + t + 1 for c in ctx for t in range(3))
    wv, _ = W.ragged_drafts(w, n_new=[1, 3])
    uv = bench.step_units(wv, 1)
    assert uv["flops"] == 2176 * w.H * int(wv.vis_lens.sum())


def _copy_sources(dst):
    for rel in bench.KERNEL_SOURCES:
        os.makedirs(os.path.join(dst, os.path.dirname(rel)), exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), os.path.join(dst, rel))


def test_kernel_hash_ignores_comments_only(tmp_path, monkeypatch):
    ref = bench.kernel_source_hash()
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_source_hash() == ref
    src = tmp_path / bench.KERNEL_SOURCES[0]
    text = src.read_text()
    src.write_text("// a new comment\n/* and a block\n comment */\n" + text.replace("\n", "\n\n", 3))
    assert bench.kernel_source_hash() == ref
    src.write_text(text + "\nstatic int extra_symbol;\n")
    assert bench.kernel_source_hash() != ref


def test_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.txt").write_text(
        "# workload kv hash bytes\n"
        f"long_ctx_142k fp8 {h} 123456\n"
        "long_ctx_142k bf16 0000000000000000 999\n")
    assert bench.recorded_traffic("long_ctx_142k", "fp8") == 123456.0
    assert bench.recorded_traffic("long_ctx_142k", "bf16") is None      # stale capture
    assert bench.recorded_traffic("batched_verify_fp8_32k", "fp8") is None
    src = tmp_path / bench.KERNEL_SOURCES[1]
    src.write_text(src.read_text() + "\nstatic int changed;\n")
    assert bench.recorded_traffic("long_ctx_142k", "fp8") is None       # kernel changed since


def test_reference_arm_line():
    """--impl reference: the oracle on host cores, one JSON line with the
    same metric, unit and config keys as the CUDA arm."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "single_query_256", "--layers", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    w = W.make_workload("single_query_256")

    class A:
        workload, layers, num_splits = "single_query_256", 2, 0

    ours = bench.workload_config(A, w, bench.step_units(w, 2), "auto", "replicas x1")
    assert set(line["config"]) == set(ours)
    for k in ("workload", "B", "T", "H", "ctx", "kv", "layers", "l2"):
        assert line["config"][k] == ours[k], k


def test_step_units_static_scale_and_depth():
    """One static FP8 scale: 576 B per position (no per-position scale);
    --T changes the number of query tokens and so the flops."""
    w = W.make_workload("long_ctx_142k", ctx_override=("fixed", 640), T=4)
    ws = W.static_scale_workload(w)
    assert ws.kv_label() == "fp8-static" and w.kv_label() == "fp8"
    u = bench.step_units(ws, 2)
    assert u["kv_bytes"] == 640 * 576 * 2
    assert u["flops"] == 2176 * 96 * sum(640 - 4 + t + 1 for t in range(4)) * 2


def test_reference_arm_static_scale_and_depth():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "spec_verify_small", "--kv", "fp8", "--static-scale", "--T", "5",
                        "--layers", "1", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["config"]["T"] == 5 and line["config"]["kv"] == "fp8-static" and line["value"] > 0


def _max_rank(rank, world, port, queue):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        queue.put((rank, bench.max_over_ranks(1.5 + rank, world, "cpu")))
    finally:
        dist.destroy_process_group()
    queue.close()
    queue.join_thread()


def test_max_over_ranks_two_gloo_ranks():
    """The timed region's duration is the slowest rank's, on every rank."""
    import multiprocessing as mp
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_max_rank, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(queue.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 2.5, 1: 2.5}
    assert bench.max_over_ranks(0.25, 1, "cpu") == 0.25


def test_reference_arm_under_torchrun_two_ranks():
    """Launched like the multi-GPU bench (torchrun, 2 ranks): rank 0 alone
    runs the oracle and prints one line; both ranks exit 0."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port),
                        os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "single_query_256", "--layers", "1", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0


def test_split_step_divides_the_timed_layer():
    """The event nodes' own latency (half the amount by which the two
    event-measured times exceed the timed layer) comes off each kernel, so
    the two add up to the step."""
    att, mer = bench.split_step(54.69, 56.75, 10.23)
    assert abs(att + mer - 54.69) < 1e-9
    assert abs(mer - (10.23 - (56.75 + 10.23 - 54.69) / 2)) < 1e-9
    # event times that do not exceed the step: nothing is taken off
    att, mer = bench.split_step(60.0, 50.0, 10.0)
    assert (att, mer) == (50.0, 10.0)
    # a merge shorter than the event latency counts as zero
    att, mer = bench.split_step(10.0, 30.0, 1.0)
    assert (att, mer) == (10.0, 0.0)
    assert bench.split_step(10.0, 0.0, 0.0) == (10.0, 0.0)
