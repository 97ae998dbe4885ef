"""CUDA path against the fp64 oracle, element by element, through the C ABI.

Small versions of every workload are compared in full (several 128-position
tiles, ragged last pages, split histories); the full-size workloads are
compared on sampled rows in the launch configuration the benchmark uses.
"""
import numpy as np
import pytest
import torch

import mla_latent_attention_b200 as mla
import mla_workloads as W
import oracle
from gpu_common import assert_matches_oracle, require_gpu

pytestmark = pytest.mark.gpu

KERNELS = ["simt", "tcgen05"]
DEV = "cuda"


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _run(w, kernel, **kw):
    wd = w.to(DEV)
    out, lse = mla.decode_workload(wd, kernel=kernel, **kw)
    torch.cuda.synchronize()
    return out, lse


SMALL = [
    ("single_query_256", {}),
    ("spec_verify_small", {}),
    ("batched_verify_fp8_32k", dict(B=3, ctx_override=("fixed", 2000))),
    ("long_ctx_142k", dict(ctx_override=("fixed", 9001))),
    ("long_ctx_142k", dict(ctx_override=("fixed", 5003), kv=W.KV_BF16)),
    ("ragged_dcp8", dict(B=5, ctx_override=("loguniform", 40, 3000))),
    # deeper drafts: T = 1 + st for st = 4 and 7
    ("spec_verify_small", dict(B=3, T=5, ctx_override=("uniform", 300, 1500))),
    ("batched_verify_fp8_32k", dict(B=2, T=8, ctx_override=("fixed", 900))),
]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name,kw", SMALL, ids=[f"{n}-{i}" for i, (n, _) in enumerate(SMALL)])
def test_small_workloads_match_oracle(name, kw, kernel):
    w = W.make_workload(name, **kw)
    ref_o, ref_l = oracle.decode_workload(w)
    out, lse = _run(w, kernel)
    assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, f"{name}/{kernel}")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("splits", [1, 2, 3, 17, 148, 700])
def test_any_split_count_matches_oracle(splits, kernel):
    w = W.make_workload("ragged_dcp8", B=6, ctx_override=("loguniform", 3, 2500))
    ref_o, ref_l = oracle.decode_workload(w)
    out, lse = _run(w, kernel, num_splits=splits)
    assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, f"splits={splits}")


@pytest.mark.parametrize("kernel", KERNELS)
def test_fp32_output(kernel):
    w = W.make_workload("spec_verify_small", B=2, ctx_override=("uniform", 300, 700))
    ref_o, ref_l = oracle.decode_workload(w)
    out, lse = _run(w, kernel, out_dtype=torch.float32)
    assert out.dtype == torch.float32
    assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, "fp32 out")


@pytest.mark.parametrize("kernel", KERNELS)
def test_page_relabelling_is_bit_identical(kernel):
    w = W.make_workload("batched_verify_fp8_32k", B=2, ctx_override=("fixed", 1500))
    a = _run(w, kernel)
    b = _run(W.permute_pages(w), kernel)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("kernel", KERNELS)
def test_padded_page_table_rows_are_bit_identical(kernel):
    """A page table whose rows are the first columns of a wider array (row
    stride larger than the row): the same pages, the same bits."""
    w = W.make_workload("spec_verify_small", B=3, kv=W.KV_FP8, ctx_override=("uniform", 200, 900))
    a = _run(w, kernel)
    B, n = w.page_table.shape
    wide = torch.full((B, n + 37), -1, dtype=torch.int32)
    wide[:, :n] = w.page_table
    wd = w.to(DEV)
    pt = wide.to(DEV)[:, :n]
    assert pt.stride(0) == n + 37 and not pt.is_contiguous()
    b = mla.decode(wd.q_lat, wd.q_pe, wd.kv_pages, wd.kv_scale, pt, wd.ctx_lens, wd.sm_scale, kernel=kernel)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("kernel", KERNELS)
def test_head_padding_is_bit_identical(kernel):
    w = W.make_workload("spec_verify_small", B=3, ctx_override=("uniform", 200, 900))
    o12, l12 = _run(w, kernel)
    o16, l16 = _run(W.pad_heads(w, 16), kernel)
    assert torch.equal(o12, o16[:, :, :12]) and torch.equal(l12, l16[:, :, :12])


@pytest.mark.parametrize("kernel", KERNELS)
def test_argmax_recovery_is_exact(kernel):
    """Each query row points at one position (latent dim 0 holds the position
    index); the recovered index must equal the row's last visible position."""
    w = W.make_workload("spec_verify_small", B=3, ctx_override=("uniform", 100, 250))
    for b in range(w.B):
        c = int(w.ctx_lens[b])
        for j in range(c):
            w.kv_pages[int(w.page_table[b, j // 16]), j % 16, 0] = float(j)
    for b in range(w.B):
        rows, _ = W.gather_logical_rows(w, b)
        rows = rows.to(torch.float32)
        for t in range(w.T):
            target = int(w.ctx_lens[b]) - w.T + t
            key = rows[target].clone()
            key[0] = 0.0
            qv = (key * (40.0 / key.norm())).to(torch.bfloat16)
            w.q_lat[b, t, :] = qv[:512]
            w.q_pe[b, t, :] = qv[512:]
    out, _ = _run(w, kernel)
    got = out[..., 0].float().cpu()
    for b in range(w.B):
        for t in range(w.T):
            target = int(w.ctx_lens[b]) - w.T + t
            assert torch.all((got[b, t] - target).abs() < 0.5), (b, t, target, got[b, t])


@pytest.mark.parametrize("kernel", KERNELS)
def test_rows_that_see_nothing(kernel):
    w = W.make_workload("spec_verify_small", B=2, ctx_override=("uniform", 50, 90))
    vis = torch.tensor([[0, 5, 17], [3, 0, 40]], dtype=torch.int32)
    w.vis_lens = vis
    ref_o, ref_l = oracle.decode_workload(w)
    out, lse = _run(w, kernel)
    assert torch.all(out[0, 0] == 0) and torch.all(lse[0, 0].cpu() == -float("inf"))
    assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, "empty rows")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("kv", [W.KV_FP8, W.KV_BF16])
def test_most_query_rows_per_sequence(kv, kernel):
    """T * H = 8 * 128 = 1024 query rows per sequence, the most a call takes:
    22 row groups of 48 for the tensor-core kernel, the last one partial."""
    w = W.make_workload("batched_verify_fp8_32k", B=2, T=8, H=128, kv=kv, ctx_override=("uniform", 300, 700))
    ref_o, ref_l = oracle.decode_workload(w)
    out, lse = _run(w, kernel)
    assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, f"1024 rows {kv}/{kernel}")


RAGGED = [
    ("spec_verify_small", dict(B=5, T=4, ctx_override=("uniform", 200, 1200))),
    ("batched_verify_fp8_32k", dict(B=4, T=8, ctx_override=("fixed", 700))),
]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name,kw", RAGGED, ids=[n for n, _ in RAGGED])
def test_ragged_draft_depths(name, kw, kernel):
    """Sequences with 1..T query tokens in one call: real tokens match the
    oracle, padding slots are the empty set (out 0, lse -inf)."""
    w, n_new = W.ragged_drafts(W.make_workload(name, **kw))
    ref_o, ref_l = oracle.decode_workload(w)
    out, lse = _run(w, kernel)
    for b in range(w.B):
        k = int(n_new[b])
        assert torch.all(out[b, k:] == 0) and torch.all(lse[b, k:].cpu() == -float("inf")), b
    assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, f"ragged {name}/{kernel}")


@pytest.mark.parametrize("kernel", KERNELS)
def test_context_partitions_merge_to_whole(kernel):
    """Round-robin 8-way context partitions, each decoded to fp32 partials,
    merged with mla_merge_partials, equal the unpartitioned decode."""
    w = W.make_workload("ragged_dcp8", B=4, ctx_override=("loguniform", 64, 3000))
    ref_o, ref_l = oracle.decode_workload(w)
    parts = W.partition_round_robin(w, 8)
    outs, lses = [], []
    for p in parts:
        o, l = _run(p, kernel, out_dtype=torch.float32)
        outs.append(o)
        lses.append(l)
    mo, ml = mla.merge_partials(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    assert_matches_oracle(mo, ml, ref_o, ref_l, w.kv_dtype, "partition merge")
    whole_o, whole_l = _run(w, kernel)
    assert (mo.float() - whole_o.float()).abs().max().item() <= 2e-2 * whole_o.float().abs().max().item()


@pytest.mark.parametrize("kernel", KERNELS)
def test_partitions_holding_none_of_a_sequence(kernel):
    """Sequences shorter than the partition count: some partitions hold none
    of their positions (no pages, visible count 0) and must return the empty
    result, out 0 and lse -inf, which the merge then ignores."""
    w = W.make_workload("ragged_dcp8", B=4, H=8, ctx_override=("uniform", 3, 12))
    ref_o, ref_l = oracle.decode_workload(w)
    parts = W.partition_round_robin(w, 8)
    empty = [(k, b) for k, p in enumerate(parts) for b in range(w.B) if int(p.ctx_lens[b]) == 0]
    assert empty
    outs, lses = [], []
    for p in parts:
        o, l = _run(p, kernel, out_dtype=torch.float32)
        outs.append(o)
        lses.append(l)
    for k, b in empty:
        assert torch.all(outs[k][b] == 0) and torch.all(lses[k][b].cpu() == -float("inf")), (k, b)
    mo, ml = mla.merge_partials(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    assert_matches_oracle(mo, ml, ref_o, ref_l, w.kv_dtype, "partitions with empty sequences")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name,kw", [("spec_verify_small", dict(B=3, kv=W.KV_FP8)),
                                     ("batched_verify_fp8_32k", dict(B=2, ctx_override=("fixed", 3000)))])
def test_static_fp8_scale_matches_oracle(name, kw, kernel):
    """A per-tensor static FP8 scale (kv_scale of one element)."""
    w = W.static_scale_workload(W.make_workload(name, **kw))
    out, lse = _run(w, kernel)
    ref_o, ref_l = oracle.decode_workload(w)
    assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, f"{name} static scale")


# 7 parts: one warp per (row, quarter); 40 parts: eight warps per (row, quarter)
@pytest.mark.parametrize("n", [7, 40])
def test_merge_partials_matches_oracle(n):
    gen = torch.Generator().manual_seed(3)
    rows = 37
    o = torch.randn((n, rows, 512), generator=gen, dtype=torch.float64)
    l = torch.randn((n, rows), generator=gen, dtype=torch.float64) * 3
    l[2, :5] = -float("inf")
    l[:, 7] = -float("inf")                  # a row no part saw
    o[2, :5] = float("nan")                  # ignored: that part weighs nothing
    ref_o, ref_l = oracle.merge(o.numpy(), l.numpy())
    mo, ml = mla.merge_partials(o.float().to(DEV), l.float().to(DEV), out_dtype=torch.float32)
    torch.cuda.synchronize()
    got_o, got_l = mo.double().cpu().numpy(), ml.double().cpu().numpy()
    assert np.array_equal(got_o[7], np.zeros(512)) and got_l[7] == -np.inf
    fin = np.isfinite(ref_l)
    assert np.abs(got_o - ref_o).max() <= 1e-5 * np.abs(ref_o).max()
    assert np.abs(got_l[fin] - ref_l[fin]).max() <= 1e-5
    # a NaN normaliser poisons its row, also when every part of the row is NaN
    l2 = l.clone()
    l2[4, 9] = float("nan")
    l2[:, 11] = float("nan")
    mo, ml = mla.merge_partials(o.float().to(DEV), l2.float().to(DEV))
    torch.cuda.synchronize()
    assert torch.isnan(mo[9].float()).all() and torch.isnan(ml[9])
    assert torch.isnan(mo[11].float()).all() and torch.isnan(ml[11])
    _, ref_l2 = oracle.merge(o.numpy(), l2.numpy())
    assert np.array_equal(np.isnan(ml.double().cpu().numpy()), np.isnan(ref_l2))


@pytest.mark.parametrize("kernel", KERNELS)
def test_device_errors_are_reported_not_trapped(kernel):
    w = W.make_workload("spec_verify_small", B=3, ctx_override=("uniform", 100, 300)).to(DEV)
    ws = torch.zeros(1 << 26, dtype=torch.uint8, device=DEV)
    # bad page index in sequence 1
    pt = w.page_table.clone()
    pt[1, 2] = w.num_pages + 3
    mla.reset_device_error(ws)
    out, lse = mla.decode(w.q_lat, w.q_pe, w.kv_pages, w.kv_scale, pt, w.ctx_lens, w.sm_scale,
                          kernel=kernel, workspace=ws)
    code, info = mla.read_device_error(ws)
    assert (code, info) == (1, 1)
    assert torch.isnan(out[1].float()).all() and torch.isnan(lse[1]).all()
    assert torch.isfinite(out[0].float()).all() and torch.isfinite(out[2].float()).all()
    # context longer than the page table allows
    ctx = w.ctx_lens.clone()
    ctx[2] = w.page_table.shape[1] * 16 + 1
    mla.reset_device_error(ws)
    out, lse = mla.decode(w.q_lat, w.q_pe, w.kv_pages, w.kv_scale, w.page_table, ctx, w.sm_scale,
                          kernel=kernel, workspace=ws)
    assert mla.read_device_error(ws) == (2, 2)
    assert torch.isnan(out[2].float()).all() and torch.isfinite(out[0].float()).all()
    # visible count beyond the context
    vis = torch.stack([w.ctx_lens - 2, w.ctx_lens - 1, w.ctx_lens]).T.contiguous()
    vis[0, 1] = int(w.ctx_lens[0]) + 1
    mla.reset_device_error(ws)
    out, lse = mla.decode(w.q_lat, w.q_pe, w.kv_pages, w.kv_scale, w.page_table, w.ctx_lens,
                          w.sm_scale, vis_lens=vis, kernel=kernel, workspace=ws)
    assert mla.read_device_error(ws) == (3, 1)
    assert torch.isnan(out[0, 1].float()).all() and torch.isfinite(out[0, 0].float()).all()
    # and a clean call leaves the word clear
    mla.reset_device_error(ws)
    mla.decode_workload(w, kernel=kernel, workspace=ws)
    assert mla.read_device_error(ws) == (0, 0)


def test_host_argument_errors_raise():
    w = W.make_workload("single_query_256").to(DEV)
    with pytest.raises(mla.MlaError):
        mla.decode(w.q_lat, w.q_pe, w.kv_pages, torch.ones(w.num_pages, 16, device=DEV),
                   w.page_table, w.ctx_lens, w.sm_scale)           # bf16 with a scale
    with pytest.raises(mla.MlaError):
        mla.decode(w.q_lat, w.q_pe, w.kv_pages, None, w.page_table, w.ctx_lens, w.sm_scale,
                   workspace=torch.empty(16, dtype=torch.uint8, device=DEV))


def test_stage_event_outside_capture():
    """The optional stage event is a plain record when the stream is not being captured."""
    w = W.make_workload("spec_verify_small", B=2).to(DEV)
    ev = torch.cuda.Event()
    ev.record()                  # torch creates the event handle on first record
    torch.cuda.synchronize()
    out, lse = mla.decode_workload(w, stage_event=ev)
    torch.cuda.synchronize()
    assert ev.query()
    ref_o, ref_l = mla.decode_workload(w)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


@pytest.mark.parametrize("kernel", KERNELS)
def test_graph_capture_replays_identically(kernel):
    w = W.make_workload("long_ctx_142k", ctx_override=("fixed", 4000)).to(DEV)
    out = torch.empty((1, 1, 96, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((1, 1, 96), dtype=torch.float32, device=DEV)
    dims = mla.make_dims(w.q_lat, w.kv_pages, w.page_table, kernel=kernel)
    ws = torch.empty(mla.workspace_size(dims), dtype=torch.uint8, device=DEV)
    mla.decode_workload(w, out=out, lse=lse, kernel=kernel, workspace=ws)
    torch.cuda.synchronize()
    ref_o, ref_l = out.clone(), lse.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            mla.decode_workload(w, out=out, lse=lse, kernel=kernel, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


FULL = ["single_query_256", "spec_verify_small", "batched_verify_fp8_32k", "long_ctx_142k",
        "ragged_dcp8"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name):
    """Full-size workload, auto kernel and auto splits (the benchmark's launch
    configuration); the oracle checks a sample of rows."""
    w = W.make_workload(name, device=DEV)
    out, lse = mla.decode_workload(w)
    torch.cuda.synchronize()
    rows = W.sample_rows(w.B, w.T, w.H, 24)
    wc = w.to("cpu")
    ref_o, ref_l = oracle.decode_workload(wc, rows=rows)
    flat_o = out.reshape(-1, 512)[rows.to(DEV)]
    flat_l = lse.reshape(-1)[rows.to(DEV)]
    assert_matches_oracle(flat_o, flat_l, ref_o, ref_l, w.kv_dtype, f"{name} sampled")


def test_full_size_bf16_long_context_sampled():
    w = W.make_workload("long_ctx_142k", device=DEV, kv=W.KV_BF16)
    out, lse = mla.decode_workload(w)
    torch.cuda.synchronize()
    rows = W.sample_rows(w.B, w.T, w.H, 12)
    ref_o, ref_l = oracle.decode_workload(w.to("cpu"), rows=rows)
    assert_matches_oracle(out.reshape(-1, 512)[rows.to(DEV)], lse.reshape(-1)[rows.to(DEV)],
                          ref_o, ref_l, w.kv_dtype, "142K bf16 sampled")


def test_full_size_partitioned_decode_sampled():
    """The ragged 8-way partitioned workload at full size: partition decodes
    merged by mla_merge_partials against the oracle on sampled rows."""
    w = W.make_workload("ragged_dcp8", device=DEV)
    parts = W.partition_round_robin(w, 8)
    outs, lses = zip(*[mla.decode_workload(p, out_dtype=torch.float32) for p in parts])
    mo, ml = mla.merge_partials(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    rows = W.sample_rows(w.B, w.T, w.H, 16)
    ref_o, ref_l = oracle.decode_workload(w.to("cpu"), rows=rows)
    assert_matches_oracle(mo.reshape(-1, 512)[rows.to(DEV)], ml.reshape(-1)[rows.to(DEV)],
                          ref_o, ref_l, w.kv_dtype, "ragged partitions sampled")
