"""Context-parallel decode over CPU ranks (gloo): each rank decodes its
round-robin share of the positions, the partials are all-gathered and merged.
The per-rank decode and the merge are stand-ins built on the oracle (this is a
test of the exchange and of the partitioning, not of the kernels); the merged
answer must equal the oracle's decode of the whole cache."""
import datetime
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, kv, queue):
    import mla_workloads as W
    import oracle
    from mla_latent_attention_b200 import dcp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = W.make_workload("ragged_dcp8", B=3, H=4, kv=kv, ctx_override=("loguniform", 30, 400))
        part = W.partition_round_robin(w, world)[rank]
        B, T, H = w.B, w.T, w.H

        def decode_fn(q_lat, q_pe, pages, scale, pt, cl, sm, vis):
            o, l = oracle.decode(q_lat, q_pe, pages, scale, pt, cl, sm, kv_dtype=kv, vis_lens=vis)
            return (torch.from_numpy(o).to(torch.float32).view(B, T, H, 512),
                    torch.from_numpy(l).to(torch.float32).view(B, T, H))

        def merge_fn(o_all, l_all, out_dtype):
            n = o_all.shape[0]
            mo, ml = oracle.merge(o_all.double().reshape(n, -1, 512).numpy(), l_all.double().reshape(n, -1).numpy())
            return torch.from_numpy(mo).view(B, T, H, 512), torch.from_numpy(ml).view(B, T, H)

        out, lse = dcp.dcp_decode(part.q_lat, part.q_pe, part.kv_pages, part.kv_scale, part.page_table,
                                  part.ctx_lens, part.sm_scale, vis_lens=part.vis_lens, decode_fn=decode_fn,
                                  merge_fn=merge_fn)
        ref_o, ref_l = oracle.decode_workload(w)
        err_o = float(np.abs(out.reshape(-1, 512).numpy() - ref_o).max())
        err_l = float(np.abs(lse.reshape(-1).numpy() - ref_l).max())
        queue.put((rank, err_o, err_l, float(np.abs(ref_o).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_dcp_over_cpu_ranks_equals_whole_decode(world, kv):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, kv, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err_o, err_l, scale in results:
        # fp32 partials, exact merge: rounding only
        assert err_o <= 1e-6 * scale + 1e-7, (rank, err_o)
        assert err_l <= 1e-5, (rank, err_l)


def _rank_sharded(rank, world, port, kv, queue):
    import mla_workloads as W
    import oracle
    from mla_latent_attention_b200 import dcp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        Hl = 2
        w = W.make_workload("ragged_dcp8", B=3, H=Hl * world, kv=kv, ctx_override=("loguniform", 30, 400))
        part = W.partition_round_robin(w, world)[rank]
        B, T, H = w.B, w.T, w.H
        heads = slice(rank * Hl, (rank + 1) * Hl)

        def decode_fn(q_lat, q_pe, pages, scale, pt, cl, sm, vis):
            assert q_lat.shape == (B, T, H, 512)
            o, l = oracle.decode(q_lat, q_pe, pages, scale, pt, cl, sm, kv_dtype=kv, vis_lens=vis)
            return (torch.from_numpy(o).to(torch.float32).view(B, T, H, 512),
                    torch.from_numpy(l).to(torch.float32).view(B, T, H))

        def merge_fn(o_all, l_all, out_dtype):
            n = o_all.shape[0]
            mo, ml = oracle.merge(o_all.double().reshape(n, -1, 512).numpy(), l_all.double().reshape(n, -1).numpy())
            return torch.from_numpy(mo), torch.from_numpy(ml)

        out, lse = dcp.dcp_decode_sharded(part.q_lat[:, :, heads], part.q_pe[:, :, heads], part.kv_pages,
                                          part.kv_scale, part.page_table, part.ctx_lens, part.sm_scale,
                                          vis_lens=part.vis_lens, decode_fn=decode_fn, merge_fn=merge_fn)
        ref_o, ref_l = oracle.decode_workload(w)
        ref_o = ref_o.reshape(B, T, H, 512)[:, :, heads]
        ref_l = ref_l.reshape(B, T, H)[:, :, heads]
        assert tuple(out.shape) == (B, T, Hl, 512) and tuple(lse.shape) == (B, T, Hl)
        err_o = float(np.abs(out.numpy() - ref_o).max())
        err_l = float(np.abs(lse.numpy() - ref_l).max())
        queue.put((rank, err_o, err_l, float(np.abs(ref_o).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_head_sharded_dcp_equals_whole_decode_of_own_heads(world, kv):
    """Queries sharded by head: all-gather q, decode, all-to-all of partials by
    head, merge; each rank's heads equal the oracle's decode of the whole cache."""
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_sharded, args=(r, world, port, kv, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r[0] for r in results) == list(range(world))
    for rank, err_o, err_l, scale in results:
        assert err_o <= 1e-6 * scale + 1e-7, (rank, err_o)
        assert err_l <= 1e-5, (rank, err_l)


def _rank_dies(rank, world, port, queue):
    import mla_workloads as W
    from mla_latent_attention_b200 import dcp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    w = W.make_workload("spec_verify_small", B=2, H=2, ctx_override=("uniform", 40, 80))
    part = W.partition_round_robin(w, world)[rank]
    if rank == 1:
        os._exit(3)                            # a rank lost before the exchange

    def decode_fn(*args):
        return torch.zeros((2, 3, 2, 512)), torch.zeros((2, 3, 2))

    try:
        dcp.dcp_decode(part.q_lat, part.q_pe, part.kv_pages, part.kv_scale, part.page_table, part.ctx_lens,
                       part.sm_scale, vis_lens=part.vis_lens, decode_fn=decode_fn, merge_fn=lambda o, l, d: (o, l))
        queue.put((rank, "completed"))
    except Exception as e:  # the collective must fail, not hang
        queue.put((rank, type(e).__name__))
    # os._exit skips the queue's feeder thread: flush the message first
    queue.close()
    queue.join_thread()
    os._exit(0)


def test_dcp_lost_rank_is_an_error_not_a_hang():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    rank, what = queue.get(timeout=90)
    for p in procs:
        p.join(timeout=60)
    assert rank == 0 and what != "completed"
    assert procs[1].exitcode == 3
