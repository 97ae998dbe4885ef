"""Context-parallel decode through the library on one GPU: a one-rank NCCL
group (the exchange is then a copy) around the CUDA decode and merge, in both
forms (partials all-gathered; heads sharded with an all-to-all), against the
oracle's whole-cache decode.  The multi-rank exchange itself is covered
on CPU ranks (test_dcp.py)."""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

import mla_workloads as W
import oracle
from gpu_common import assert_matches_oracle, require_gpu

pytestmark = pytest.mark.gpu


def test_dcp_one_rank_nccl():
    require_gpu()
    from mla_latent_attention_b200 import dcp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = W.make_workload("ragged_dcp8", B=3, H=8, ctx_override=("loguniform", 100, 2000))
        part = W.partition_round_robin(w, 1)[0].to("cuda")
        out, lse = dcp.dcp_decode(part.q_lat, part.q_pe, part.kv_pages, part.kv_scale, part.page_table,
                                  part.ctx_lens, part.sm_scale, vis_lens=part.vis_lens)
        torch.cuda.synchronize()
        ref_o, ref_l = oracle.decode_workload(w)
        assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, "dcp one rank")
        # the head-sharded form: with one rank it owns every head
        out_s, lse_s = dcp.dcp_decode_sharded(part.q_lat, part.q_pe, part.kv_pages, part.kv_scale,
                                              part.page_table, part.ctx_lens, part.sm_scale,
                                              vis_lens=part.vis_lens)
        torch.cuda.synchronize()
        assert tuple(out_s.shape) == tuple(out.shape) and tuple(lse_s.shape) == tuple(lse.shape)
        assert_matches_oracle(out_s, lse_s, ref_o, ref_l, w.kv_dtype, "head-sharded dcp one rank")
    finally:
        dist.destroy_process_group()
