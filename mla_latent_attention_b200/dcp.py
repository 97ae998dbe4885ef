"""Context-parallel decode (DCP) across a process group.

Every rank holds a subset of each sequence's cached positions (for example
position p on rank p mod N, as in ``mla_workloads.partition_round_robin``):
its own page pool, page table, per-rank position counts and, for causality
inside the compacted subset, ``vis_lens``.  Each rank decodes its subset for
every query row into fp32 partials with their log-sum-exps, the partials are
all-gathered, and every rank merges them with the exact LSE rule — the one
exchange step of DCP ("Inside Kimi K3 optimisation work", section 1, DCP: the
history is split over the ranks and each partial answer carries the
normalisation information that lets the shards be weighted correctly).

The query rows are an input on every rank (gather them across ranks first
when the heads are sharded).  On GPUs the decode and the merge are the
library's kernels and the exchange runs over NCCL; ``decode_fn`` and
``merge_fn`` exist so that the exchange can be exercised on CPU ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import decode, merge_partials


def _gpu_decode(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, vis_lens):
    return decode(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, vis_lens=vis_lens,
                  out_dtype=torch.float32)


def _gpu_merge(out_parts, lse_parts, out_dtype):
    return merge_partials(out_parts, lse_parts, out_dtype=out_dtype)


def dcp_decode(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, *, vis_lens, group=None,
               out_dtype=torch.bfloat16, decode_fn=None, merge_fn=None):
    """Decode this rank's positions, all-gather the partials, merge.

    Arguments are those of ``mla_latent_attention_b200.decode`` for this
    rank's subset (``vis_lens`` [B,T]: how many of this rank's positions each
    query token sees).  Returns (out [B,T,H,512] out_dtype, lse [B,T,H] fp32),
    the same on every rank."""
    decode_fn = decode_fn or _gpu_decode
    merge_fn = merge_fn or _gpu_merge
    world = dist.get_world_size(group)
    part_o, part_l = decode_fn(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, vis_lens)
    part_o, part_l = part_o.contiguous(), part_l.contiguous()
    gathered_o = [torch.empty_like(part_o) for _ in range(world)]
    gathered_l = [torch.empty_like(part_l) for _ in range(world)]
    dist.all_gather(gathered_o, part_o, group=group)
    dist.all_gather(gathered_l, part_l, group=group)
    return merge_fn(torch.stack(gathered_o), torch.stack(gathered_l), out_dtype)
