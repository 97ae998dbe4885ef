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

Two forms:
  * ``dcp_decode``: every rank holds all query rows and ends with the merged
    result for all of them (partials all-gathered);
  * ``dcp_decode_sharded``: every rank holds the queries of its own H/N heads
    (the heads sharded over the group as the layers around attention shard
    them); the queries are all-gathered, every rank decodes all heads over its
    positions, and an all-to-all sends each rank only the partials of its own
    heads, so a rank receives (N-1)/N of one partial set instead of N-1 sets.

On GPUs the decode and the merge are the library's kernels and the exchange
runs over NCCL; ``decode_fn`` and ``merge_fn`` exist so that the exchange can
be exercised on CPU ranks.
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
    query token sees); every rank passes the same query rows.  Returns
    (out [B,T,H,512] out_dtype, lse [B,T,H] fp32), the same on every rank."""
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


def dcp_decode_sharded(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, *, vis_lens, group=None,
                       out_dtype=torch.bfloat16, decode_fn=None, merge_fn=None):
    """Head-sharded DCP: ``q_lat`` [B,T,Hl,512] and ``q_pe`` [B,T,Hl,64] are
    this rank's heads (rank r owns heads r*Hl .. r*Hl + Hl - 1 of H = N*Hl).

    Gathers the queries of all heads, decodes them over this rank's positions
    (the other arguments as for ``dcp_decode``), exchanges the fp32 partials
    all-to-all by head, and merges the N partials of this rank's heads.
    Every rank must pass the same B, T and Hl (the collectives move equal
    blocks).  Returns (out [B,T,Hl,512] out_dtype, lse [B,T,Hl] fp32)."""
    decode_fn = decode_fn or _gpu_decode
    merge_fn = merge_fn or _gpu_merge
    world = dist.get_world_size(group)
    B, T, Hl = q_lat.shape[:3]
    ql = [torch.empty_like(q_lat) for _ in range(world)]
    qp = [torch.empty_like(q_pe) for _ in range(world)]
    dist.all_gather(ql, q_lat.contiguous(), group=group)
    dist.all_gather(qp, q_pe.contiguous(), group=group)
    q_lat_all = torch.cat(ql, dim=2)            # [B,T,N*Hl,512], heads rank-major
    q_pe_all = torch.cat(qp, dim=2)
    part_o, part_l = decode_fn(q_lat_all, q_pe_all, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, vis_lens)
    # [B,T,N,Hl,...] -> [N,B,T,Hl,...]: block s holds the heads of rank s
    send_o = part_o.reshape(B, T, world, Hl, 512).permute(2, 0, 1, 3, 4).contiguous()
    send_l = part_l.reshape(B, T, world, Hl).permute(2, 0, 1, 3).contiguous()
    recv_o = torch.empty_like(send_o)
    recv_l = torch.empty_like(send_l)
    dist.all_to_all_single(recv_o, send_o, group=group)
    dist.all_to_all_single(recv_l, send_l, group=group)
    # recv block s: rank s's partial for this rank's heads
    out, lse = merge_fn(recv_o.reshape(world, -1, 512), recv_l.reshape(world, -1), out_dtype)
    return out.reshape(B, T, Hl, 512), lse.reshape(B, T, Hl)
