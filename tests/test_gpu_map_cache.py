"""Tensor maps remembered across calls follow the buffers they describe.

The library keeps the encoded tensor maps of recently used buffers, keyed by
address and extents.  Calls whose KV pool and output start at the same
addresses but have other extents (page count, sequences, rows) must each get
maps of their own: every result is compared with the oracle, and the first
call is repeated after the second.
"""
import pytest
import torch

import mla_latent_attention_b200 as mla
import mla_workloads as W
import oracle
from gpu_common import assert_matches_oracle, require_gpu

pytestmark = pytest.mark.gpu


def _decode_in(w, pool, scales, out_store, lse_store):
    """Decode w with its pages copied into the front of `pool` and its outputs
    written to the front of the output stores (views at the same addresses)."""
    P = w.kv_pages.shape[0]
    kv = pool[:P]
    kv.copy_(w.kv_pages.to("cuda"))
    sc = None
    if w.kv_scale is not None:
        sc = scales[:P]
        sc.copy_(w.kv_scale.to("cuda"))
    B, T, H = w.q_lat.shape[:3]
    out = out_store[:B * T * H * 512].view(B, T, H, 512)
    lse = lse_store[:B * T * H].view(B, T, H)
    ws = torch.zeros(1 << 26, dtype=torch.uint8, device="cuda")
    mla.decode(w.q_lat.to("cuda"), w.q_pe.to("cuda"), kv, sc, w.page_table.to("cuda"), w.ctx_lens.to("cuda"),
               w.sm_scale, out=out, lse=lse, vis_lens=None if w.vis_lens is None else w.vis_lens.to("cuda"),
               workspace=ws)
    torch.cuda.synchronize()
    assert mla.read_device_error(ws) == (0, 0)
    return out, lse


def test_maps_follow_extents_at_one_address():
    require_gpu()
    wa = W.make_workload("long_ctx_142k", ctx_override=("fixed", 3000))                    # 1 x 96 rows
    wb = W.make_workload("batched_verify_fp8_32k", B=2, ctx_override=("fixed", 2500))      # 2 x 288 rows
    assert wa.kv_pages.shape[0] != wb.kv_pages.shape[0]
    pages = max(wa.kv_pages.shape[0], wb.kv_pages.shape[0])
    pool = torch.empty((pages, 16, 576), dtype=wa.kv_pages.dtype, device="cuda")
    scales = torch.empty((pages, 16), dtype=torch.float32, device="cuda")
    rows = max(wa.q_lat.shape[:3].numel(), wb.q_lat.shape[:3].numel())
    out_store = torch.empty(rows * 512, dtype=torch.bfloat16, device="cuda")
    lse_store = torch.empty(rows, dtype=torch.float32, device="cuda")
    refs = {id(w): oracle.decode_workload(w) for w in (wa, wb)}
    for w in (wa, wb, wa):
        out, lse = _decode_in(w, pool, scales, out_store, lse_store)
        ref_o, ref_l = refs[id(w)]
        assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, f"{w.name} at shared addresses")
