"""The allocation-free decode entry point, checked against the ordinary one.

``mla_decode_noalloc`` is for callers that cannot allocate device memory at
the point where they decode -- a runtime whose device memory all belongs to
another allocator, or a plugin that must not grow the process's device
footprint per call.  It runs the same kernels as ``mla_decode`` with a fixed
scratch array defined inside the library instead of a caller-provided
workspace.

Each case calls it twice in a row, through the C ABI, and compares both
results with ``mla_decode`` on the same inputs: within the parity tolerance
used elsewhere in the suite, and bit for bit, since both entry points run
the same deterministic kernels (a stale value left in the shared scratch
array would show up as a difference).  The device's free memory must not
change across the second call.  This file is named to be collected last, so
that a run stopping at the first failure has run everything else first.
"""
import ctypes

import pytest
import torch

import mla_latent_attention_b200 as mla
import mla_workloads as W
from gpu_common import LSE_TOL, out_rel_tol, require_gpu

pytestmark = pytest.mark.gpu


def _noalloc(w, out, lse):
    lib = mla.load_library()
    dims = mla.make_dims(w.q_lat, w.kv_pages, w.page_table, vis_lens=w.vis_lens)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.mla_decode_noalloc(p(w.q_lat), p(w.q_pe), p(w.kv_pages), p(w.kv_scale), p(w.page_table),
                                  p(w.ctx_lens), ctypes.c_float(w.sm_scale), p(out), p(lse),
                                  ctypes.byref(dims), stream)


@pytest.mark.parametrize("name,kw", [
    ("long_ctx_142k", {}),
    ("spec_verify_small", {}),
    ("ragged_dcp8", dict(B=6, ctx_override=("loguniform", 40, 3000))),
])
def test_noalloc_matches_decode_twice(name, kw):
    require_gpu()
    w = W.make_workload(name, device="cuda", **kw)
    ref_o, ref_l = mla.decode_workload(w)
    torch.cuda.synchronize()
    tol = out_rel_tol(w.kv_dtype) * ref_o.float().abs().max().item() + 1e-3
    outs = [torch.full_like(ref_o, float("nan")) for _ in range(2)]
    lses = [torch.full_like(ref_l, float("nan")) for _ in range(2)]
    free_before = None
    for i in range(2):
        if i == 1:
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
        assert _noalloc(w, outs[i], lses[i]) == 0
        torch.cuda.synchronize()
        if i == 1:
            assert torch.cuda.mem_get_info()[0] == free_before
        out, lse = outs[i], lses[i]
        assert torch.isfinite(out.float()).all()
        assert (out.float() - ref_o.float()).abs().max().item() <= tol
        fin = torch.isfinite(ref_l)
        assert torch.equal(fin, torch.isfinite(lse))
        assert (lse[fin] - ref_l[fin]).abs().max().item() <= LSE_TOL
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_noalloc_rejects_work_beyond_its_scratch():
    require_gpu()
    w = W.make_workload("ragged_dcp8", device="cuda", B=64, ctx_override=("fixed", 64))
    lib = mla.load_library()
    dims = mla.make_dims(w.q_lat, w.kv_pages, w.page_table, num_splits=4000)
    assert lib.mla_decode_workspace_size(ctypes.byref(dims)) > (32 << 20)
    out = torch.empty((w.B, w.T, w.H, 512), dtype=torch.bfloat16, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.mla_decode_noalloc(p(w.q_lat), p(w.q_pe), p(w.kv_pages), p(w.kv_scale), p(w.page_table),
                                p(w.ctx_lens), ctypes.c_float(w.sm_scale), p(out), None,
                                ctypes.byref(dims), None)
    assert rc == -3
