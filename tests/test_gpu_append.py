"""The cache writer (mla_append_kv) against the oracle: bytes and scales bit
for bit, nothing else touched, and a decode of the appended cache against the
oracle's decode of its own appended cache."""
import dataclasses

import numpy as np
import pytest
import torch

import mla_latent_attention_b200 as mla
import mla_workloads as W
import oracle
from gpu_common import assert_matches_oracle, require_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _fresh_rows(B, T, seed, scale=1.0):
    gen = torch.Generator().manual_seed(seed)
    c = (torch.randn((B, T, 512), generator=gen) * scale).to(torch.bfloat16)
    k = (torch.randn((B, T, 64), generator=gen) * scale).to(torch.bfloat16)
    return c, k


@pytest.mark.parametrize("kv", [W.KV_FP8, W.KV_BF16])
@pytest.mark.parametrize("T", [1, 3, 8])
def test_append_bit_exact(kv, T):
    w = W.make_workload("ragged_dcp8", B=5, T=T, H=4, kv=kv, ctx_override=("loguniform", 20, 900))
    c_new, k_new = _fresh_rows(w.B, T, 31 + T)
    c_new[1, 0, 5] = -0.0
    c_new[2] = 0                              # an all-zero latent part
    if T > 1:
        c_new[3, 1] = 0
        k_new[3, 1] = 0                       # an all-zero row: scale 1
    ref_pages, ref_scales, ok = oracle.append_kv(c_new, k_new, w.kv_pages, w.kv_scale, w.page_table, w.ctx_lens,
                                                 kv_dtype=kv)
    assert ok
    wd = w.to(DEV)
    pages = wd.kv_pages.clone()
    scales = None if wd.kv_scale is None else wd.kv_scale.clone()
    mla.append_kv(c_new.to(DEV), k_new.to(DEV), pages, scales, wd.page_table, wd.ctx_lens)
    torch.cuda.synchronize()
    got = pages.cpu()
    got = got.view(torch.int16).numpy().view(np.uint16) if kv == W.KV_BF16 else got.numpy()
    assert np.array_equal(got, ref_pages)
    if kv == W.KV_FP8:
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))


def test_append_with_static_scale_bit_exact():
    """A per-tensor static scale: codes e4m3(x / s), the scale untouched."""
    w = W.static_scale_workload(W.make_workload("ragged_dcp8", B=4, H=4, ctx_override=("loguniform", 20, 500)))
    c_new, k_new = _fresh_rows(w.B, w.T, 71, scale=3.0)
    ref_pages, ref_scales, ok = oracle.append_kv(c_new, k_new, w.kv_pages, w.kv_scale, w.page_table, w.ctx_lens,
                                                 kv_dtype=W.KV_FP8)
    assert ok
    wd = w.to(DEV)
    pages, scales = wd.kv_pages.clone(), wd.kv_scale.clone()
    mla.append_kv(c_new.to(DEV), k_new.to(DEV), pages, scales, wd.page_table, wd.ctx_lens)
    torch.cuda.synchronize()
    assert np.array_equal(pages.cpu().numpy(), ref_pages)
    assert np.array_equal(scales.cpu().numpy(), ref_scales)


@pytest.mark.parametrize("kv", [W.KV_FP8, W.KV_BF16])
def test_decode_after_append(kv):
    """Append the drafts' rows, then verify-decode them: GPU append + GPU
    decode against oracle append + oracle decode."""
    w = W.make_workload("spec_verify_small", B=4, kv=kv, ctx_override=("uniform", 100, 700))
    c_new, k_new = _fresh_rows(w.B, w.T, 41, scale=2.0)
    ref_pages, ref_scales, ok = oracle.append_kv(c_new, k_new, w.kv_pages, w.kv_scale, w.page_table, w.ctx_lens,
                                                 kv_dtype=kv)
    assert ok
    pages_t = torch.from_numpy(ref_pages.view(np.int16)).view(torch.bfloat16) if kv == W.KV_BF16 \
        else torch.from_numpy(ref_pages)
    w_ref = dataclasses.replace(w, kv_pages=pages_t,
                                kv_scale=None if ref_scales is None else torch.from_numpy(ref_scales))
    ref_o, ref_l = oracle.decode_workload(w_ref)
    wd = w.to(DEV)
    mla.append_kv(c_new.to(DEV), k_new.to(DEV), wd.kv_pages, wd.kv_scale, wd.page_table, wd.ctx_lens)
    out, lse = mla.decode_workload(wd)
    torch.cuda.synchronize()
    assert_matches_oracle(out, lse, ref_o, ref_l, kv, "decode after append")


def test_append_device_errors():
    w = W.make_workload("spec_verify_small", B=3, kv=W.KV_FP8, ctx_override=("uniform", 100, 300))
    c_new, k_new = _fresh_rows(w.B, w.T, 51)
    wd = w.to(DEV)
    err = torch.zeros(2, dtype=torch.int32, device=DEV)
    bad_ctx = wd.ctx_lens.clone()
    bad_ctx[1] = 1                            # fewer positions than new tokens
    pages = wd.kv_pages.clone()
    mla.append_kv(c_new.to(DEV), k_new.to(DEV), pages, wd.kv_scale.clone(), wd.page_table, bad_ctx,
                  device_error=err)
    torch.cuda.synchronize()
    assert err.tolist() == [2, 1]             # MLA_DEV_BAD_CTX, sequence 1
    err.zero_()
    pt = wd.page_table.clone()
    pos = int(w.ctx_lens[2]) - w.T
    pt[2, pos // 16] = 10 ** 6
    mla.append_kv(c_new.to(DEV), k_new.to(DEV), pages, wd.kv_scale.clone(), pt, wd.ctx_lens, device_error=err)
    torch.cuda.synchronize()
    assert err.tolist() == [1, 2]             # MLA_DEV_BAD_PAGE, sequence 2


def test_append_through_padded_page_table():
    """Page-table rows inside a wider array (row stride larger than the row)
    place the tokens exactly as the contiguous table does."""
    w = W.make_workload("spec_verify_small", B=3, kv=W.KV_FP8, ctx_override=("uniform", 60, 300))
    c_new, k_new = _fresh_rows(w.B, w.T, 83)
    wd = w.to(DEV)
    B, n = w.page_table.shape
    wide = torch.full((B, n + 5), -1, dtype=torch.int32, device=DEV)
    wide[:, :n] = wd.page_table
    p1, s1 = wd.kv_pages.clone(), wd.kv_scale.clone()
    p2, s2 = wd.kv_pages.clone(), wd.kv_scale.clone()
    mla.append_kv(c_new.to(DEV), k_new.to(DEV), p1, s1, wd.page_table, wd.ctx_lens)
    mla.append_kv(c_new.to(DEV), k_new.to(DEV), p2, s2, wide[:, :n], wd.ctx_lens)
    torch.cuda.synchronize()
    # bit patterns: unused slots hold NaN scales, which compare unequal as floats
    assert torch.equal(p1, p2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))


def test_append_host_errors():
    w = W.make_workload("single_query_256").to(DEV)
    c_new, k_new = _fresh_rows(1, 1, 61)
    with pytest.raises(mla.MlaError):        # a bf16 cache takes no scales
        mla.append_kv(c_new.to(DEV), k_new.to(DEV), w.kv_pages, torch.ones((w.kv_pages.shape[0], 16),
                      device=DEV), w.page_table, w.ctx_lens)
    with pytest.raises(mla.MlaError):        # wrong shape
        mla.append_kv(c_new[:, :, :256].contiguous().to(DEV), k_new.to(DEV), w.kv_pages, None, w.page_table,
                      w.ctx_lens)
    w8 = W.make_workload("spec_verify_small", B=1, T=1, kv=W.KV_FP8, ctx_override=("fixed", 40)).to(DEV)
    with pytest.raises(mla.MlaError):        # one scale per page instead of per position
        mla.append_kv(c_new.to(DEV), k_new.to(DEV), w8.kv_pages, w8.kv_scale[:, 0].contiguous(), w8.page_table,
                      w8.ctx_lens)
    with pytest.raises(mla.MlaError):        # page table of another batch size
        mla.append_kv(c_new.to(DEV), k_new.to(DEV), w8.kv_pages, w8.kv_scale, w8.page_table.repeat(2, 1),
                      w8.ctx_lens)
    with pytest.raises(mla.MlaError):        # pages not [P,16,576]
        mla.append_kv(c_new.to(DEV), k_new.to(DEV), w8.kv_pages.view(-1, 576), w8.kv_scale, w8.page_table,
                      w8.ctx_lens)
