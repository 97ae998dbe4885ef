"""Pins that tie the fp64 oracle to facts outside itself.

Each pin takes a loaded oracle library (the real one, or a deliberately
broken copy built by the mutation test) and raises AssertionError when the
oracle disagrees with:
  * library routines: torch's e4m3fn and bf16 conversions, and torch's CPU
    flash-attention kernel (output and log-sum-exp) on gathered rows;
  * closed forms: one visible position, a zero query, identical value rows,
    two positions (logistic weights);
  * invariants: relabelling physical pages, zero-padding extra heads (the
    12 -> 16 head-padding adapter, "Inside Kimi K3 optimisation work",
    section 4), split-and-merge of round-robin context partitions (section 1,
    DCP: partial answers carry normalisation information);
  * an argmax-recovery case that checks page-table indexing and the causal
    mask among draft tokens position by position.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import mla_workloads as W
import oracle


def _small(kv, T=1, H=3, B=2, ctx=("uniform", 17, 70), seed=3, shuffle=True):
    cfg = W.Config("pin", B=B, T=T, H=H, ctx=ctx, kv=kv, shuffle=shuffle, seed=seed)
    return W.make_from_config(cfg)


def _dequant_rows(w, b):
    rows, sc = W.gather_logical_rows(w, b)
    if w.kv_dtype == W.KV_BF16:
        return rows.to(torch.float64)
    return rows.view(torch.float8_e4m3fn).to(torch.float64) * sc.to(torch.float64)[:, None]


def _vis(w, b, t):
    if w.vis_lens is not None:
        return int(w.vis_lens[b, t])
    return int(w.ctx_lens[b]) - w.T + t + 1


def pin_e4m3_table(lib):
    """All 256 e4m3fn codes decode like torch's float8_e4m3fn -> float64."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(i, lib) for i in range(256)])
    nan_ref = np.isnan(ref)
    assert np.array_equal(nan_ref, np.isnan(got)), "NaN codes differ"
    assert np.array_equal(ref[~nan_ref], got[~nan_ref]), "finite e4m3 values differ"


def pin_bf16_widening(lib):
    """bf16 bit patterns widen like torch's bfloat16 -> float64."""
    gen = torch.Generator().manual_seed(9)
    bits = torch.randint(0, 65536, (4000,), generator=gen, dtype=torch.int32)
    bits = torch.cat([bits, torch.tensor([0, 0x8000, 0x7F80, 0xFF80, 0x0001, 0x3F80, 0xC000])])
    ref = bits.to(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(int(v) & 0xFFFF, lib) for v in bits.tolist()])
    nan_ref = np.isnan(ref)
    assert np.array_equal(nan_ref, np.isnan(got))
    assert np.array_equal(ref[~nan_ref], got[~nan_ref])


def _library_attention(w):
    """torch CPU flash attention (fp64) on rows gathered through the page table."""
    B, T, H = w.B, w.T, w.H
    outs = np.zeros((B, T, H, 512))
    lses = np.zeros((B, T, H))
    for b in range(B):
        kv = _dequant_rows(w, b)                       # [ctx,576]
        n = kv.shape[0]
        q = torch.cat([w.q_lat[b], w.q_pe[b]], dim=-1).to(torch.float64)   # [T,H,576]
        q = q.permute(1, 0, 2).unsqueeze(0)            # [1,H,T,576]
        k = kv.unsqueeze(0).unsqueeze(0).expand(1, H, n, 576)
        v = torch.cat([kv[:, :512], torch.zeros(n, 64, dtype=torch.float64)], dim=-1)
        v = v.unsqueeze(0).unsqueeze(0).expand(1, H, n, 576)
        mask = torch.full((T, n), float("-inf"), dtype=torch.float64)
        for t in range(T):
            mask[t, :_vis(w, b, t)] = 0.0
        o, lse = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(
            q.contiguous(), k.contiguous(), v.contiguous(), 0.0, False,
            attn_mask=mask, scale=w.sm_scale)[:2]
        outs[b] = o[0, :, :, :512].permute(1, 0, 2).numpy()
        lses[b] = lse[0].permute(1, 0).numpy()
    return outs.reshape(-1, 512), lses.reshape(-1)


def pin_library_attention(lib):
    """Paged decode equals torch's fp64 attention on the gathered rows."""
    for kv in (W.KV_BF16, W.KV_FP8):
        for T in (1, 3):
            w = _small(kv, T=T, seed=10 + T)
            out, lse = oracle.decode_workload(w, lib=lib)
            ref_o, ref_l = _library_attention(w)
            assert np.abs(out - ref_o).max() <= 1e-12 * max(1.0, np.abs(ref_o).max()), (kv, T)
            assert np.abs(lse - ref_l).max() <= 1e-12 * max(1.0, np.abs(ref_l).max()), (kv, T)


def pin_single_position(lib):
    """One visible position: out is that position's latent row, lse its score."""
    for kv in (W.KV_BF16, W.KV_FP8):
        w = _small(kv, T=1, H=2, B=1, ctx=("fixed", 1), seed=21)
        out, lse = oracle.decode_workload(w, lib=lib)
        row = _dequant_rows(w, 0)[0].numpy()
        q = torch.cat([w.q_lat[0, 0], w.q_pe[0, 0]], -1).to(torch.float64).numpy()   # [H,576]
        assert np.array_equal(out, np.broadcast_to(row[:512], out.shape)), kv
        assert np.allclose(lse, w.sm_scale * (q @ row), rtol=1e-13, atol=0), kv


def pin_zero_query(lib):
    """A zero query weighs every visible position equally: out = mean, lse = ln n."""
    for kv in (W.KV_BF16, W.KV_FP8):
        w = _small(kv, T=3, H=2, B=2, ctx=("uniform", 20, 50), seed=22)
        w.q_lat.zero_()
        w.q_pe.zero_()
        out, lse = oracle.decode_workload(w, lib=lib)
        out = out.reshape(w.B, w.T, w.H, 512)
        lse = lse.reshape(w.B, w.T, w.H)
        for b in range(w.B):
            rows = _dequant_rows(w, b).numpy()
            for t in range(w.T):
                n = _vis(w, b, t)
                for h in range(w.H):
                    assert np.allclose(out[b, t, h], rows[:n, :512].mean(0), rtol=1e-12, atol=1e-14)
                    assert abs(lse[b, t, h] - math.log(n)) <= 1e-12


def pin_constant_values(lib):
    """If every visible latent row is the same vector, out is that vector for any query."""
    w = _small(W.KV_BF16, T=3, H=2, B=2, seed=23)
    vec = torch.randn(512, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    for b in range(w.B):
        c = int(w.ctx_lens[b])
        for j in range(c):
            w.kv_pages[int(w.page_table[b, j // 16]), j % 16, :512] = vec
    out, _ = oracle.decode_workload(w, lib=lib)
    assert np.allclose(out, vec.to(torch.float64).numpy()[None, :], rtol=1e-13, atol=1e-15)


def pin_two_positions(lib):
    """Two positions: weights are logistic in the score difference."""
    w = _small(W.KV_FP8, T=1, H=3, B=1, ctx=("fixed", 2), seed=24)
    out, lse = oracle.decode_workload(w, lib=lib)
    rows = _dequant_rows(w, 0).numpy()
    q = torch.cat([w.q_lat[0, 0], w.q_pe[0, 0]], -1).to(torch.float64).numpy()
    s = w.sm_scale * (q @ rows.T)                       # [H,2]
    w1 = 1.0 / (1.0 + np.exp(s[:, 0] - s[:, 1]))
    ref = (1 - w1)[:, None] * rows[0, :512] + w1[:, None] * rows[1, :512]
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-14)
    ref_lse = np.maximum(s[:, 0], s[:, 1]) + np.log1p(np.exp(-np.abs(s[:, 0] - s[:, 1])))
    assert np.allclose(lse, ref_lse, rtol=1e-13, atol=1e-14)


def pin_page_permutation(lib):
    """Relabelling physical pages (and the table with them) changes no bit."""
    for kv in (W.KV_BF16, W.KV_FP8):
        w = _small(kv, T=3, H=2, seed=25)
        a = oracle.decode_workload(w, lib=lib)
        b = oracle.decode_workload(W.permute_pages(w), lib=lib)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]), kv


def pin_head_padding(lib):
    """Zero-padding 12 heads to 16 leaves the first 12 heads' results bit-identical."""
    w = _small(W.KV_FP8, T=3, H=12, B=2, ctx=("uniform", 30, 60), seed=26)
    o12, l12 = oracle.decode_workload(w, lib=lib)
    o16, l16 = oracle.decode_workload(W.pad_heads(w, 16), lib=lib)
    o16 = o16.reshape(w.B, w.T, 16, 512)[:, :, :12].reshape(-1, 512)
    l16 = l16.reshape(w.B, w.T, 16)[:, :, :12].reshape(-1)
    assert np.array_equal(o12, o16) and np.array_equal(l12, l16)


def pin_split_merge(lib):
    """Round-robin context partitions, decoded apart and LSE-merged, equal the whole."""
    for kv in (W.KV_BF16, W.KV_FP8):
        w = _small(kv, T=3, H=2, B=3, ctx=("uniform", 9, 60), seed=27)
        whole_o, whole_l = oracle.decode_workload(w, lib=lib)
        parts = W.partition_round_robin(w, 4)
        outs, lses = zip(*[oracle.decode_workload(p, lib=lib) for p in parts])
        mo, ml = oracle.merge(np.stack(outs), np.stack(lses), lib=lib)
        assert np.abs(mo - whole_o).max() <= 1e-12, kv
        assert np.abs(ml - whole_l).max() <= 1e-12, kv


def pin_argmax_recovery(lib):
    """Make one position dominate each query row and recover its logical index.

    Latent dim 0 of position j holds j (exactly representable in bf16 for
    j < 256).  The query of draft token t points at the key of its own last
    visible position, scaled up so that position takes essentially all the
    weight.  A wrong page lookup, slot, or off-by-one mask moves the answer.
    """
    w = _small(W.KV_BF16, T=3, H=2, B=2, ctx=("uniform", 40, 200), seed=28)
    for b in range(w.B):
        c = int(w.ctx_lens[b])
        for j in range(c):
            w.kv_pages[int(w.page_table[b, j // 16]), j % 16, 0] = float(j)
    for b in range(w.B):
        rows = _dequant_rows(w, b)
        for t in range(w.T):
            target = _vis(w, b, t) - 1
            key = rows[target].clone()
            key[0] = 0.0
            for h in range(w.H):
                qv = (key * (40.0 / key.norm())).to(torch.bfloat16)
                w.q_lat[b, t, h] = qv[:512]
                w.q_pe[b, t, h] = qv[512:]
    out, _ = oracle.decode_workload(w, lib=lib)
    out = out.reshape(w.B, w.T, w.H, 512)
    for b in range(w.B):
        for t in range(w.T):
            target = _vis(w, b, t) - 1
            got = out[b, t, :, 0]
            assert np.all(np.abs(got - target) < 0.5), (b, t, target, got)


def pin_merge_rules(lib):
    """Merge: one part is the identity; -inf parts weigh nothing; all -inf is
    empty; equal normalisers average; a NaN normaliser poisons its row."""
    rng = np.random.default_rng(4)
    o = rng.standard_normal((1, 5, 8))
    l = rng.standard_normal((1, 5))
    mo, ml = oracle.merge(o, l, lib=lib)
    assert np.array_equal(mo, o[0]) and np.array_equal(ml, l[0])
    o2 = np.concatenate([o, rng.standard_normal((1, 5, 8))])
    l2 = np.concatenate([l, np.full((1, 5), -np.inf)])
    mo, ml = oracle.merge(o2, l2, lib=lib)
    assert np.allclose(mo, o[0], rtol=1e-15) and np.allclose(ml, l[0], rtol=1e-15)
    mo, ml = oracle.merge(o2, np.full((2, 5), -np.inf), lib=lib)
    assert np.all(mo == 0.0) and np.all(ml == -np.inf)
    # two parts with equal lse average their outputs and add ln 2
    l3 = np.zeros((2, 5))
    mo, ml = oracle.merge(o2, l3, lib=lib)
    assert np.allclose(mo, o2.mean(0), rtol=1e-14) and np.allclose(ml, math.log(2.0), rtol=1e-15)
    # a NaN normaliser poisons its row only, also when every part of it is NaN
    l4 = np.zeros((2, 5))
    l4[1, 1] = np.nan
    l4[:, 3] = np.nan
    mo, ml = oracle.merge(o2, l4, lib=lib)
    assert np.isnan(mo[[1, 3]]).all() and np.isnan(ml[[1, 3]]).all()
    ok = [0, 2, 4]
    assert np.allclose(mo[ok], o2.mean(0)[ok], rtol=1e-14) and np.isfinite(ml[ok]).all()


def pin_e4m3_encode_inverts_decoder(lib):
    """The cache writer's encoder is the inverse of the (pinned) decoder on
    every finite code, both zeros included."""
    bad = [c for c in range(256)
           if c not in (0x7F, 0xFF) and oracle.e4m3_encode(oracle.e4m3_to_f64(c, lib=lib), lib=lib) != c]
    assert bad == [], bad[:8]


def pin_e4m3_encode_rounding(lib):
    """Round to nearest even with the clamp at 448, against torch's
    float8_e4m3fn conversion: a dense grid past the clamp, every midpoint
    between neighbouring codes (the ties) and the subnormal range."""
    vals = [float(v) for v in torch.linspace(-480, 480, 9601, dtype=torch.float32)]
    pos = sorted(oracle.e4m3_to_f64(c, lib=lib) for c in range(0x00, 0x7F))
    mids = [(a + b) / 2 for a, b in zip(pos, pos[1:])]
    vals += mids + [-m for m in mids] + [k * 2.0 ** -11 for k in range(-40, 41)]
    x = torch.tensor(vals, dtype=torch.float32)
    ref = x.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_encode(float(v), lib=lib) for v in x.numpy()], dtype=np.uint8)
    assert np.array_equal(ref, mine)


def pin_row_quantiser(lib):
    """Per-token quantiser = mla_workloads.quantize_fp8_rows (torch binary32
    arithmetic: amax / 448, x / scale, clamp, round) bit for bit."""
    gen = torch.Generator().manual_seed(11)
    rows = (torch.randn((32, 576), generator=gen) * torch.rand((32, 1), generator=gen) * 8).to(torch.bfloat16)
    rows[3] = 0
    rows[4, 7] = -0.0
    codes_ref, scales_ref = W.quantize_fp8_rows(rows.float())
    for i in range(rows.shape[0]):
        codes, scale = oracle.quantize_row_e4m3(rows[i], lib=lib)
        assert np.array_equal(codes, codes_ref[i].numpy()), i
        assert np.float32(scale) == scales_ref[i].numpy(), i


def pin_append_positions(lib):
    """Token t of sequence b lands at position ctx - T + t through the page
    table, latent then RoPE values, and nothing else changes (bf16 cache:
    exact copy of the written row)."""
    gen = torch.Generator().manual_seed(12)
    B, T, ctx = 3, 3, [5, 17, 40]
    pages0, _, pt = W.build_paged_cache(ctx, W.KV_BF16, gen, shuffle=True)
    c_new = torch.randn((B, T, 512), generator=gen).to(torch.bfloat16)
    k_new = torch.randn((B, T, 64), generator=gen).to(torch.bfloat16)
    pages, _, ok = oracle.append_kv(c_new, k_new, pages0, None, pt, torch.tensor(ctx, dtype=torch.int32),
                                    kv_dtype=W.KV_BF16, lib=lib)
    assert ok
    expect = pages0.view(torch.int16).numpy().view(np.uint16).copy()
    for b in range(B):
        for t in range(T):
            pos = ctx[b] - T + t
            row = torch.cat([c_new[b, t], k_new[b, t]]).view(torch.int16).numpy().view(np.uint16)
            expect[int(pt[b, pos // 16]), pos % 16] = row
    assert np.array_equal(pages, expect)
    # FP8 cache: the written rows are the generator's quantisation of the new rows
    pages0, scales0, pt = W.build_paged_cache(ctx, W.KV_FP8, gen, shuffle=True)
    pages, scales, ok = oracle.append_kv(c_new, k_new, pages0, scales0, pt, torch.tensor(ctx, dtype=torch.int32),
                                         kv_dtype=W.KV_FP8, lib=lib)
    assert ok
    expect = pages0.numpy().copy()
    expect_s = scales0.numpy().copy()
    rows = torch.cat([c_new, k_new], dim=-1).float().reshape(B * T, 576)
    codes, sc = W.quantize_fp8_rows(rows)
    for b in range(B):
        for t in range(T):
            pos = ctx[b] - T + t
            page, slot = int(pt[b, pos // 16]), pos % 16
            expect[page, slot] = codes[b * T + t].numpy()
            expect_s[page, slot] = sc[b * T + t].numpy()
    assert np.array_equal(pages, expect)
    assert np.array_equal(scales.view(np.uint32), expect_s.view(np.uint32)) or \
        np.array_equal(np.isnan(scales), np.isnan(expect_s)) and np.array_equal(scales[~np.isnan(scales)],
                                                                                expect_s[~np.isnan(expect_s)])


def pin_static_scale(lib):
    """A per-tensor scale s is the per-position cache whose every scale is s:
    both decode to the same bits; and the writer with a static scale stores
    e4m3(clamp(x / s)) (torch arithmetic) and leaves the scale alone."""
    w = W.make_workload("spec_verify_small", B=2, kv=W.KV_FP8, ctx_override=("uniform", 40, 90))
    ws = W.static_scale_workload(w)
    s = float(ws.kv_scale[0])
    full = ws.kv_scale.expand(ws.kv_pages.shape[0], 16).contiguous()
    o1, l1 = oracle.decode(ws.q_lat, ws.q_pe, ws.kv_pages, ws.kv_scale, ws.page_table, ws.ctx_lens, ws.sm_scale,
                           kv_dtype=W.KV_FP8, lib=lib)
    o2, l2 = oracle.decode(ws.q_lat, ws.q_pe, ws.kv_pages, full, ws.page_table, ws.ctx_lens, ws.sm_scale,
                           kv_dtype=W.KV_FP8, lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    gen = torch.Generator().manual_seed(14)
    c_new = (torch.randn((2, 3, 512), generator=gen) * 3).to(torch.bfloat16)
    k_new = torch.randn((2, 3, 64), generator=gen).to(torch.bfloat16)
    pages, scales, ok = oracle.append_kv(c_new, k_new, ws.kv_pages, ws.kv_scale, ws.page_table, ws.ctx_lens,
                                         kv_dtype=W.KV_FP8, lib=lib)
    assert ok and scales.shape == (1,) and np.float32(scales[0]) == np.float32(s)
    rows = torch.cat([c_new, k_new], dim=-1).float()
    codes = (rows / torch.tensor(s, dtype=torch.float32)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    ctx = ws.ctx_lens.tolist()
    for b in range(2):
        for t in range(3):
            pos = ctx[b] - 3 + t
            assert np.array_equal(pages[int(ws.page_table[b, pos // 16]), pos % 16], codes[b, t].numpy())


def pin_ragged_drafts(lib):
    """A batch whose sequences carry 1..T query tokens (the rest of the T slots
    padding, visible count 0) decodes each sequence's real tokens exactly as
    that sequence decoded alone with its own token count and the default
    causality; padding rows come out as the empty set: out 0, lse -inf."""
    for kv in (W.KV_BF16, W.KV_FP8):
        w0 = _small(kv, T=4, H=2, B=4, ctx=("uniform", 20, 75), seed=29)
        w, n_new = W.ragged_drafts(w0, n_new=[1, 4, 2, 3])
        out, lse = oracle.decode_workload(w, lib=lib)
        out = out.reshape(w.B, w.T, w.H, 512)
        lse = lse.reshape(w.B, w.T, w.H)
        for b in range(w.B):
            k = int(n_new[b])
            ao, al = oracle.decode_workload(W.one_sequence(w, b, T=k), lib=lib)
            assert np.array_equal(out[b, :k], ao.reshape(k, w.H, 512)), (kv, b)
            assert np.array_equal(lse[b, :k], al.reshape(k, w.H)), (kv, b)
            assert np.all(out[b, k:] == 0.0) and np.all(lse[b, k:] == -np.inf), (kv, b)


PINS = [pin_e4m3_table, pin_bf16_widening, pin_library_attention, pin_single_position,
        pin_zero_query, pin_constant_values, pin_two_positions, pin_page_permutation,
        pin_head_padding, pin_split_merge, pin_argmax_recovery, pin_merge_rules,
        pin_e4m3_encode_inverts_decoder, pin_e4m3_encode_rounding, pin_row_quantiser, pin_append_positions,
        pin_static_scale, pin_ragged_drafts]
