"""Seeded synthetic inputs for paged MLA decode.

This module only builds input tensors: query vectors, a paged compressed KV
cache, page tables, context lengths and (for context-partitioned decode) the
per-partition caches with their visibility counts.  It holds none of the
attention arithmetic, so that both the fp64 oracle and the CUDA library can be
fed from it without sharing any of the method's code.

Workloads follow the problem statement of the pages:
  * each cached position holds 576 values, a 512-d latent ``c_kv`` followed by
    a 64-d RoPE key ``k_pe`` ("Inside Kimi K3 optimisation work", section 1,
    DCP: 24 layers x 142,000 positions x 576 FP8 bytes);
  * the cache is paged in 16-token blocks ("Kimi K2.6 DFlash on 8x MI300X",
    hardware stack: BLOCK_SIZE=16 is required for DFlash + MLA);
  * queries are 1 token, or 1 + st speculative-verification tokens per
    sequence (section 1 of the Kimi K3 page, #51705 multi-token verification);
  * FP8 caches are e4m3 with one fp32 scale per token (scale = max|row|/448).

Unused tail slots of each sequence's last page, and pages that no sequence
owns, are poisoned with NaN so that any read outside the visible range shows
up in the output.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

PAGE = 16          # tokens per page
D_LATENT = 512     # c_kv width, also the value width
D_ROPE = 64        # k_pe width
D_QK = D_LATENT + D_ROPE  # 576 values per cached position
FP8_MAX = 448.0    # largest finite e4m3fn magnitude

KV_BF16 = "bf16"
KV_FP8 = "fp8"

BF16_NAN_BITS = 0x7FC0
FP8_NAN_BYTE = 0x7F


@dataclasses.dataclass(frozen=True)
class Config:
    """One decode workload: batch B, query tokens T, heads H, context recipe."""
    name: str
    B: int
    T: int
    H: int
    ctx: tuple            # ("fixed", n) | ("uniform", lo, hi) | ("loguniform", lo, hi)
    kv: str               # KV_BF16 | KV_FP8
    shuffle: bool         # shuffled global page table (else identity)
    seed: int
    partitions: int = 1   # >1: round-robin context partitioning + merge
    note: str = ""


# The five workloads of the problem statement, smallest first.
CONFIGS = {
    c.name: c
    for c in [
        Config("single_query_256", B=1, T=1, H=16, ctx=("fixed", 256), kv=KV_BF16,
               shuffle=False, seed=1001,
               note="single-query sanity, identity page table"),
        Config("spec_verify_small", B=8, T=3, H=12, ctx=("uniform", 1024, 8192), kv=KV_BF16,
               shuffle=True, seed=1002,
               note="1 + st=2 causal drafts, 12 heads per rank"),
        Config("batched_verify_fp8_32k", B=32, T=3, H=96, ctx=("fixed", 32768), kv=KV_FP8,
               shuffle=True, seed=1003,
               note="FP8 e4m3 per-token-scaled KV, causal drafts"),
        Config("long_ctx_142k", B=1, T=1, H=96, ctx=("fixed", 142000), kv=KV_FP8,
               shuffle=True, seed=1004,
               note="long-context single stream, split-KV over >=148 chunks"),
        Config("ragged_dcp8", B=64, T=3, H=96, ctx=("loguniform", 512, 131072), kv=KV_FP8,
               shuffle=True, seed=1005, partitions=8,
               note="ragged batch, 8-way round-robin context partitions merged by LSE"),
    ]
}
CONFIG_ORDER = list(CONFIGS)


@dataclasses.dataclass
class Workload:
    """Inputs of one ``mla_decode`` call (all tensors on one device)."""
    q_lat: torch.Tensor          # [B,T,H,512] bf16
    q_pe: torch.Tensor           # [B,T,H,64] bf16
    kv_pages: torch.Tensor       # [P,16,576] bf16, or uint8 holding e4m3fn bytes
    kv_scale: Optional[torch.Tensor]   # [P,16] fp32 (FP8 only)
    page_table: torch.Tensor     # [B,max_pages] int32, -1 where unused
    ctx_lens: torch.Tensor       # [B] int32
    vis_lens: Optional[torch.Tensor]   # [B,T] int32 or None
    sm_scale: float
    kv_dtype: str
    name: str = ""

    @property
    def B(self):
        return self.q_lat.shape[0]

    @property
    def T(self):
        return self.q_lat.shape[1]

    @property
    def H(self):
        return self.q_lat.shape[2]

    @property
    def num_pages(self):
        return self.kv_pages.shape[0]

    def to(self, device) -> "Workload":
        mv = lambda t: None if t is None else t.to(device)
        return dataclasses.replace(
            self, q_lat=mv(self.q_lat), q_pe=mv(self.q_pe), kv_pages=mv(self.kv_pages),
            kv_scale=mv(self.kv_scale), page_table=mv(self.page_table),
            ctx_lens=mv(self.ctx_lens), vis_lens=mv(self.vis_lens))

    def visible_positions(self) -> int:
        """Number of (sequence, position) pairs whose KV row is read once."""
        return int(self.ctx_lens.to(torch.int64).sum())

    def kv_bytes_per_position(self) -> int:
        """bf16: 1,152; FP8: 576 codes + a 4-byte scale, or 576 with one static scale."""
        if self.kv_dtype == KV_BF16:
            return D_QK * 2
        return D_QK if self.kv_scale is not None and self.kv_scale.numel() == 1 else D_QK + 4

    def kv_label(self) -> str:
        """Cache format: "bf16", "fp8" (per-position scales) or "fp8-static"."""
        if self.kv_dtype == KV_FP8 and self.kv_scale is not None and self.kv_scale.numel() == 1:
            return KV_FP8 + "-static"
        return self.kv_dtype


DEFAULT_SM_SCALE = 1.0 / math.sqrt(192.0)


def _ctx_lengths(cfg: Config, gen: torch.Generator) -> torch.Tensor:
    kind = cfg.ctx[0]
    if kind == "fixed":
        return torch.full((cfg.B,), int(cfg.ctx[1]), dtype=torch.int64)
    if kind == "uniform":
        lo, hi = cfg.ctx[1], cfg.ctx[2]
        return torch.randint(lo, hi + 1, (cfg.B,), generator=gen, dtype=torch.int64)
    if kind == "loguniform":
        lo, hi = cfg.ctx[1], cfg.ctx[2]
        u = torch.rand((cfg.B,), generator=gen, dtype=torch.float64)
        v = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
        return torch.round(v).to(torch.int64).clamp_(lo, hi)
    raise ValueError(kind)


def quantize_fp8_rows(x: torch.Tensor):
    """Per-row e4m3fn quantisation of fp32 rows: scale = max|row|/448.

    Returns (uint8 codes, fp32 scales).  A row of zeros gets scale 1.
    """
    amax = x.abs().amax(dim=-1)
    scale = amax / FP8_MAX
    scale = torch.where(scale > 0, scale, torch.ones_like(scale))
    codes = (x / scale.unsqueeze(-1)).clamp_(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    return codes.view(torch.uint8), scale.to(torch.float32)


def _normal(shape, gen, device, dtype=torch.float32):
    return torch.randn(shape, generator=gen, device=device, dtype=dtype)


def build_paged_cache(rows_per_seq, kv: str, gen: torch.Generator, device="cpu",
                      shuffle=True, spare_pages=3, row_source=None):
    """Allocate a page pool holding each sequence's rows in 16-token pages.

    rows_per_seq: list of context lengths.  row_source(b) -> [ctx_b, 576] fp32
    rows for sequence b; when None the rows are drawn from N(0,1) with ``gen``.
    Returns (kv_pages, kv_scale, page_table) with unused slots NaN-poisoned.
    """
    ctx = [int(c) for c in rows_per_seq]
    npages = [(c + PAGE - 1) // PAGE for c in ctx]
    total = sum(npages) + spare_pages
    max_pages = max(max(npages), 1)
    if shuffle:
        perm = torch.randperm(total, generator=gen).to(torch.int64)
    else:
        perm = torch.arange(total, dtype=torch.int64)
    page_table = torch.full((len(ctx), max_pages), -1, dtype=torch.int32)
    if kv == KV_BF16:
        pages = torch.empty((total, PAGE, D_QK), dtype=torch.bfloat16, device=device)
        pages.view(torch.int16).fill_(BF16_NAN_BITS)
        scales = None
    else:
        pages = torch.full((total, PAGE, D_QK), FP8_NAN_BYTE, dtype=torch.uint8, device=device)
        scales = torch.full((total, PAGE), float("nan"), dtype=torch.float32, device=device)
    cursor = 0
    for b, c in enumerate(ctx):
        ids = perm[cursor:cursor + npages[b]]
        cursor += npages[b]
        page_table[b, :npages[b]] = ids.to(torch.int32)
        if c == 0:
            continue
        rows = row_source(b) if row_source is not None else _normal((c, D_QK), gen, device)
        pad = npages[b] * PAGE - c
        dev_ids = ids.to(device)
        if kv == KV_BF16:
            full = torch.empty((npages[b] * PAGE, D_QK), dtype=torch.bfloat16, device=device)
            full.view(torch.int16).fill_(BF16_NAN_BITS)
            full[:c] = rows.to(torch.bfloat16)
            pages[dev_ids] = full.view(npages[b], PAGE, D_QK)
        else:
            codes, sc = quantize_fp8_rows(rows.to(torch.float32))
            full = torch.full((npages[b] * PAGE, D_QK), FP8_NAN_BYTE, dtype=torch.uint8, device=device)
            full[:c] = codes
            fsc = torch.full((npages[b] * PAGE,), float("nan"), dtype=torch.float32, device=device)
            fsc[:c] = sc
            pages[dev_ids] = full.view(npages[b], PAGE, D_QK)
            scales[dev_ids] = fsc.view(npages[b], PAGE)
        del pad
    return pages, scales, page_table.to(device)


def make_workload(name: str, device="cpu", kv: Optional[str] = None, seed: Optional[int] = None,
                  B: Optional[int] = None, ctx_override=None, H: Optional[int] = None,
                  T: Optional[int] = None) -> Workload:
    """Build the named workload deterministically from its seed.

    ``kv`` switches the cache format (e.g. the bf16 variant of the 142K
    workload); ``B``/``ctx_override``/``H``/``T`` shrink a workload for tests
    while keeping its structure (shuffled pages, draft tokens, FP8 scales).
    Random draws happen on ``device`` with a generator seeded there.
    """
    cfg = CONFIGS[name]
    if B is not None or ctx_override is not None or H is not None or T is not None:
        cfg = dataclasses.replace(cfg, B=B or cfg.B, H=H or cfg.H, T=T or cfg.T,
                                  ctx=ctx_override or cfg.ctx)
    return make_from_config(cfg, device=device, kv=kv, seed=seed)


def make_from_config(cfg: Config, device="cpu", kv: Optional[str] = None,
                     seed: Optional[int] = None) -> Workload:
    """Build a workload from an explicit ``Config`` (see ``make_workload``)."""
    kv = kv or cfg.kv
    gen_cpu = torch.Generator(device="cpu")
    gen_cpu.manual_seed(cfg.seed if seed is None else seed)
    gen_dev = gen_cpu if str(device) == "cpu" else torch.Generator(device=device)
    if gen_dev is not gen_cpu:
        gen_dev.manual_seed((cfg.seed if seed is None else seed) + 7919)
    ctx = _ctx_lengths(cfg, gen_cpu)
    q_lat = _normal((cfg.B, cfg.T, cfg.H, D_LATENT), gen_dev, device).to(torch.bfloat16)
    q_pe = _normal((cfg.B, cfg.T, cfg.H, D_ROPE), gen_dev, device).to(torch.bfloat16)
    row_src = lambda b: _normal((int(ctx[b]), D_QK), gen_dev, device)
    pages, scales, pt = build_paged_cache(ctx.tolist(), kv, gen_cpu, device=device,
                                          shuffle=cfg.shuffle, row_source=row_src)
    return Workload(q_lat=q_lat, q_pe=q_pe, kv_pages=pages, kv_scale=scales, page_table=pt,
                    ctx_lens=ctx.to(torch.int32).to(device), vis_lens=None,
                    sm_scale=DEFAULT_SM_SCALE, kv_dtype=kv, name=cfg.name)


def gather_logical_rows(w: Workload, b: int) -> torch.Tensor:
    """The stored rows of sequence b in logical position order (raw storage dtype)."""
    c = int(w.ctx_lens[b])
    npg = (c + PAGE - 1) // PAGE
    ids = w.page_table[b, :npg].to(torch.int64)
    rows = w.kv_pages[ids].reshape(npg * PAGE, D_QK)[:c]
    if w.kv_scale is None:
        return rows, None
    return rows, w.kv_scale[ids].reshape(npg * PAGE)[:c]


def partition_round_robin(w: Workload, n_parts: int, gen_seed: int = 77) -> list:
    """Split every sequence's positions round-robin into ``n_parts`` caches.

    Position p of sequence b goes to partition p % n_parts at compacted index
    p // n_parts, the layout a context-parallel decode (DCP) gives each rank.
    Each partition gets its own shuffled page pool and a [B,T] ``vis_lens``
    holding how many of its positions each query token may see: query token t
    sits at absolute position ctx - T + t and sees every position <= itself.
    """
    B, T = w.B, w.T
    ctx = w.ctx_lens.to("cpu").to(torch.int64)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(gen_seed)
    parts = []
    logical = [gather_logical_rows(w, b) for b in range(B)]
    for k in range(n_parts):
        ctx_k = [max(0, (int(ctx[b]) - k + n_parts - 1) // n_parts) for b in range(B)]
        vis = torch.zeros((B, T), dtype=torch.int32)
        for b in range(B):
            for t in range(T):
                last = int(ctx[b]) - T + t       # absolute position of query token t
                vis[b, t] = (last - k) // n_parts + 1 if last >= k else 0
        npages = [(c + PAGE - 1) // PAGE for c in ctx_k]
        total = sum(npages) + 1
        perm = torch.randperm(total, generator=gen)
        pt = torch.full((B, max(max(npages), 1)), -1, dtype=torch.int32)
        dev = w.kv_pages.device
        if w.kv_dtype == KV_BF16:
            pages = torch.empty((total, PAGE, D_QK), dtype=torch.bfloat16, device=dev)
            pages.view(torch.int16).fill_(BF16_NAN_BITS)
            scales = None
        else:
            pages = torch.full((total, PAGE, D_QK), FP8_NAN_BYTE, dtype=torch.uint8, device=dev)
            scales = torch.full((total, PAGE), float("nan"), dtype=torch.float32, device=dev)
        cur = 0
        for b in range(B):
            ids = perm[cur:cur + npages[b]]
            cur += npages[b]
            pt[b, :npages[b]] = ids.to(torch.int32)
            if ctx_k[b] == 0:
                continue
            rows, sc = logical[b]
            sel = rows[k::n_parts]
            full = torch.empty((npages[b] * PAGE, D_QK), dtype=pages.dtype, device=dev)
            if w.kv_dtype == KV_BF16:
                full.view(torch.int16).fill_(BF16_NAN_BITS)
            else:
                full.fill_(FP8_NAN_BYTE)
            full[:ctx_k[b]] = sel
            pages[ids.to(dev)] = full.view(npages[b], PAGE, D_QK)
            if scales is not None:
                fsc = torch.full((npages[b] * PAGE,), float("nan"), dtype=torch.float32, device=dev)
                fsc[:ctx_k[b]] = sc[k::n_parts]
                scales[ids.to(dev)] = fsc.view(npages[b], PAGE)
        parts.append(Workload(q_lat=w.q_lat, q_pe=w.q_pe, kv_pages=pages, kv_scale=scales,
                              page_table=pt.to(dev),
                              ctx_lens=torch.tensor(ctx_k, dtype=torch.int32, device=dev),
                              vis_lens=vis.to(dev), sm_scale=w.sm_scale, kv_dtype=w.kv_dtype,
                              name=f"{w.name}/part{k}"))
    return parts


def ragged_drafts(w: Workload, n_new=None, seed: int = 23) -> Workload:
    """The same batch with a per-sequence number of query tokens n_new[b] in
    [1, T] (drawn uniformly unless given), packed into the first n_new[b] of
    the T query slots.  Sequence b's last n_new[b] cached positions are its
    new tokens: slot t < n_new[b] sits at position ctx - n_new[b] + t and sees
    every position up to itself; the remaining slots are padding and see
    nothing (``vis_lens`` 0).  Returns the workload and n_new."""
    B, T = w.B, w.T
    if n_new is None:
        gen = torch.Generator(device="cpu")
        gen.manual_seed(seed)
        n_new = torch.randint(1, T + 1, (B,), generator=gen)
    n_new = torch.as_tensor(n_new, dtype=torch.int64).cpu()
    ctx = w.ctx_lens.to("cpu").to(torch.int64)
    if n_new.shape != (B,) or bool((n_new < 1).any()) or bool((n_new > T).any()) or bool((n_new > ctx).any()):
        raise ValueError("need 1 <= n_new[b] <= min(T, ctx_lens[b])")
    t = torch.arange(T).unsqueeze(0)
    vis = torch.where(t < n_new.unsqueeze(1), ctx.unsqueeze(1) - n_new.unsqueeze(1) + t + 1, 0)
    return dataclasses.replace(w, vis_lens=vis.to(torch.int32).to(w.ctx_lens.device)), n_new


def one_sequence(w: Workload, b: int, T: Optional[int] = None) -> Workload:
    """Sequence b alone with its first T query slots (default all) and the
    default causality (no ``vis_lens``); the cache is shared."""
    T = w.T if T is None else T
    return dataclasses.replace(w, q_lat=w.q_lat[b:b + 1, :T].contiguous(),
                               q_pe=w.q_pe[b:b + 1, :T].contiguous(),
                               page_table=w.page_table[b:b + 1].contiguous(),
                               ctx_lens=w.ctx_lens[b:b + 1].contiguous(), vis_lens=None)


def static_scale_workload(w: Workload) -> Workload:
    """The same FP8 workload re-quantised with one per-tensor scale: the
    dequantised cache values (unused slots stay NaN) divided by
    s = max|value| / 448, rounded to e4m3; kv_scale becomes the one-element
    tensor [s]."""
    if w.kv_dtype != KV_FP8:
        raise ValueError("a static scale applies to FP8 caches")
    v = w.kv_pages.view(torch.float8_e4m3fn).to(torch.float32) * w.kv_scale.unsqueeze(-1)
    s = torch.nan_to_num(v.abs(), nan=0.0).amax() / FP8_MAX
    s = torch.where(s > 0, s, torch.ones_like(s)).to(torch.float32)
    codes = (v / s).clamp(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
    return dataclasses.replace(w, kv_pages=codes, kv_scale=s.reshape(1))


def permute_pages(w: Workload, seed: int = 5) -> Workload:
    """Same logical cache with physical pages relabelled by a random permutation."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    P = w.num_pages
    perm = torch.randperm(P, generator=gen)           # new slot of old page i
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(P)
    dev = w.kv_pages.device
    pages = w.kv_pages[inv.to(dev)]
    scales = None if w.kv_scale is None else w.kv_scale[inv.to(dev)]
    pt = w.page_table.to("cpu").to(torch.int64)
    new_pt = torch.where(pt >= 0, perm[pt.clamp(min=0)], pt).to(torch.int32)
    return dataclasses.replace(w, kv_pages=pages, kv_scale=scales, page_table=new_pt.to(dev))


def pad_heads(w: Workload, H_to: int) -> Workload:
    """Zero-fill extra query heads (the 12 -> 16 head-padding adapter, queries only)."""
    B, T, H = w.B, w.T, w.H
    ql = torch.zeros((B, T, H_to, D_LATENT), dtype=w.q_lat.dtype, device=w.q_lat.device)
    qp = torch.zeros((B, T, H_to, D_ROPE), dtype=w.q_pe.dtype, device=w.q_pe.device)
    ql[:, :, :H] = w.q_lat
    qp[:, :, :H] = w.q_pe
    return dataclasses.replace(w, q_lat=ql, q_pe=qp)


def sample_rows(B: int, T: int, H: int, n: int, seed: int = 11) -> torch.Tensor:
    """Flat row ids (b*T*H + t*H + h) for sampled parity; always includes the
    first and last row of the batch and every draft token of sequence 0."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    total = B * T * H
    picks = set(torch.randint(0, total, (n,), generator=gen).tolist())
    picks.update({0, total - 1})
    picks.update(t * H for t in range(T))
    picks.update(t * H + H - 1 for t in range(T))
    return torch.tensor(sorted(picks), dtype=torch.int64)
