"""Seeded synthetic inputs for the unified sparse-attention path.

This module is shared by the tests, the bench and the oracle checks.  It holds
none of the attention arithmetic: only random draws, one rounding to bf16,
memory layout (scattering contiguous K/V into a shuffled page pool) and the
shapes of the five workloads.  Neither the oracle nor the CUDA binding imports
anything else from the other side.

Shapes follow the long-context serving cases described for LServe (mlsanity
"LServe: Efficient Long-sequence LLM Serving with Unified Sparse Attention",
Abstract; LServe + SampleAttention blog post, "LServe - Prefill Phase" and
"LServe - Decode Phase"):

* half of the KV heads are streaming heads (sink + local window), the rest are
  dense (retrieval) heads;
* keys carry a few "anchor" positions (a shared direction u added to keys and
  queries) so that query-aware page selection has something to find, in the
  spirit of the column pattern of the blog's "SampleAttention - Column Pattern";
* the long-prefill workload carries a vertical-slash block mask (the blog's
  "Column Pattern" + "Slash Pattern", Fig. 3).

Every tensor is drawn in fp32 from a seeded ``torch.Generator`` on the device
the caller asks for, rounded once to bf16 (round-to-nearest-even) and never
touched again.  CPU and CUDA generators give different (each deterministic)
streams; a test always hands the very same bf16 tensor to both sides.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import torch

PAGE = 64          # tokens per physical KV page
LOGICAL = 16       # tokens per logical page (granularity of the key min/max summary)
TILE = 64          # prefill tile (query rows and KV columns)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload (shape + distribution recipe)."""
    name: str
    seed: int
    # prefill shape
    B: int
    S: int
    Hq: int
    Hkv: int
    d: int
    n_streaming: int          # number of streaming KV heads (chosen by a seeded permutation)
    sink: int
    local: int
    anchors: int              # anchor key positions per (batch, KV head)
    outlier_channels: int = 0  # channels per KV head whose keys are scaled
    outlier_scale: float = 1.0
    # block mask on dense heads (vertical-slash); None = no mask
    mask_columns: int = 0
    mask_band: int = 0
    mask_fill: Optional[float] = None
    # decode shape
    dec_B: int = 0
    ctx: int = 0
    token_budget: int = 0
    pool_pages: int = 0        # physical pages in the pool (>= dec_B * ceil(ctx / PAGE))
    dec_anchors: int = 0
    has_prefill: bool = True
    has_decode: bool = True

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


# Vertical-slash fill fraction that brings the long-prefill mask to ~30 % of the
# causal tiles: 16 columns + an 8-tile band cover ~1.55 % of the 2048x2048 causal
# tiles, and 0.0155 + 0.9845 * 0.289 = 0.300.
FILL_30PCT = 0.289

WORKLOADS = {
    "tiny": Workload(
        name="tiny", seed=1000, B=1, S=1024, Hq=4, Hkv=2, d=64, n_streaming=1,
        sink=64, local=256, anchors=8, dec_B=1, ctx=1024, token_budget=256,
        pool_pages=16, dec_anchors=8),
    "llama3_8b_32k": Workload(
        name="llama3_8b_32k", seed=1001, B=1, S=32768, Hq=32, Hkv=8, d=128,
        n_streaming=4, sink=64, local=256, anchors=32, dec_B=1, ctx=32768,
        token_budget=4096, pool_pages=512, dec_anchors=32),
    "llama3_8b_decode_b16_64k": Workload(
        name="llama3_8b_decode_b16_64k", seed=1002, B=0, S=0, Hq=32, Hkv=8,
        d=128, n_streaming=4, sink=64, local=256, anchors=0,
        outlier_channels=4, outlier_scale=8.0, dec_B=16, ctx=65536,
        token_budget=4096, pool_pages=16384, dec_anchors=64, has_prefill=False),
    "llama3_8b_prefill_128k_vslash": Workload(
        name="llama3_8b_prefill_128k_vslash", seed=1003, B=1, S=131072, Hq=32,
        Hkv=8, d=128, n_streaming=4, sink=64, local=256, anchors=32,
        mask_columns=16, mask_band=8, mask_fill=FILL_30PCT, has_decode=False),
    "llama2_7b_mha": Workload(
        name="llama2_7b_mha", seed=1004, B=1, S=65536, Hq=32, Hkv=32, d=128,
        n_streaming=16, sink=64, local=256, anchors=64, dec_B=4, ctx=262144,
        token_budget=8192, pool_pages=16384, dec_anchors=64),
}
# Half-length version of the long prefill (same recipe), sized for profiler captures.
WORKLOADS["llama3_8b_prefill_64k_vslash"] = dataclasses.replace(
    WORKLOADS["llama3_8b_prefill_128k_vslash"], name="llama3_8b_prefill_64k_vslash", S=65536)
# The MHA decode at 4 x 64K (a quarter of the context), sized for profiler captures of the
# G = 1 scoring path: 4.3 GB of pool, 134 MB of summaries (more than L2 holds).
WORKLOADS["llama2_7b_mha_decode_b4_64k"] = dataclasses.replace(
    WORKLOADS["llama2_7b_mha"], name="llama2_7b_mha_decode_b4_64k", ctx=65536, pool_pages=4096)
# The literal reading of the long-prefill mask (5 % random fill, ~6.5 % density).
WORKLOADS["llama3_8b_prefill_128k_vslash_literal"] = dataclasses.replace(
    WORKLOADS["llama3_8b_prefill_128k_vslash"],
    name="llama3_8b_prefill_128k_vslash_literal", mask_fill=0.05)


def _seed(*parts) -> int:
    """Deterministic 63-bit seed from any tuple of ints/strings."""
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def head_kind(w: Workload) -> torch.Tensor:
    """uint8[Hkv]: 0 = dense KV head, 1 = streaming KV head.

    A seeded permutation picks ``n_streaming`` heads, so streaming heads are not
    contiguous and no kernel may assume they are.
    """
    g = _gen("cpu", w.seed, "head_kind")
    perm = torch.randperm(w.Hkv, generator=g)
    kind = torch.zeros(w.Hkv, dtype=torch.uint8)
    kind[perm[: w.n_streaming]] = 1
    return kind


def anchor_dirs(w: Workload, device="cpu") -> torch.Tensor:
    """fp32[Hkv, d]: one seeded unit vector u per KV head."""
    g = _gen(device, w.seed, "u")
    u = torch.randn(w.Hkv, w.d, generator=g, device=device, dtype=torch.float32)
    return u / u.norm(dim=-1, keepdim=True)


def _keys(w: Workload, b: int, n_tok: int, n_anchor: int, tag: str, device) -> torch.Tensor:
    """fp32[n_tok, Hkv, d] keys of one sequence: N(0,1), outlier channels, anchors."""
    g = _gen(device, w.seed, tag, "k", b)
    k = torch.randn(n_tok, w.Hkv, w.d, generator=g, device=device, dtype=torch.float32)
    if w.outlier_channels:
        go = _gen("cpu", w.seed, "outlier")
        for h in range(w.Hkv):
            ch = torch.randperm(w.d, generator=go)[: w.outlier_channels].to(device)
            k[:, h, ch] *= w.outlier_scale
    if n_anchor:
        u = anchor_dirs(w, device)
        ga = _gen("cpu", w.seed, tag, "anchors", b)
        for h in range(w.Hkv):
            pos = torch.randperm(n_tok, generator=ga)[:n_anchor].to(device)
            k[pos, h, :] += 3.0 * u[h]
    return k


def _queries(w: Workload, b: int, n_tok: int, tag: str, device, with_anchor: bool) -> torch.Tensor:
    g = _gen(device, w.seed, tag, "q", b)
    q = torch.randn(n_tok, w.Hq, w.d, generator=g, device=device, dtype=torch.float32)
    if with_anchor:
        u = anchor_dirs(w, device)                      # [Hkv, d]
        q += u.repeat_interleave(w.G, dim=0)[None]     # query head h uses KV head h // G
    return q


def _values(w: Workload, b: int, n_tok: int, tag: str, device) -> torch.Tensor:
    g = _gen(device, w.seed, tag, "v", b)
    return torch.randn(n_tok, w.Hkv, w.d, generator=g, device=device, dtype=torch.float32)


def prefill_inputs(w: Workload, device="cpu", S: Optional[int] = None, B: Optional[int] = None):
    """q bf16[B,S,Hq,d], k,v bf16[B,S,Hkv,d] (optionally at a smaller S / B)."""
    S = w.S if S is None else S
    B = w.B if B is None else B
    qs, ks, vs = [], [], []
    for b in range(B):
        n_anchor = min(w.anchors, S)
        qs.append(_bf16(_queries(w, b, S, "prefill", device, n_anchor > 0)))
        ks.append(_bf16(_keys(w, b, S, n_anchor, "prefill", device)))
        vs.append(_bf16(_values(w, b, S, "prefill", device)))
    return torch.stack(qs), torch.stack(ks), torch.stack(vs)


def block_mask(w: Workload, S: Optional[int] = None, fill: Optional[float] = None,
               device="cpu", B: Optional[int] = None) -> Optional[torch.Tensor]:
    """uint8[B, Hkv, S/64, S/64] vertical-slash block mask, or None.

    1 marks a kept KV tile.  Per (batch, KV head): every tile of ``mask_columns``
    seeded KV-tile columns, the diagonal band of ``mask_band`` tiles
    (0 <= qt - kt < band) and a seeded Bernoulli(fill) draw elsewhere.  Entries
    above the diagonal are drawn too: the attention ANDs the mask with
    causality, so they must have no effect.  Entries of streaming heads are drawn
    as well and must be ignored.
    """
    fill = w.mask_fill if fill is None else fill
    if fill is None:
        return None
    S = w.S if S is None else S
    B = w.B if B is None else B
    n = S // TILE
    out = torch.empty(B, w.Hkv, n, n, dtype=torch.uint8, device=device)
    qt = torch.arange(n, device=device)[:, None]
    kt = torch.arange(n, device=device)[None, :]
    band = (qt - kt >= 0) & (qt - kt < w.mask_band)
    for b in range(B):
        for h in range(w.Hkv):
            g = _gen(device, w.seed, "mask", b, h)
            m = torch.rand(n, n, generator=g, device=device) < fill
            gc = _gen("cpu", w.seed, "mask_cols", b, h)
            cols = torch.randperm(n, generator=gc)[: min(w.mask_columns, n)].to(device)
            m[:, cols] = True
            m |= band
            out[b, h] = m.to(torch.uint8)
    return out


@dataclasses.dataclass
class PagedCache:
    """A paged KV pool plus the per-sequence page table.

    k_pages, v_pages : bf16[NP, Hkv, PAGE, d]
    page_table       : int32[B, maxP]; entry i of row b is the physical page that
                       holds tokens [64 i, 64 i + 64) of sequence b (-1 = unused)
    seq_lens         : int32[B]
    """
    k_pages: torch.Tensor
    v_pages: torch.Tensor
    page_table: torch.Tensor
    seq_lens: torch.Tensor


def page_table(w: Workload, B: int, ctx_pages: int, NP: int, maxP: Optional[int] = None) -> torch.Tensor:
    """int32[B, maxP]: a seeded random permutation of the pool's pages."""
    maxP = ctx_pages if maxP is None else maxP
    g = _gen("cpu", w.seed, "page_perm")
    perm = torch.randperm(NP, generator=g)[: B * ctx_pages].to(torch.int32)
    pt = torch.full((B, maxP), -1, dtype=torch.int32)
    pt[:, :ctx_pages] = perm.view(B, ctx_pages)
    return pt


def scatter_to_pages(k: torch.Tensor, v: torch.Tensor, pt: torch.Tensor, NP: int) -> PagedCache:
    """Lay contiguous bf16 K/V [B, n_tok, Hkv, d] out into a page pool.

    Pure layout: token t of sequence b goes to page pt[b, t // 64], row t % 64.
    Rows of a partially filled last page, and pool pages no sequence uses, are
    filled with NaN so that a kernel that reads them poisons its result.
    """
    B, n_tok, Hkv, d = k.shape
    dev = k.device
    kp = torch.full((NP, Hkv, PAGE, d), float("nan"), dtype=torch.bfloat16, device=dev)
    vp = torch.full((NP, Hkv, PAGE, d), float("nan"), dtype=torch.bfloat16, device=dev)
    n_pages = (n_tok + PAGE - 1) // PAGE
    for b in range(B):
        pad = n_pages * PAGE - n_tok
        kb = torch.nn.functional.pad(k[b].float(), (0, 0, 0, 0, 0, pad), value=float("nan")).to(torch.bfloat16)
        vb = torch.nn.functional.pad(v[b].float(), (0, 0, 0, 0, 0, pad), value=float("nan")).to(torch.bfloat16)
        kb = kb.view(n_pages, PAGE, Hkv, d).permute(0, 2, 1, 3)
        vb = vb.view(n_pages, PAGE, Hkv, d).permute(0, 2, 1, 3)
        idx = pt[b, :n_pages].to(device=dev, dtype=torch.long)
        kp[idx] = kb
        vp[idx] = vb
    seq_lens = torch.full((B,), n_tok, dtype=torch.int32)
    return PagedCache(kp, vp, pt.clone(), seq_lens)


def decode_cache(w: Workload, device="cpu", B: Optional[int] = None, ctx: Optional[int] = None,
                 seq_lens: Optional[list] = None, NP: Optional[int] = None) -> PagedCache:
    """The decode workload's paged cache, filled one sequence at a time.

    ``seq_lens`` (optional) gives ragged lengths <= ctx per sequence; tokens past
    a sequence's length are NaN in the pool.
    """
    B = w.dec_B if B is None else B
    ctx = w.ctx if ctx is None else ctx
    n_pages = (ctx + PAGE - 1) // PAGE
    NP = max(w.pool_pages, B * n_pages) if NP is None else NP
    pt = page_table(w, B, n_pages, NP)
    kp = torch.full((NP, w.Hkv, PAGE, w.d), float("nan"), dtype=torch.bfloat16, device=device)
    vp = torch.full((NP, w.Hkv, PAGE, w.d), float("nan"), dtype=torch.bfloat16, device=device)
    lens = [ctx] * B if seq_lens is None else list(seq_lens)
    for b in range(B):
        n_anchor = min(w.dec_anchors, lens[b])
        kb = _keys(w, b, ctx, n_anchor, "decode", device)
        vb = _values(w, b, ctx, "decode", device)
        kb[lens[b]:] = float("nan")
        vb[lens[b]:] = float("nan")
        pad = n_pages * PAGE - ctx
        if pad:
            kb = torch.cat([kb, torch.full((pad, w.Hkv, w.d), float("nan"), device=device)])
            vb = torch.cat([vb, torch.full((pad, w.Hkv, w.d), float("nan"), device=device)])
        idx = pt[b, :n_pages].to(device=device, dtype=torch.long)
        kp[idx] = _bf16(kb).view(n_pages, PAGE, w.Hkv, w.d).permute(0, 2, 1, 3)
        vp[idx] = _bf16(vb).view(n_pages, PAGE, w.Hkv, w.d).permute(0, 2, 1, 3)
        del kb, vb
    return PagedCache(kp, vp, pt, torch.tensor(lens, dtype=torch.int32))


def decode_query(w: Workload, device="cpu", B: Optional[int] = None, step: int = 0) -> torch.Tensor:
    """bf16[B, Hq, d]: one query token per sequence (N(0,1) + u of its KV head)."""
    B = w.dec_B if B is None else B
    qs = [_queries(w, b, 1, f"decode_q{step}", device, w.dec_anchors > 0)[0] for b in range(B)]
    return _bf16(torch.stack(qs))
