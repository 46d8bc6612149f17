"""INT4 KV pages: quantisation, dequantisation and the page summaries of the
dequantised keys.

Test infrastructure only (see the package docstring).

Source: LServe + SampleAttention blog post, "LServe - Decode Phase" (combined
with INT4 KV quantization the gains stack: sparsity cuts the number of pages
touched, quantization the bytes of each page) and Fig. 2 ("INT4 KV further
reduces bytes per read").  The pages name no scheme; the one declared here (a
reading) is asymmetric INT4 with one step and offset

  * per (page, KV head, channel) for keys, over the page's valid tokens, and
  * per (page, KV head, token) for values, over the d channels,

which keeps an outlier channel of the keys from flattening the others.  With
lo, hi the minimum and maximum of the group (bf16 values taken as float32), in
float32 arithmetic:

    s     = (hi - lo) / 15                       IEEE division
    code  = clamp(rint((x - lo) / s), 0, 15)     (code 0 when s == 0)
    deq   = bf16(fma(code, s, lo))               the float32 fused multiply-add,
                                                 rounded to bf16 (nearest even)

s and lo are stored as float32.  Rows past a sequence's end get code 0 and, for
values, s = lo = 0.  Codes decide integers, so both sides take them in float32:
this module mirrors those float32 steps (a fused multiply-add is the exact
product and sum rounded once; code * s + lo is exact in float64 here).

Layouts (d channels, pages of 64 token rows):
    kq, vq   uint8 [NP, Hkv, 64, d/2]   (byte j of a row: channel 2j in the low nibble)
    kpar     fp32  [NP, Hkv, 2, d]      (row 0: s per channel, row 1: lo)
    vpar     fp32  [NP, Hkv, 2, 64]     (row 0: s per token,   row 1: lo)
"""
from __future__ import annotations

import numpy as np
import torch

from .selection import PAGE, n_pages, page_stats


def bf16_round(x) -> np.ndarray:
    """float32 -> nearest bf16 (ties to even), returned as float32 values."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _step(lo, hi):
    return ((hi - lo) / np.float32(15.0)).astype(np.float32)


def _codes(x, lo, s):
    with np.errstate(divide="ignore", invalid="ignore"):
        c = np.rint(((x - lo).astype(np.float32) / s).astype(np.float32))
    c = np.where(s > 0, c, 0.0)
    return np.clip(c, 0, 15).astype(np.uint8)


def dequant(code, s, lo) -> np.ndarray:
    """bf16(fma(code, s, lo)) as float32 values."""
    exact = code.astype(np.float64) * s.astype(np.float64) + lo.astype(np.float64)
    return bf16_round(exact.astype(np.float32))


def quantize_pages(k_pages, v_pages, page_table, seq_lens):
    """(kq, kpar, vq, vpar, kdeq, vdeq) for every page a sequence holds; pages no
    sequence holds stay zero.  k_pages/v_pages: bf16 values [NP, Hkv, 64, d]."""
    k = np.asarray(k_pages, dtype=np.float32)
    v = np.asarray(v_pages, dtype=np.float32)
    NP, Hkv, P, d = k.shape
    kq = np.zeros((NP, Hkv, P, d // 2), np.uint8)
    vq = np.zeros((NP, Hkv, P, d // 2), np.uint8)
    kpar = np.zeros((NP, Hkv, 2, d), np.float32)
    vpar = np.zeros((NP, Hkv, 2, P), np.float32)
    kdeq = np.zeros_like(k)
    vdeq = np.zeros_like(v)
    for b in range(len(seq_lens)):
        L = int(seq_lens[b])
        for i in range(n_pages(L)):
            p = int(page_table[b][i])
            nv = min(PAGE, L - i * PAGE)
            for g in range(Hkv):
                kk = k[p, g, :nv, :]
                lo, hi = kk.min(axis=0), kk.max(axis=0)
                st = _step(lo, hi)
                codes = np.zeros((P, d), np.uint8)
                codes[:nv] = _codes(kk, lo[None, :], st[None, :])
                kq[p, g] = codes[:, 0::2] | (codes[:, 1::2] << 4)
                kpar[p, g, 0], kpar[p, g, 1] = st, lo
                kdeq[p, g] = dequant(codes, st[None, :], lo[None, :])
                vv = v[p, g, :nv, :]
                lo, hi = vv.min(axis=1), vv.max(axis=1)
                st = _step(lo, hi)
                codes = np.zeros((P, d), np.uint8)
                codes[:nv] = _codes(vv, lo[:, None], st[:, None])
                vq[p, g] = codes[:, 0::2] | (codes[:, 1::2] << 4)
                vpar[p, g, 0, :nv], vpar[p, g, 1, :nv] = st, lo
                vdeq[p, g] = dequant(codes, vpar[p, g, 0][:, None], vpar[p, g, 1][:, None])
    return kq, kpar, vq, vpar, kdeq, vdeq


def quantized_stats(kdeq, page_table, seq_lens, head_kind):
    """Page summaries of the dequantised keys (what the decode step attends to)."""
    return page_stats(kdeq, page_table, seq_lens, head_kind)
