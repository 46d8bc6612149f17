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
    deq   = fma(code, s, lo)                     the float32 fused multiply-add

s and lo are stored as float32.  Rows past a sequence's end get code 0 and, for
values, s = lo = 0.  Codes decide integers, so both sides take them in float32:
this module mirrors those float32 steps (a fused multiply-add is the exact
product and sum rounded once; code * s + lo is exact in float64 here).

The dequantised values stay float32: the decode step never forms them in bf16
(it multiplies the integer codes by the steps folded into the other operand).
The page summaries are bf16, so the summaries of the dequantised keys round
the minimum down and the maximum up: the bound stays a bound.

Everything here is in the plain index order of the pages: codes [page, KV
head, token, channel], key steps and offsets [page, KV head, channel], value
steps and offsets [page, KV head, token].  How the library packs codes into
bytes is a storage format, not part of the method; the tests unpack the
library's bytes into this order before comparing.
"""
from __future__ import annotations

from typing import NamedTuple

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


def bf16_round_down(x) -> np.ndarray:
    """float32 -> the largest bf16 <= x (toward -inf), as float32 values."""
    return _bf16_directed(x, up=False)


def bf16_round_up(x) -> np.ndarray:
    """float32 -> the smallest bf16 >= x (toward +inf), as float32 values."""
    return _bf16_directed(x, up=True)


def _bf16_directed(x, up):
    # bf16 is the top half of a float32: truncating the low 16 bits rounds the
    # magnitude down; one more unit of the top half (when bits were dropped)
    # rounds it up.  Infinities have no low bits and pass through.
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32)
    trunc = b & np.uint32(0xFFFF0000)
    inexact = (b & np.uint32(0xFFFF)) != 0
    neg = (b >> np.uint32(31)) == 1
    away = inexact & (neg != up)        # magnitude must grow: up for x > 0, down for x < 0
    out = np.where(away, trunc + np.uint32(0x10000), trunc).astype(np.uint32)
    return out.view(np.float32)


def dequant(code, s, lo) -> np.ndarray:
    """fma(code, s, lo) in float32: the exact value rounded once."""
    exact = code.astype(np.float64) * s.astype(np.float64) + lo.astype(np.float64)
    return exact.astype(np.float32)


class Int4Pages(NamedTuple):
    """INT4 pages in plain index order (pages no sequence holds stay zero)."""
    kcode: np.ndarray   # uint8 [NP, Hkv, 64, d]
    kstep: np.ndarray   # float32 [NP, Hkv, d]
    klo: np.ndarray     # float32 [NP, Hkv, d]
    vcode: np.ndarray   # uint8 [NP, Hkv, 64, d]
    vstep: np.ndarray   # float32 [NP, Hkv, 64]
    vlo: np.ndarray     # float32 [NP, Hkv, 64]
    kdeq: np.ndarray    # float32 [NP, Hkv, 64, d]
    vdeq: np.ndarray    # float32 [NP, Hkv, 64, d]


def quantize_pages(k_pages, v_pages, page_table, seq_lens) -> Int4Pages:
    """Codes, steps, offsets and dequantised values of every page a sequence
    holds.  k_pages/v_pages: bf16 values [NP, Hkv, 64, d].  Keys: one group per
    (page, KV head, channel) over the page's valid tokens; values: one group per
    (page, KV head, token) over the d channels.  Rows past a sequence's end keep
    code 0 (and, for values, s = lo = 0)."""
    k = np.asarray(k_pages, dtype=np.float32)
    v = np.asarray(v_pages, dtype=np.float32)
    NP, Hkv, P, d = k.shape
    kcode = np.zeros((NP, Hkv, P, d), np.uint8)
    vcode = np.zeros((NP, Hkv, P, d), np.uint8)
    kstep = np.zeros((NP, Hkv, d), np.float32)
    klo = np.zeros((NP, Hkv, d), np.float32)
    vstep = np.zeros((NP, Hkv, P), np.float32)
    vlo = np.zeros((NP, Hkv, P), np.float32)
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
                kcode[p, g, :nv] = _codes(kk, lo[None, :], st[None, :])
                kstep[p, g], klo[p, g] = st, lo
                kdeq[p, g] = dequant(kcode[p, g], st[None, :], lo[None, :])
                vv = v[p, g, :nv, :]
                lo, hi = vv.min(axis=1), vv.max(axis=1)
                st = _step(lo, hi)
                vcode[p, g, :nv] = _codes(vv, lo[:, None], st[:, None])
                vstep[p, g, :nv], vlo[p, g, :nv] = st, lo
                vdeq[p, g] = dequant(vcode[p, g], vstep[p, g][:, None], vlo[p, g][:, None])
    return Int4Pages(kcode, kstep, klo, vcode, vstep, vlo, kdeq, vdeq)


def quantized_stats(kdeq, page_table, seq_lens, head_kind):
    """Page summaries (bf16 values) of the dequantised keys, what the decode step
    attends to: the minimum rounded down, the maximum rounded up."""
    st = page_stats(kdeq, page_table, seq_lens, head_kind)
    out = st.copy()
    out[..., 0, :] = bf16_round_down(st[..., 0, :].astype(np.float32))
    out[..., 1, :] = bf16_round_up(st[..., 1, :].astype(np.float32))
    return out
