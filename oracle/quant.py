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

Layouts (d channels, pages of 64 token rows; a byte holds two codes, the one
with the even nibble index n in its low four bits; nibble n of a 32-bit word
sits in byte n // 2 of the word, little-endian).  The order of the codes is a
permutation chosen so that a decode lane's share of a page is a few contiguous
words (see `k_code_position` and `v_code_position`):

    kq     uint8 [NP, Hkv, 64, d/2]   row = token; codes in k_code_position order
    vq     uint8 [NP, Hkv, 64 * d/2]  codes in v_code_position order
    kpar   fp32  [NP, Hkv, 2, d]      [0] = s, [1] = lo, channels in k_param_order
    vpar   fp32  [NP, Hkv, 64, 2]     (s, lo) per token
"""
from __future__ import annotations

import numpy as np
import torch

from .selection import PAGE, n_pages, page_stats


def k_code_position(d):
    """Nibble position of channel c within a key row of d/2 bytes: an array P of
    length d with P[c] = 2 * byte + (1 if high nibble).  A row is four chunks of
    d/8 bytes; chunk t holds the channels 16 k + 8 h + 2 t + e (k < d/16,
    h, e < 2).  Within chunk t, word w holds the eight nibbles n = j + 4 e of
    the channel pairs r = 4 w + j (j < 4), pair r being channels
    16 (r // 2) + 8 (r % 2) + 2 t + e.  d is a multiple of 32 (64 or 128)."""
    if d % 32:
        raise ValueError("the INT4 layouts need d to be a multiple of 32")
    pos = np.empty(d, np.int64)
    for t in range(4):
        for r in range(d // 8):
            w, j = divmod(r, 4)
            for e in range(2):
                c = 16 * (r // 2) + 8 * (r % 2) + 2 * t + e
                n = j + 4 * e
                byte = t * (d // 8) + 4 * w + n // 2
                pos[c] = 2 * byte + (n % 2)
    return pos


def k_param_order(d):
    """Channel held at each index of a kpar row: four chunks of d/4 entries;
    entry i of chunk t is channel 16 (i // 4) + 8 ((i // 2) % 2) + 2 t + i % 2."""
    return np.array([16 * (i // 4) + 8 * ((i // 2) % 2) + 2 * t + i % 2 for t in range(4) for i in range(d // 4)],
                    np.int64)


def v_code_position(d):
    """Nibble position of (token u, channel c) within a page's d/2 * 64 value
    bytes: an array P[64, d].  The page is four slices of 16 tokens; slice s is
    32 chunks of d/4 bytes, chunk 4 g + t holding, in word m (m < d/16), the
    nibbles n = j + 4 e with channel 16 m + g + 8 (j % 2) and token
    16 s + 2 t + 8 (j // 2) + e.  d is a multiple of 16."""
    if d % 16:
        raise ValueError("the INT4 layouts need d to be a multiple of 16")
    pos = np.empty((64, d), np.int64)
    for sl in range(4):
        for g in range(8):
            for t in range(4):
                chunk = (sl * 32 + 4 * g + t) * (d // 4)
                for m in range(d // 16):
                    for j in range(4):
                        for e in range(2):
                            c = 16 * m + g + 8 * (j % 2)
                            u = 16 * sl + 2 * t + 8 * (j // 2) + e
                            n = j + 4 * e
                            pos[u, c] = 2 * (chunk + 4 * m + n // 2) + (n % 2)
    return pos


def pack_nibbles(codes, pos, nbytes):
    """Place codes (any shape, values < 16) at nibble positions pos (same shape)."""
    out = np.zeros(2 * nbytes, np.uint8)
    out[pos.ravel()] = codes.ravel()
    return (out[0::2] | (out[1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed, pos):
    """Inverse of pack_nibbles: the codes at nibble positions pos."""
    nib = np.empty(2 * packed.size, np.uint8)
    nib[0::2] = packed & 15
    nib[1::2] = packed >> 4
    return nib[pos]


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


def quantize_pages(k_pages, v_pages, page_table, seq_lens):
    """(kq, kpar, vq, vpar, kdeq, vdeq) for every page a sequence holds; pages no
    sequence holds stay zero.  k_pages/v_pages: bf16 values [NP, Hkv, 64, d]."""
    k = np.asarray(k_pages, dtype=np.float32)
    v = np.asarray(v_pages, dtype=np.float32)
    NP, Hkv, P, d = k.shape
    kpos, vpos, korder = k_code_position(d), v_code_position(d), k_param_order(d)
    kq = np.zeros((NP, Hkv, P, d // 2), np.uint8)
    vq = np.zeros((NP, Hkv, P * d // 2), np.uint8)
    kpar = np.zeros((NP, Hkv, 2, d), np.float32)
    vpar = np.zeros((NP, Hkv, P, 2), np.float32)
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
                for r in range(P):
                    kq[p, g, r] = pack_nibbles(codes[r], kpos, d // 2)
                kpar[p, g, 0], kpar[p, g, 1] = st[korder], lo[korder]
                kdeq[p, g] = dequant(codes, st[None, :], lo[None, :])
                vv = v[p, g, :nv, :]
                lo, hi = vv.min(axis=1), vv.max(axis=1)
                st = _step(lo, hi)
                codes = np.zeros((P, d), np.uint8)
                codes[:nv] = _codes(vv, lo[:, None], st[:, None])
                vq[p, g] = pack_nibbles(codes, vpos, P * d // 2)
                vpar[p, g, :nv, 0], vpar[p, g, :nv, 1] = st, lo
                vdeq[p, g] = dequant(codes, vpar[p, g, :, 0][:, None], vpar[p, g, :, 1][:, None])
    return kq, kpar, vq, vpar, kdeq, vdeq


def quantized_stats(kdeq, page_table, seq_lens, head_kind):
    """Page summaries (bf16 values) of the dequantised keys, what the decode step
    attends to: the minimum rounded down, the maximum rounded up."""
    st = page_stats(kdeq, page_table, seq_lens, head_kind)
    out = st.copy()
    out[..., 0, :] = bf16_round_down(st[..., 0, :].astype(np.float32))
    out[..., 1, :] = bf16_round_up(st[..., 1, :].astype(np.float32))
    return out
