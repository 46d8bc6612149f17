"""Token-level decode attention over the selected pages.

Test infrastructure only (see the package docstring).

Sources: LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2
(fine-grained, token-level attention only inside the selected pages);
mlsanity LServe page, Abstract (streaming heads in both the prefilling and the
decoding stages).

Readings where the pages are silent: the cache holds all ``seq_len`` tokens of
the sequence, the current token's key and value included, and the query sits at
position seq_len - 1.  A dense KV head attends to every valid token (t <
seq_len) of its selected pages; a streaming KV head attends to the tokens t <
sink or t >= seq_len - local (exactly the last row of the prefill Lambda mask).
An empty token set gives out = 0 and lse = -inf.
"""
from __future__ import annotations

import numpy as np

from .selection import PAGE, select


def token_set(seq_len: int, streaming: bool, sink: int, local: int, pages=None) -> np.ndarray:
    """Ascending token positions one (sequence, KV head) attends to."""
    L = int(seq_len)
    if streaming:
        t = np.arange(L)
        return t[(t < sink) | (t >= L - local)]
    pages = np.asarray(pages, dtype=np.int64)
    if len(pages) == 0:
        return np.zeros(0, np.int64)
    t = (pages[:, None] * PAGE + np.arange(PAGE)[None, :]).reshape(-1)
    return t[t < L]


def gather_tokens(pages_pool, page_table, b, kvh, tokens):
    """float64[len(tokens), d]: rows of a paged pool for sequence b, KV head kvh."""
    pool = np.asarray(pages_pool)
    pt = np.asarray(page_table)
    tokens = np.asarray(tokens, dtype=np.int64)
    phys = pt[b, tokens // PAGE]
    return np.asarray(pool[phys, kvh, tokens % PAGE, :], dtype=np.float64)


def attend(qv, K, V, scale):
    """Softmax attention of one query over the rows of K, V (float64)."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1]), -np.inf
    logits = scale * (K @ qv)
    m = logits.max()
    w = np.exp(logits - m)
    l = w.sum()
    return (w @ V) / l, m + np.log(l)


def decode_attention(q, k_pages, v_pages, page_table, seq_lens, head_kind, sel, sink, local, scale=None):
    """out float64[B, Hq, d], lse float64[B, Hq] for given per-(b, kvh) page selections."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = len(head_kind)
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None or scale <= 0 else float(scale)
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        L = int(seq_lens[b])
        for kvh in range(Hkv):
            streaming = bool(head_kind[kvh])
            toks = token_set(L, streaming, sink, local, None if streaming else sel[(b, kvh)])
            K = gather_tokens(k_pages, page_table, b, kvh, toks)
            V = gather_tokens(v_pages, page_table, b, kvh, toks)
            for h in range(kvh * G, (kvh + 1) * G):
                out[b, h], lse[b, h] = attend(q[b, h], K, V, scale)
    return out, lse


def sparse_decode(q, k_pages, v_pages, page_table, seq_lens, stats, head_kind,
                  token_budget, sink, local, scale=None):
    """The whole decode step: select pages, then attend.  Returns
    (out, lse, sel, margin, scores)."""
    sel, margin, scores = select(q, stats, page_table, seq_lens, head_kind, token_budget, sink, local)
    out, lse = decode_attention(q, k_pages, v_pages, page_table, seq_lens, head_kind, sel,
                                sink, local, scale)
    return out, lse, sel, margin, scores


def reuse_decode(q, k_pages, v_pages, page_table, seq_lens, head_kind, kept_sel, sink, local, scale=None):
    """A decode step that keeps the page selection of an earlier step.

    LServe + SampleAttention blog post, "LServe - Decode Phase": selection
    results are reused across a small window of decode steps.  Reading where
    the page is silent: a dense KV head attends to every token t < seq_len of
    the kept pages (tokens appended since the selection count where they fall
    in a kept page, not elsewhere); a streaming KV head takes its sink and local
    window from the current seq_len.  This is decode_attention with the kept
    selection.  Returns (out, lse)."""
    return decode_attention(q, k_pages, v_pages, page_table, seq_lens, head_kind, kept_sel, sink, local, scale)
