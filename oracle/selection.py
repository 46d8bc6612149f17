"""Query-aware hierarchical KV page selection -- the decode selector.

Test infrastructure only (see the package docstring).

Sources: LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2
(every page is scored cheaply from a summary vector kept per page, the top-k
pages are kept); mlsanity LServe page, Abstract (a hierarchical page selection
policy driven by query-centric similarity; a constant number of KV pages,
independent of context length).  The summary and the score are those of Quest
(listed under "Builds on" on the mlsanity LServe page): per channel the minimum
and maximum key over a page, and the upper bound

    s(page) = sum_c max(q_c * kmax_c, q_c * kmin_c)  >=  q . k_j   for every j in the page.

Hierarchy (plainest reading of "hierarchical"): summaries are kept per logical
page of 16 tokens; a physical page of 64 tokens holds 4 logical pages and takes
the max of their scores.  With grouped-query attention the score of a KV head is
the max over the bounds of its G query heads (one selection per KV head).

Layouts (token t of sequence b lives in physical page page_table[b, t // 64],
row t % 64):

    k_pages   [NP, Hkv, 64, d]
    stats     [NP, Hkv, 4, 2, d]   (index 0 = min, 1 = max)
    scores    [B, Hkv, maxP]
"""
from __future__ import annotations

import numpy as np

PAGE = 64
LOGICAL = 16
NL = PAGE // LOGICAL


def n_pages(seq_len: int) -> int:
    return (int(seq_len) + PAGE - 1) // PAGE


def page_stats(k_pages, page_table, seq_lens, head_kind, first_logical_page=0, stats=None):
    """Per (physical page, dense KV head, logical page): channelwise min and max
    of the keys of that logical page's valid tokens (t < seq_len).

    A logical page with no valid token gets min = +inf and max = -inf (the
    identities of min and max); such pages are never scored.  Logical pages
    below ``first_logical_page`` (an index within each sequence) are left as
    they are in ``stats`` (incremental update after appending tokens).
    Streaming heads get no summary (their entries are left untouched).

    Returns float64[NP, Hkv, 4, 2, d] (NaN where nothing was written unless a
    ``stats`` array to update is passed in).
    """
    k_pages = np.asarray(k_pages, dtype=np.float64)
    NP, Hkv, P, d = k_pages.shape
    out = np.full((NP, Hkv, NL, 2, d), np.nan) if stats is None else np.array(stats, dtype=np.float64)
    for b in range(len(seq_lens)):
        L = int(seq_lens[b])
        for i in range(n_pages(L)):
            pp = int(page_table[b][i])
            for h in range(Hkv):
                if head_kind[h]:
                    continue
                for l in range(NL):
                    lp = i * NL + l
                    if lp < first_logical_page:
                        continue
                    t0 = i * PAGE + l * LOGICAL
                    n_valid = max(0, min(LOGICAL, L - t0))
                    if n_valid == 0:
                        out[pp, h, l, 0, :] = np.inf
                        out[pp, h, l, 1, :] = -np.inf
                        continue
                    rows = k_pages[pp, h, l * LOGICAL: l * LOGICAL + n_valid, :]
                    out[pp, h, l, 0, :] = rows.min(axis=0)
                    out[pp, h, l, 1, :] = rows.max(axis=0)
    return out


def logical_bounds(q, stats, page_table, seq_len, b, h, G):
    """float64[n_pages, 4]: the bound of query head ``h`` (batch ``b``) for each
    logical page of the sequence; -inf for logical pages with no valid token.

    s(l) = sum_c max(q_c * kmax_c, q_c * kmin_c), summed in float64 (each term
    is the exact product of two bf16 numbers).
    """
    q = np.asarray(q, dtype=np.float64)
    kvh = h // G
    n = n_pages(seq_len)
    out = np.full((n, NL), -np.inf)
    qv = q[b, h, :]
    for i in range(n):
        pp = int(page_table[b][i])
        for l in range(NL):
            if i * PAGE + l * LOGICAL >= seq_len:
                continue
            kmin = np.asarray(stats[pp, kvh, l, 0, :], dtype=np.float64)
            kmax = np.asarray(stats[pp, kvh, l, 1, :], dtype=np.float64)
            out[i, l] = np.maximum(qv * kmax, qv * kmin).sum()
    return out


def page_scores(q, stats, page_table, seq_lens, head_kind, maxP=None):
    """float64[B, Hkv, maxP]: physical-page score of every dense KV head.

    Group score of a logical page = max over the G query heads of the KV head;
    physical score = max over its logical pages that hold a valid token.  Pages
    at or past n_pages(seq_len), and streaming heads, are -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = len(head_kind)
    G = Hq // Hkv
    maxP = np.asarray(page_table).shape[1] if maxP is None else maxP
    out = np.full((B, Hkv, maxP), -np.inf)
    for b in range(B):
        L = int(seq_lens[b])
        n = n_pages(L)
        for kvh in range(Hkv):
            if head_kind[kvh]:
                continue
            per_head = np.stack([logical_bounds(q, stats, page_table, L, b, h, G)
                                 for h in range(kvh * G, (kvh + 1) * G)])  # [G, n, NL]
            group = per_head.max(axis=0)          # [n, NL]
            out[b, kvh, :n] = group.max(axis=1)   # [n]
    return out


def budget_pages(token_budget: int, seq_len: int) -> int:
    """k = min(floor(budget / 64), n_pages): the constant page count of the Abstract."""
    return min(int(token_budget) // PAGE, n_pages(seq_len))


def topk_pages(scores_row, k):
    """Indices of the k largest scores, ties to the lower page index, sorted ascending.

    Also returns the tie margin |s_(k) - s_(k+1)| / max(|s_(k)|, tiny) of the
    sorted scores (inf when fewer than k+1 pages exist).
    """
    s = np.asarray(scores_row, dtype=np.float64)
    n = len(s)
    order = np.lexsort((np.arange(n), -s))   # primary -score, secondary index
    chosen = np.sort(order[:k])
    if k < n and k > 0:
        a, c = s[order[k - 1]], s[order[k]]
        margin = abs(a - c) / max(abs(a), np.finfo(np.float64).tiny)
    else:
        margin = np.inf
    return chosen, margin


def streaming_pages(seq_len: int, sink: int, local: int):
    """Pages holding a token of [0, sink) or [seq_len - local, seq_len), ascending."""
    L = int(seq_len)
    toks = set(range(0, min(sink, L))) | set(range(max(0, L - local), L))
    return np.array(sorted({t // PAGE for t in toks}), dtype=np.int64)


def select(q, stats, page_table, seq_lens, head_kind, token_budget, sink, local):
    """Full selector: per (b, kvh) the ascending list of selected page indices
    (indices within the sequence, not physical ids) and the tie margin.

    Dense KV heads: top-k by physical-page score; streaming KV heads: the fixed
    sink + local pages.  Returns (sel: dict[(b,kvh)] -> array, margin: dict).
    """
    scores = page_scores(q, stats, page_table, seq_lens, head_kind)
    sel, margin = {}, {}
    for b in range(len(seq_lens)):
        L = int(seq_lens[b])
        for kvh in range(len(head_kind)):
            if head_kind[kvh]:
                sel[(b, kvh)] = streaming_pages(L, sink, local)
                margin[(b, kvh)] = np.inf
            else:
                k = budget_pages(token_budget, L)
                sel[(b, kvh)], margin[(b, kvh)] = topk_pages(scores[b, kvh, :n_pages(L)], k)
    return sel, margin, scores
