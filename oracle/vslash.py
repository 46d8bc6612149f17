"""Vertical-slash block-mask construction for dense heads from sampled queries.

Test infrastructure only (see the package docstring).

Source: LServe + SampleAttention blog post, "SampleAttention - Column Pattern"
and "Slash Pattern" (Fig. 3): a few key positions draw attention from almost
every query (columns), and attention concentrates at fixed relative offsets
(slashes, diagonals); "CRA - The Accuracy Proxy" (Fig. 4): a mask is judged by
the minimum, over queries, of the share of the causal softmax mass it keeps,
and SampleAttention keeps adding column and slash candidates until that share
reaches a threshold tau.  The post leaves the estimator and its sampling
schedule to the paper; the reading built here, at the 64 x 64 tile grain of
the prefill:

* sampled queries: the last row (64 qt + 63) of query tiles qt = nQT - 1,
  nQT - 1 - stride, nQT - 1 - 2 stride, ... (>= 0), for each of the G query
  heads of the KV head;
* tile masses: r[s, h, kt] = sum of row s's causal softmax weights (query head
  h) over the keys of tile kt (kt <= qt(s));
* candidates: column kt (tiles (qt, kt), qt >= kt) scores sum_{s,h} r[s, h, kt];
  slash delta (tiles (qt, qt - delta)) scores sum_{s,h} r[s, h, qt(s) - delta];
* order: the diagonal slash (delta = 0) first, always (every row keeps the tile
  of its own query); then by score, descending; equal scores: columns before
  slashes, then the lower index;
* greedy: take candidates in that order; after each, the sampled CRA is the
  minimum over (s, h) of the retained mass sum of r over the row's covered
  tiles; stop as soon as it is >= tau (or when none is left);
* output: block_mask[qt, kt] = 1 for every tile kt <= qt covered by a taken
  column or slash, 0 elsewhere (above the diagonal too).

Streaming heads get an all-zero mask (they use the Lambda support instead).
"""
from __future__ import annotations

import numpy as np

TILE = 64


def sampled_tiles(nQT: int, stride: int) -> np.ndarray:
    """Query tiles whose last row is sampled: nQT-1, nQT-1-stride, ... >= 0 (ascending)."""
    if stride < 1:
        raise ValueError("stride must be >= 1")
    return np.arange(nQT - 1, -1, -stride)[::-1].copy()


def tile_masses(q, k, stride: int, scale=None, b: int = 0, g: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """(tiles, r): r float64[n_rows, G, nKT] of one (sequence b, KV head g); row s is the
    last row of query tile tiles[s]; r[s, h, kt] = 0 for kt > tiles[s]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    S, Hq, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    nQT = S // TILE
    scale = 1.0 / np.sqrt(d) if scale is None or scale <= 0 else float(scale)
    tiles = sampled_tiles(nQT, stride)
    r = np.zeros((len(tiles), G, nQT))
    for s, qt in enumerate(tiles):
        i = TILE * qt + TILE - 1
        K = k[b, : i + 1, g, :]
        for h in range(G):
            logits = scale * (K @ q[b, i, g * G + h, :])
            w = np.exp(logits - logits.max())
            w /= w.sum()
            r[s, h, : qt + 1] = np.add.reduceat(w, np.arange(0, i + 1, TILE))
    return tiles, r


def candidate_order(tiles: np.ndarray, r: np.ndarray) -> list[tuple[str, int, float]]:
    """[(kind, index, score)] in the order the greedy takes them: ('slash', 0) first,
    then by score descending, columns before slashes on equal scores, lower index first."""
    nKT = r.shape[2]
    col = r.sum(axis=(0, 1))
    sla = np.zeros(nKT)
    for s, qt in enumerate(tiles):
        for delta in range(qt + 1):
            sla[delta] += r[s, :, qt - delta].sum()
    rest = [("column", kt, col[kt]) for kt in range(nKT)] + \
           [("slash", dl, sla[dl]) for dl in range(1, nKT)]
    rest.sort(key=lambda c: (-c[2], 0 if c[0] == "column" else 1, c[1]))
    return [("slash", 0, sla[0])] + rest


def covered(kind: str, idx: int, qt: int, kt: int) -> bool:
    return kt <= qt and ((kind == "column" and kt == idx) or (kind == "slash" and qt - kt == idx))


def greedy(tiles: np.ndarray, r: np.ndarray, tau: float):
    """(taken candidates, sampled CRA after each) of the greedy rule above."""
    order = candidate_order(tiles, r)
    n_rows, G, nKT = r.shape
    cov = np.zeros((n_rows, nKT), bool)
    taken, cras = [], []
    for kind, idx, _ in order:
        for s, qt in enumerate(tiles):
            for kt in range(qt + 1):
                if covered(kind, idx, qt, kt):
                    cov[s, kt] = True
        taken.append((kind, idx))
        retained = (r * cov[:, None, :]).sum(axis=2)
        cras.append(retained.min())
        if cras[-1] >= tau:
            break
    return taken, cras


def mask_from(taken, nQT: int) -> np.ndarray:
    m = np.zeros((nQT, nQT), np.uint8)
    for qt in range(nQT):
        for kt in range(qt + 1):
            if any(covered(kind, idx, qt, kt) for kind, idx in taken):
                m[qt, kt] = 1
    return m


def build_vslash_mask(q, k, head_kind, stride: int, tau: float, scale=None):
    """(block_mask uint8[B, Hkv, nQT, nQT], cra float64[B, Hkv], n_columns, n_slashes int[B, Hkv])."""
    q = np.asarray(q, dtype=np.float64)
    B, S = q.shape[0], q.shape[1]
    Hkv = k.shape[2]
    nQT = S // TILE
    mask = np.zeros((B, Hkv, nQT, nQT), np.uint8)
    cra = np.zeros((B, Hkv))
    ncol = np.zeros((B, Hkv), np.int64)
    nsla = np.zeros((B, Hkv), np.int64)
    for b in range(B):
        for g in range(Hkv):
            if head_kind[g]:
                continue
            tiles, r = tile_masses(q, k, stride, scale, b, g)
            taken, cras = greedy(tiles, r, tau)
            mask[b, g] = mask_from(taken, nQT)
            cra[b, g] = cras[-1]
            ncol[b, g] = sum(1 for kind, _ in taken if kind == "column")
            nsla[b, g] = sum(1 for kind, _ in taken if kind == "slash")
    return mask, cra, ncol, nsla
