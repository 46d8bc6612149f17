"""Masked causal softmax attention -- the prefill half of the method.

Test infrastructure only (see the package docstring).

Definition (LServe + SampleAttention blog post, "LServe - Prefill Phase",
Fig. 1(a) and 1(b); mlsanity LServe page, Abstract):

    o_i = sum_{j in K(i)} softmax_j(scale * q_i . k_j) v_j,   scale = 1/sqrt(d)

with query head h reading KV head h // G (G = Hq / Hkv) and the kept set K(i):

* dense KV head:      K(i) = { j <= i : block_mask[i // 64, j // 64] != 0 }
                      (every j <= i when no block mask is given);
* streaming KV head:  K(i) = { j <= i : j < sink  or  i - j < local }
                      (the Lambda-shaped support: sink tokens plus a local window
                      that ends at, and includes, the query itself).

Readings where the pages are silent: the Lambda support is defined per token
(the kernel keeps every 64x64 tile that meets it and masks inside boundary
tiles); a block mask applies to dense heads only and is given per KV head; a
row with an empty kept set yields o_i = 0 and lse_i = -inf.

Tile-level Lambda (``lambda_tiles=True``): the same post's "no partial blocks"
(each KV block is fully computed or fully skipped, Fig. 1(a)/(b)) read for the
streaming heads too.  A streaming head then attends every causal key of every
64x64 tile that meets the Lambda support:

* streaming, tile level:  K(i) = { j <= i : 64 (j // 64) < sink  or
                                   max(64 (i // 64) - 64 (j // 64) - 63, 0) < local }

i.e. the tiles of ``tile_kept`` in full, with only the causal mask inside the
diagonal tile.  Dense heads are unchanged.
"""
from __future__ import annotations

import numpy as np

TILE = 64


def kept_mask(rows: np.ndarray, S: int, streaming: bool, sink: int, local: int,
              tile_mask: np.ndarray | None, lambda_tiles: bool = False) -> np.ndarray:
    """bool[len(rows), S]: element (r, j) is True iff key j is in K(rows[r]).

    ``tile_mask`` is this (batch, KV head)'s uint8[S/64, S/64] block mask or None;
    ``lambda_tiles`` selects the tile-level Lambda support of streaming heads.
    """
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(S, dtype=np.int64)[None, :]
    causal = j <= i
    if streaming and lambda_tiles:
        qt, kt = i // TILE, j // TILE
        return causal & ((TILE * kt < sink) | (np.maximum(TILE * qt - TILE * kt - (TILE - 1), 0) < local))
    if streaming:
        return causal & ((j < sink) | (i - j < local))
    if tile_mask is None:
        return causal
    return causal & (tile_mask[i // TILE, j // TILE] != 0)


def masked_attention(q, k, v, head_kind, sink, local, block_mask=None, scale=None,
                     rows=None, row_chunk=256, q_at_rows=False, lambda_tiles=False):
    """Exact masked attention in float64.

    q : [B, S, Hq, d]; k, v : [B, S, Hkv, d] (any float dtype, up-cast to f64)
    head_kind : [Hkv] (0 dense, 1 streaming)
    block_mask : [B, Hkv, S/64, S/64] or None
    rows : optional 1-D array of query positions to evaluate (all when None);
           rows are independent, so a sampled row is an exact row.
    q_at_rows : q is given only at ``rows`` ([B, R, Hq, d]) instead of [B, S, Hq, d].
    lambda_tiles : streaming heads use the tile-level Lambda support.

    Returns (out [B, R, Hq, d], lse [B, Hq, R]) with R = len(rows).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, _, Hq, d = q.shape
    S = k.shape[1]
    Hkv = k.shape[2]
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None or scale <= 0 else float(scale)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    R = len(rows)
    out = np.zeros((B, R, Hq, d))
    lse = np.full((B, Hq, R), -np.inf)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            streaming = bool(head_kind[kvh])
            tm = None if (block_mask is None or streaming) else np.asarray(block_mask[b, kvh])
            K = k[b, :, kvh, :]
            V = v[b, :, kvh, :]
            for c0 in range(0, R, row_chunk):
                r = rows[c0:c0 + row_chunk]
                keep = kept_mask(r, S, streaming, sink, local, tm, lambda_tiles)
                qr = q[b, c0:c0 + len(r), h, :] if q_at_rows else q[b, r, h, :]
                logits = scale * (qr @ K.T)
                logits = np.where(keep, logits, -np.inf)
                m = logits.max(axis=1, keepdims=True)
                has = np.isfinite(m[:, 0])
                m_safe = np.where(np.isfinite(m), m, 0.0)
                w = np.where(keep, np.exp(logits - m_safe), 0.0)
                l = w.sum(axis=1)
                o = (w @ V) / np.where(has, l, 1.0)[:, None]
                out[b, c0:c0 + len(r), h, :] = np.where(has[:, None], o, 0.0)
                lse[b, h, c0:c0 + len(r)] = np.where(has, m_safe[:, 0] + np.log(np.where(has, l, 1.0)), -np.inf)
    return out, lse


def attention_weights(q, k, head_kind, sink, local, block_mask=None, scale=None, b=0, h=0,
                      lambda_tiles=False):
    """float64[S, S] softmax weights of one (batch, query head); zero rows for empty K(i)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    S, d = q.shape[1], q.shape[3]
    G = q.shape[2] // k.shape[2]
    kvh = h // G
    streaming = bool(head_kind[kvh])
    scale = 1.0 / np.sqrt(d) if scale is None or scale <= 0 else float(scale)
    tm = None if (block_mask is None or streaming) else np.asarray(block_mask[b, kvh])
    keep = kept_mask(np.arange(S), S, streaming, sink, local, tm, lambda_tiles)
    logits = np.where(keep, scale * (q[b, :, h, :] @ k[b, :, kvh, :].T), -np.inf)
    m = logits.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    w = np.where(keep, np.exp(logits - m), 0.0)
    l = w.sum(axis=1, keepdims=True)
    return w / np.where(l > 0, l, 1.0)


def tile_kept(S: int, streaming: bool, sink: int, local: int, tile_mask=None) -> np.ndarray:
    """bool[S/64, S/64]: tile (qt, kt) is kept iff it holds at least one kept element.

    This is the whole-tile skipping rule of the blog's "LServe - Prefill Phase"
    (each KV block is fully computed or fully skipped, Fig. 1(a)) applied to the
    element set K(i) above.  Written per tile from the element definition:

    * dense:     some j <= i exists in the tile iff kt <= qt; the block mask then
                 keeps or drops the tile as a whole;
    * streaming: the tile's smallest key index is 64 kt (so it meets the sink
                 iff 64 kt < sink) and the smallest distance i - j over its
                 causal pairs is max(64 qt - 64 kt - 63, 0) (so it meets the
                 local window iff that distance is < local).
    """
    n = S // TILE
    qt = np.arange(n)[:, None]
    kt = np.arange(n)[None, :]
    causal = kt <= qt
    if streaming:
        mind = np.maximum(TILE * qt - TILE * kt - (TILE - 1), 0)
        return causal & ((TILE * kt < sink) | (mind < local))
    if tile_mask is None:
        return causal
    return causal & (np.asarray(tile_mask)[:n, :n] != 0)


def tile_lists(B: int, S: int, head_kind, sink: int, local: int, block_mask=None):
    """CSR of kept KV tiles per (b, kvh, qt), rows in that order, kt ascending.

    Returns (offsets int64[B*Hkv*nQT + 1], kt int64[nnz]).
    """
    Hkv = len(head_kind)
    n = S // TILE
    counts, cols = [], []
    for b in range(B):
        for h in range(Hkv):
            streaming = bool(head_kind[h])
            tm = None if (block_mask is None or streaming) else block_mask[b, h]
            kept = tile_kept(S, streaming, sink, local, tm)
            for qt in range(n):
                ks = np.nonzero(kept[qt])[0]
                counts.append(len(ks))
                cols.append(ks)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return offsets, (np.concatenate(cols).astype(np.int64) if cols else np.zeros(0, np.int64))
