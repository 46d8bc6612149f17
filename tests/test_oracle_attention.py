"""Pins for the oracle's masked attention (prefill) and kept-tile lists.

Each check ties ``oracle.attention`` to something other than itself:
pure-Python brute force on tiny inputs, PyTorch's scaled_dot_product_attention
(a library routine) on the special cases that reduce to it, hand-derived values
(tests/golden/hand_examples.json) and invariants (weights sum to 1, S = 1).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as A

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


def rand_qkv(B, S, Hq, Hkv, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, S, Hq, d))
    k = rng.standard_normal((B, S, Hkv, d))
    v = rng.standard_normal((B, S, Hkv, d))
    return q, k, v


def sdpa(q, k, v, mask=None, causal=False, scale=None):
    """Library reference: torch SDPA in float64 on [B,S,H,d] numpy arrays (GQA expanded)."""
    G = q.shape[2] // k.shape[2]
    Q = torch.from_numpy(q).permute(0, 2, 1, 3)
    K = torch.from_numpy(k).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    V = torch.from_numpy(v).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(
        Q, K, V, attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- brute force

def brute_kept(i, streaming, sink, local, tm):
    """K(i) restated as explicit index lists (no arrays, no shared helper)."""
    if streaming:
        return sorted(set(range(min(sink, i + 1))) | set(range(max(0, i - local + 1), i + 1)))
    if tm is None:
        return list(range(i + 1))
    return [j for j in range(i + 1) if tm[i // 64][j // 64]]


def brute_attention(q, k, v, head_kind, sink, local, bm, scale):
    B, S, Hq, d = q.shape
    G = Hq // k.shape[2]
    out = np.zeros_like(q)
    lse = np.full((B, Hq, S), -math.inf)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            st = bool(head_kind[kvh])
            tm = None if (bm is None or st) else bm[b][kvh]
            for i in range(S):
                js = brute_kept(i, st, sink, local, tm)
                if not js:
                    continue
                logits = [scale * math.fsum(q[b, i, h, c] * k[b, j, kvh, c] for c in range(d)) for j in js]
                m = max(logits)
                w = [math.exp(x - m) for x in logits]
                l = math.fsum(w)
                for c in range(d):
                    out[b, i, h, c] = math.fsum(wj * v[b, j, kvh, c] for wj, j in zip(w, js)) / l
                lse[b, h, i] = m + math.log(l)
    return out, lse


@pytest.mark.parametrize("sink,local", [(64, 32), (5, 40), (0, 7), (100, 1)])
def test_brute_force_tiny(sink, local):
    B, S, Hq, Hkv, d = 1, 192, 4, 2, 8
    q, k, v = rand_qkv(B, S, Hq, Hkv, d, 7)
    kind = np.array([0, 1], np.uint8)
    rng = np.random.default_rng(3)
    bm = (rng.random((B, Hkv, 3, 3)) < 0.6).astype(np.uint8)
    bm[0, 0, 1, 0] = 0          # drop a below-diagonal tile
    bm[0, 0, 2, 2] = 1
    scale = 1 / math.sqrt(d)
    o_ref, lse_ref = brute_attention(q, k, v, kind, sink, local, bm, scale)
    o, lse = A.masked_attention(q, k, v, kind, sink, local, bm)
    np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)


def test_empty_rows_are_zero():
    """A dense head whose block mask drops the diagonal tile has rows with no key."""
    B, S, Hq, Hkv, d = 1, 128, 2, 1, 4
    q, k, v = rand_qkv(B, S, Hq, Hkv, d, 1)
    bm = np.zeros((1, 1, 2, 2), np.uint8)
    bm[0, 0, 1, 0] = 1
    o, lse = A.masked_attention(q, k, v, np.array([0], np.uint8), 0, 0, bm)
    assert np.all(o[0, :64] == 0) and np.all(np.isneginf(lse[0, :, :64]))
    assert np.all(np.isfinite(lse[0, :, 64:]))


# ------------------------------------------------------- library special cases

@pytest.mark.parametrize("G", [1, 2, 4])
def test_all_tiles_kept_equals_dense_causal(G):
    B, S, Hkv, d = 2, 256, 2, 16
    q, k, v = rand_qkv(B, S, Hkv * G, Hkv, d, 11 + G)
    bm = np.ones((B, Hkv, S // 64, S // 64), np.uint8)
    o, _ = A.masked_attention(q, k, v, np.zeros(Hkv, np.uint8), 0, 0, bm)
    np.testing.assert_allclose(o, sdpa(q, k, v, causal=True), atol=1e-12)
    o2, _ = A.masked_attention(q, k, v, np.zeros(Hkv, np.uint8), 0, 0, None)
    np.testing.assert_allclose(o2, o, atol=0)


@pytest.mark.parametrize("sink,local", [(0, 256), (200, 56), (256, 0), (17, 300)])
def test_streaming_covering_sequence_equals_dense(sink, local):
    B, S, Hq, Hkv, d = 1, 256, 2, 1, 16
    q, k, v = rand_qkv(B, S, Hq, Hkv, d, 5)
    o, _ = A.masked_attention(q, k, v, np.array([1], np.uint8), sink, local)
    np.testing.assert_allclose(o, sdpa(q, k, v, causal=True), atol=1e-12)


def band_mask(S, sink, local):
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    return ((j <= i) & ((j < sink) | (j > i - local))).numpy()


@pytest.mark.parametrize("sink,local", [(0, 1), (0, 64), (0, 65), (3, 1), (64, 256), (70, 10)])
def test_streaming_equals_sdpa_with_lambda_mask(sink, local):
    """Sliding window of ``local`` tokens ending at the query, plus ``sink`` first tokens."""
    B, S, Hq, Hkv, d = 1, 320, 2, 1, 8
    q, k, v = rand_qkv(B, S, Hq, Hkv, d, 9)
    o, _ = A.masked_attention(q, k, v, np.array([1], np.uint8), sink, local)
    np.testing.assert_allclose(o, sdpa(q, k, v, mask=band_mask(S, sink, local)), atol=1e-12)


def test_block_mask_equals_sdpa_with_expanded_mask():
    B, S, Hq, Hkv, d = 1, 256, 4, 2, 8
    q, k, v = rand_qkv(B, S, Hq, Hkv, d, 21)
    rng = np.random.default_rng(2)
    bm = (rng.random((B, Hkv, 4, 4)) < 0.5).astype(np.uint8)
    for t in range(4):
        bm[0, :, t, t] = 1
    kind = np.zeros(Hkv, np.uint8)
    o, _ = A.masked_attention(q, k, v, kind, 0, 0, bm)
    for h in range(Hkv):
        full = np.kron(bm[0, h], np.ones((64, 64), np.uint8)).astype(bool) & np.tril(np.ones((S, S), bool))
        ref = sdpa(q[:, :, 2 * h:2 * h + 2], k[:, :, h:h + 1], v[:, :, h:h + 1], mask=full)
        np.testing.assert_allclose(o[:, :, 2 * h:2 * h + 2], ref, atol=1e-12)


def test_lse_equals_torch_logsumexp():
    B, S, Hq, Hkv, d = 1, 128, 2, 2, 8
    q, k, v = rand_qkv(B, S, Hq, Hkv, d, 4)
    kind = np.array([0, 1], np.uint8)
    _, lse = A.masked_attention(q, k, v, kind, 4, 20)
    for h, (mask) in enumerate([np.tril(np.ones((S, S), bool)), band_mask(S, 4, 20)]):
        logits = torch.from_numpy(q[0, :, h] @ k[0, :, h].T / math.sqrt(d))
        ref = torch.logsumexp(logits.masked_fill(~torch.from_numpy(mask), -math.inf), dim=1).numpy()
        np.testing.assert_allclose(lse[0, h], ref, atol=1e-12)


# ------------------------------------------------------------------ invariants

def test_weights_rows_sum_to_one():
    B, S, Hq, Hkv, d = 1, 256, 2, 2, 8
    q, k, v = rand_qkv(B, S, Hq, Hkv, d, 8)
    kind = np.array([0, 1], np.uint8)
    rng = np.random.default_rng(0)
    bm = (rng.random((1, 2, 4, 4)) < 0.5).astype(np.uint8)
    for t in range(4):
        bm[0, 0, t, t] = 1
    for h in range(2):
        w = A.attention_weights(q, k, kind, 32, 48, bm, h=h)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-12)
        assert np.all(np.triu(w, 1) == 0)


def test_single_token_equals_v0():
    q, k, v = rand_qkv(1, 1, 2, 1, 8, 3)
    for kind in (0, 1):
        o, lse = A.masked_attention(q, k, v, np.array([kind], np.uint8), 0, 1)
        np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], atol=1e-15)
        np.testing.assert_allclose(lse[0, :, 0], (q[0, 0] @ k[0, 0, 0]) / math.sqrt(8), atol=1e-14)


def test_row_sampling_is_exact():
    B, S, Hq, Hkv, d = 1, 256, 2, 1, 8
    q, k, v = rand_qkv(B, S, Hq, Hkv, d, 12)
    kind = np.array([1], np.uint8)
    o, lse = A.masked_attention(q, k, v, kind, 16, 40)
    rows = np.array([0, 5, 63, 64, 200, 255])
    o2, lse2 = A.masked_attention(q, k, v, kind, 16, 40, rows=rows, row_chunk=4)
    np.testing.assert_array_equal(o2, o[:, rows])
    np.testing.assert_array_equal(lse2, lse[:, :, rows])


def test_hand_example_lambda_row():
    g = GOLD["lambda_row"]
    q = np.array(g["q"])[None, :, None, :]
    k = np.array(g["k"])[None, :, None, :]
    v = np.array(g["v"])[None, :, None, :]
    o, lse = A.masked_attention(q, k, v, np.array([0], np.uint8), 0, 0, scale=1.0)
    np.testing.assert_allclose(o[0, 2, 0], g["dense_row2"], atol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 2], g["dense_row2_lse"], atol=1e-15)
    o, lse = A.masked_attention(q, k, v, np.array([1], np.uint8), 1, 1, scale=1.0)
    np.testing.assert_allclose(o[0, 2, 0], g["stream_sink1_local1_row2"], atol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 2], g["stream_sink1_local1_row2_lse"], atol=1e-15)


# ------------------------------------------------------------------ tile lists

@pytest.mark.parametrize("sink,local", [(64, 256), (1, 1), (65, 63), (0, 200), (130, 0), (0, 0)])
def test_tile_kept_matches_element_definition(sink, local):
    S = 640
    rng = np.random.default_rng(5)
    tm = (rng.random((10, 10)) < 0.4).astype(np.uint8)
    for streaming in (False, True):
        for mask in (None, tm):
            keep = A.kept_mask(np.arange(S), S, streaming, sink, local, None if streaming else mask)
            by_tile = keep.reshape(10, 64, 10, 64).any(axis=(1, 3))
            np.testing.assert_array_equal(A.tile_kept(S, streaming, sink, local, mask), by_tile)


def test_tile_counts_tiny_workload():
    g = GOLD["tiny_workload_counts"]
    assert A.tile_kept(1024, False, 64, 256).sum() == g["dense_tiles"]
    assert A.tile_kept(1024, True, 64, 256).sum() == g["streaming_tiles"]
    off, kt = A.tile_lists(1, 1024, np.array([0, 1], np.uint8), 64, 256)
    assert off[-1] == g["dense_tiles"] + g["streaming_tiles"]
    assert len(kt) == off[-1]
    # rows are ascending and causal
    for r in range(32):
        row = kt[off[r]:off[r + 1]]
        assert np.all(np.diff(row) > 0) and np.all(row <= r % 16)


def test_tile_counts_closed_form_dense():
    for n in (1, 2, 7, 33):
        assert A.tile_kept(64 * n, False, 0, 0).sum() == n * (n + 1) // 2


def test_q_at_rows_matches_full_q():
    q, k, v = rand_qkv(1, 192, 2, 1, 8, 31)
    kind = np.array([1], np.uint8)
    rows = np.array([3, 64, 191])
    o, lse = A.masked_attention(q, k, v, kind, 5, 20, rows=rows)
    o2, lse2 = A.masked_attention(q[:, rows], k, v, kind, 5, 20, rows=rows, q_at_rows=True, row_chunk=2)
    np.testing.assert_allclose(o, o2, atol=1e-14, rtol=0)
    np.testing.assert_allclose(lse, lse2, atol=1e-14, rtol=0)


# ---------------------------------------------------------------- tile-level Lambda

def brute_tile_lambda(S, sink, local):
    """Pure-Python: a tile is kept iff some causal pair inside it meets the token-level
    Lambda support; K(i) is then every causal key of the kept tiles of row i's tile."""
    n = S // 64
    kept = [[False] * n for _ in range(n)]
    for qt in range(n):
        for kt in range(qt + 1):
            kept[qt][kt] = any(j <= i and (j < sink or i - j < local)
                               for i in range(64 * qt, 64 * qt + 64) for j in range(64 * kt, 64 * kt + 64))
    m = np.zeros((S, S), bool)
    for i in range(S):
        for j in range(i + 1):
            m[i, j] = kept[i // 64][j // 64]
    return m


@pytest.mark.parametrize("sink,local", [(64, 256), (0, 1), (1, 0), (70, 130), (0, 65), (130, 0)])
def test_tile_level_lambda_brute_force(sink, local):
    S = 320
    got = A.kept_mask(np.arange(S), S, True, sink, local, None, lambda_tiles=True)
    np.testing.assert_array_equal(got, brute_tile_lambda(S, sink, local))
    # a superset of the token-level support, equal to it when every boundary is tile-aligned
    tok = A.kept_mask(np.arange(S), S, True, sink, local, None)
    assert np.all(got[tok])


def test_tile_level_lambda_hand_count():
    g = GOLD["tile_lambda_pairs"]
    m = A.kept_mask(np.arange(g["S"]), g["S"], True, g["sink"], g["local"], None, lambda_tiles=True)
    assert int(m.sum()) == g["kept_pairs"]


def test_tile_level_lambda_equals_sdpa_with_its_mask():
    q, k, v = rand_qkv(1, 256, 4, 2, 16, seed=31)
    kind, sink, local = [1, 0], 30, 70
    out, _ = A.masked_attention(q, k, v, kind, sink, local, lambda_tiles=True)
    m = brute_tile_lambda(256, sink, local)
    mask = np.where(m, 0.0, -np.inf)[None, None]
    ref_s = sdpa(q[:, :, :2], k[:, :, :1], v[:, :, :1], mask=mask)   # query heads 0, 1 read KV head 0 (streaming)
    np.testing.assert_allclose(out[:, :, :2], ref_s, atol=1e-12)
    ref_d = sdpa(q[:, :, 2:], k[:, :, 1:], v[:, :, 1:], causal=True)   # the dense head is unchanged
    np.testing.assert_allclose(out[:, :, 2:], ref_d, atol=1e-12)


def test_tile_level_lambda_covering_sequence_equals_dense():
    q, k, v = rand_qkv(1, 192, 2, 1, 8, seed=32)
    out, _ = A.masked_attention(q, k, v, [1], 192, 0, lambda_tiles=True)
    np.testing.assert_allclose(out, sdpa(q, k, v, causal=True), atol=1e-12)
