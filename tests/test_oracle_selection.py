"""Pins for the oracle's page summaries, bound scores, hierarchical max and top-k.

* stats: closed form on the contiguous key tensor (NumPy min/max over 16-token
  groups, reached through the page table in the other direction);
* bound: the invariant s >= q . k_j for every token of the logical page (exact
  in float64), equality on single-token pages, the hand example;
* hierarchy: brute force by Python loops over channels, logical pages, heads;
* top-k: brute force by Python's ``sorted`` with an explicit key, count
  invariant, budget >= context selects every page.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import workloads as W
from oracle import selection as Sel

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


def small_cache(seed, B=2, ctx=300, Hkv=2, d=16, NP=None, lens=None):
    rng = np.random.default_rng(seed)
    n_pages = (ctx + 63) // 64
    NP = NP or B * n_pages + 3
    perm = rng.permutation(NP)[: B * n_pages].reshape(B, n_pages).astype(np.int32)
    k = rng.standard_normal((B, ctx, Hkv, d)).astype(np.float32)
    k = torch.from_numpy(k).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((B, ctx, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    pc = W.scatter_to_pages(k, v, torch.from_numpy(perm), NP)
    lens = [ctx] * B if lens is None else lens
    return k.double().numpy(), v.double().numpy(), pc.k_pages.double().numpy(), \
        pc.v_pages.double().numpy(), perm, np.array(lens, np.int32)


def test_stats_closed_form_on_contiguous_keys():
    ctx = 300                                      # ragged: last page has 44 tokens
    k, _, kp, _, pt, lens = small_cache(1, ctx=ctx)
    kind = np.array([0, 1], np.uint8)
    st = Sel.page_stats(kp, pt, lens, kind)
    B, _, Hkv, d = k.shape
    for b in range(B):
        n_full = ctx // 16
        kb = k[b, : n_full * 16, 0, :].reshape(n_full, 16, d)
        mins, maxs = kb.min(axis=1), kb.max(axis=1)
        tail = k[b, n_full * 16:, 0, :]
        for lp in range((ctx + 15) // 16):
            page, l = divmod(lp, 4)
            got_min = st[pt[b, page], 0, l, 0]
            got_max = st[pt[b, page], 0, l, 1]
            if lp < n_full:
                np.testing.assert_array_equal(got_min, mins[lp])
                np.testing.assert_array_equal(got_max, maxs[lp])
            else:
                np.testing.assert_array_equal(got_min, tail.min(axis=0))
                np.testing.assert_array_equal(got_max, tail.max(axis=0))
        # logical pages past the end of the sequence: empty (+inf, -inf)
        last_page = (ctx - 1) // 64
        for l in range(4):
            if last_page * 64 + 16 * l >= ctx:
                assert np.all(st[pt[b, last_page], 0, l, 0] == np.inf)
                assert np.all(st[pt[b, last_page], 0, l, 1] == -np.inf)
        # streaming head 1 gets no summary
        assert np.all(np.isnan(st[pt[b], 1]))


def test_stats_incremental_update_matches_full_rebuild():
    k, _, kp, _, pt, lens = small_cache(2, ctx=260)
    kind = np.array([0, 0], np.uint8)
    full = Sel.page_stats(kp, pt, lens, kind)
    stale = full.copy()
    stale[pt[:, 3:]] = 0.0                   # pretend pages >= 3 are stale
    upd = Sel.page_stats(kp, pt, lens, kind, first_logical_page=12, stats=stale)
    np.testing.assert_array_equal(np.nan_to_num(upd, nan=7.0), np.nan_to_num(full, nan=7.0))


def test_bound_hand_example():
    g = GOLD["bound"]
    keys = np.array(g["keys"])
    np.testing.assert_array_equal(keys.min(axis=0), g["kmin"])
    np.testing.assert_array_equal(keys.max(axis=0), g["kmax"])
    st = np.zeros((1, 1, 4, 2, 3))
    st[0, 0, 0, 0], st[0, 0, 0, 1] = g["kmin"], g["kmax"]
    q = np.array(g["q"])[None, None, :]
    s = Sel.logical_bounds(q, st, np.array([[0]]), 16, 0, 0, 1)
    assert s[0, 0] == g["score"]
    assert np.all(np.isneginf(s[0, 1:]))


@pytest.mark.parametrize("G", [1, 4])
def test_bound_dominates_every_dot_product(G):
    ctx, Hkv, d = 256 + 37, 2, 16
    k, _, kp, _, pt, lens = small_cache(3, B=1, ctx=ctx, Hkv=Hkv, d=d)
    kind = np.zeros(Hkv, np.uint8)
    st = Sel.page_stats(kp, pt, lens, kind)
    rng = np.random.default_rng(4)
    q = torch.from_numpy(rng.standard_normal((1, Hkv * G, d)).astype(np.float32)).to(torch.bfloat16).double().numpy()
    for h in range(Hkv * G):
        s = Sel.logical_bounds(q, st, pt, ctx, 0, h, G)
        for t in range(ctx):
            dot = float(np.dot(q[0, h], k[0, t, h // G]))
            assert s[t // 64, (t % 64) // 16] >= dot
    scores = Sel.page_scores(q, st, pt, lens, kind)
    for kvh in range(Hkv):
        for t in range(ctx):
            for h in range(kvh * G, (kvh + 1) * G):
                assert scores[0, kvh, t // 64] >= float(np.dot(q[0, h], k[0, t, kvh]))


def test_bound_single_token_page_is_exact():
    """A logical page holding one token: kmin = kmax = k, so the bound is q . k."""
    ctx = 64 * 2 + 16 + 1               # logical page 9 holds exactly token 144
    k, _, kp, _, pt, lens = small_cache(5, B=1, ctx=ctx, Hkv=1, d=16)
    st = Sel.page_stats(kp, pt, lens, np.zeros(1, np.uint8))
    q = np.random.default_rng(1).standard_normal((1, 1, 16))
    s = Sel.logical_bounds(q, st, pt, ctx, 0, 0, 1)
    assert s[2, 1] == float(np.dot(q[0, 0], k[0, 144, 0]))
    assert np.all(np.isneginf(s[2, 2:]))


def test_hierarchical_max_brute_force():
    ctx, Hkv, G, d = 200, 2, 2, 8
    _, _, kp, _, pt, lens = small_cache(6, B=2, ctx=ctx, Hkv=Hkv, d=d, lens=[200, 130])
    kind = np.array([0, 1], np.uint8)
    st = Sel.page_stats(kp, pt, lens, kind)
    q = np.random.default_rng(2).standard_normal((2, Hkv * G, d))
    scores = Sel.page_scores(q, st, pt, lens, kind)
    for b in range(2):
        L = int(lens[b])
        for i in range(pt.shape[1]):
            best = -math.inf
            for l in range(4):
                if i * 64 + l * 16 >= L:
                    continue
                for h in range(G):
                    tot = math.fsum(max(q[b, h, c] * st[pt[b, i], 0, l, 1, c],
                                        q[b, h, c] * st[pt[b, i], 0, l, 0, c]) for c in range(d))
                    best = max(best, tot)
            assert scores[b, 0, i] == pytest.approx(best, abs=1e-12) if best > -math.inf else scores[b, 0, i] == -math.inf
        assert np.all(np.isneginf(scores[b, 1]))


def brute_topk(s, k):
    order = sorted(range(len(s)), key=lambda i: (-s[i], i))
    return sorted(order[:k])


@pytest.mark.parametrize("seed", range(5))
def test_topk_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(0, 6, size=57).astype(np.float64)   # many exact ties
    for k in (0, 1, 5, 17, 56, 57):
        got, margin = Sel.topk_pages(s, k)
        assert list(got) == brute_topk(list(s), k)
        if 0 < k < 57:
            srt = sorted(s, reverse=True)
            assert margin == abs(srt[k - 1] - srt[k]) / max(abs(srt[k - 1]), np.finfo(float).tiny)


def test_budget_counts_and_full_budget():
    for L in (1, 63, 64, 65, 1000, 4096, 262144):
        n = (L + 63) // 64
        assert Sel.budget_pages(4096, L) == min(64, n)
        assert Sel.budget_pages(10**9, L) == n
    g = GOLD["tiny_workload_counts"]
    assert Sel.budget_pages(256, 1024) == g["decode_pages"]
    s = np.random.default_rng(0).standard_normal(40)
    got, _ = Sel.topk_pages(s, 40)
    assert list(got) == list(range(40))


@pytest.mark.parametrize("L,sink,local", [(1024, 64, 256), (1000, 64, 256), (100, 64, 256),
                                          (5000, 0, 1), (5000, 1, 0), (130, 65, 1)])
def test_streaming_pages_closed_form(L, sink, local):
    first = list(range((min(sink, L) + 63) // 64))
    last = list(range(max(0, L - local) // 64, (L - 1) // 64 + 1)) if local > 0 else []
    assert list(Sel.streaming_pages(L, sink, local)) == sorted(set(first) | set(last))
