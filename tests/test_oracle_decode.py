"""Pins for the oracle's decode attention and the CRA report.

* budget >= context selects every page, and the result equals dense decode
  computed by torch SDPA on the contiguous K/V;
* cross-mode: decoding the last prefill query against the prefill's own K/V
  equals the last prefill row (dense head: full budget; streaming head: the same
  sink/local);
* an explicit selection equals SDPA with the corresponding token mask;
* CRA equals 1 when nothing is dropped and matches brute-force weight sums;
* the paged gather against a per-token walk of the page table.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as A
from oracle import cra as C
from oracle import decode as D
from oracle import selection as Sel


def make(seed, B=2, ctx=333, Hq=4, Hkv=2, d=16, lens=None):
    rng = np.random.default_rng(seed)
    k = torch.from_numpy(rng.standard_normal((B, ctx, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((B, ctx, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    q = torch.from_numpy(rng.standard_normal((B, Hq, d)).astype(np.float32)).to(torch.bfloat16)
    n = (ctx + 63) // 64
    NP = B * n + 2
    pt = torch.from_numpy(rng.permutation(NP)[: B * n].reshape(B, n).astype(np.int32))
    pc = W.scatter_to_pages(k, v, pt, NP)
    lens = np.array([ctx] * B if lens is None else lens, np.int32)
    return (q.double().numpy(), k.double().numpy(), v.double().numpy(),
            pc.k_pages.double().numpy(), pc.v_pages.double().numpy(), pt.numpy(), lens)


def sdpa_one(qv, K, V, mask=None):
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qv)[None, None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        attn_mask=None if mask is None else torch.from_numpy(mask)[None])
    return o[0, 0].numpy()


@pytest.mark.parametrize("lens", [None, [333, 65]])
def test_full_budget_equals_dense_decode(lens):
    q, k, v, kp, vp, pt, L = make(1, lens=lens)
    kind = np.zeros(2, np.uint8)
    st = Sel.page_stats(kp, pt, L, kind)
    out, lse, sel, _, _ = D.sparse_decode(q, kp, vp, pt, L, st, kind, 10**6, 64, 256)
    for b in range(2):
        for h in range(4):
            kvh = h // 2
            ref = sdpa_one(q[b, h], k[b, : L[b], kvh], v[b, : L[b], kvh])
            np.testing.assert_allclose(out[b, h], ref, atol=1e-12)
        assert list(sel[(b, 0)]) == list(range((L[b] + 63) // 64))


def test_cross_mode_last_prefill_row():
    B, S, Hq, Hkv, d = 1, 320, 4, 2, 16
    rng = np.random.default_rng(3)
    qf = torch.from_numpy(rng.standard_normal((B, S, Hq, d)).astype(np.float32)).to(torch.bfloat16)
    k = torch.from_numpy(rng.standard_normal((B, S, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((B, S, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    kind = np.array([0, 1], np.uint8)
    sink, local = 64, 100
    pre, _ = A.masked_attention(qf.double().numpy(), k.double().numpy(), v.double().numpy(), kind, sink, local)
    pt = torch.arange(5, dtype=torch.int32)[None].flip(1)
    pc = W.scatter_to_pages(k, v, pt, 5)
    kp, vp = pc.k_pages.double().numpy(), pc.v_pages.double().numpy()
    L = np.array([S], np.int32)
    st = Sel.page_stats(kp, pt.numpy(), L, kind)
    qd = qf[:, S - 1].double().numpy()
    out, _, _, _, _ = D.sparse_decode(qd, kp, vp, pt.numpy(), L, st, kind, 10**6, sink, local)
    np.testing.assert_allclose(out[0], pre[0, S - 1], atol=1e-12)


def test_selection_equals_sdpa_with_token_mask():
    q, k, v, kp, vp, pt, L = make(7, B=1, ctx=500)
    kind = np.array([0, 1], np.uint8)
    st = Sel.page_stats(kp, pt, L, kind)
    out, _, sel, _, _ = D.sparse_decode(q, kp, vp, pt, L, st, kind, 192, 16, 40)
    assert len(sel[(0, 0)]) == 3
    t = np.arange(500)
    m_dense = np.isin(t // 64, sel[(0, 0)])
    m_stream = (t < 16) | (t >= 500 - 40)
    for h in range(4):
        m = m_dense if h < 2 else m_stream
        ref = sdpa_one(q[0, h], k[0, :, h // 2], v[0, :, h // 2], mask=m[None])
        np.testing.assert_allclose(out[0, h], ref, atol=1e-12)


def test_poisoned_pool_outside_selection_is_not_read():
    """NaN in every pool row outside the attended token set leaves the result finite."""
    q, k, v, kp, vp, pt, L = make(8, B=1, ctx=400)
    kind = np.array([0, 1], np.uint8)
    st = Sel.page_stats(kp, pt, L, kind)
    out, _, sel, _, _ = D.sparse_decode(q, kp, vp, pt, L, st, kind, 128, 8, 30)
    kp2, vp2 = kp.copy(), vp.copy()
    for i in range(pt.shape[1]):
        for kvh in range(2):
            toks = D.token_set(400, bool(kind[kvh]), 8, 30, sel[(0, kvh)] if kvh == 0 else None)
            keep = set(int(x) for x in toks if x // 64 == i)
            for r in range(64):
                if i * 64 + r not in keep:
                    kp2[pt[0, i], kvh, r] = np.nan
                    vp2[pt[0, i], kvh, r] = np.nan
    out2, _ = D.decode_attention(q, kp2, vp2, pt, L, kind, sel, 8, 30)
    np.testing.assert_array_equal(out2, out)


def test_cra_is_one_without_dropping_and_matches_weight_sums():
    B, S, Hq, Hkv, d = 1, 192, 2, 2, 8
    rng = np.random.default_rng(1)
    q, k, v = (rng.standard_normal((B, S, h, d)) for h in (Hq, Hkv, Hkv))
    kind = np.array([0, 1], np.uint8)
    np.testing.assert_allclose(C.cra(q, k, v, kind, 0, S), 1.0, atol=1e-12)
    r = C.retained_mass(q, k, v, kind, 5, 30)
    full = A.attention_weights(q, k, np.zeros(2, np.uint8), 0, 0, h=1)
    keep = A.kept_mask(np.arange(S), S, True, 5, 30, None)
    np.testing.assert_allclose(r[0, 1], (full * keep).sum(axis=1), atol=1e-12)
    np.testing.assert_allclose(r[0, 0], 1.0, atol=1e-12)
    # CRA is the worst-kept row: the minimum of those brute-force sums
    np.testing.assert_allclose(C.cra(q, k, v, kind, 5, 30)[0, 1], (full * keep).sum(axis=1).min(), atol=1e-12)


def test_reuse_at_the_same_lengths_is_the_selection_step():
    """Keeping a selection at the step that made it reproduces that step."""
    q, k, v, kp, vp, pt, L = make(5, lens=[333, 200])
    kind = np.array([0, 1], np.uint8)
    st = Sel.page_stats(kp, pt, L, kind)
    out, lse, sel, _, _ = D.sparse_decode(q, kp, vp, pt, L, st, kind, 128, 64, 100)
    out2, lse2 = D.reuse_decode(q, kp, vp, pt, L, kind, sel, 64, 100)
    np.testing.assert_array_equal(out2, out)
    np.testing.assert_array_equal(lse2, lse)


def test_reuse_after_appending_tokens_matches_sdpa_with_the_kept_pages():
    """Tokens appended since the selection count where they fall in a kept page;
    a streaming head's window follows the current length (SDPA with the token
    mask written out from the reading)."""
    ctx = 333
    q, k, v, kp, vp, pt, _ = make(6, ctx=ctx)
    kind = np.array([0, 1], np.uint8)
    L0 = np.array([250, 130], np.int32)          # lengths at the selection step
    L1 = np.array([333, 200], np.int32)          # lengths now
    st = Sel.page_stats(kp, pt, L0, kind)
    _, _, sel, _, _ = D.sparse_decode(q, kp, vp, pt, L0, st, kind, 128, 64, 100)
    out, _ = D.reuse_decode(q, kp, vp, pt, L1, kind, sel, 64, 100)
    t = np.arange(ctx)
    for b in range(2):
        dense_mask = np.isin(t // 64, np.asarray(sel[(b, 0)])) & (t < L1[b])
        stream_mask = ((t < 64) | (t >= L1[b] - 100)) & (t < L1[b])
        for h in range(4):
            kvh = h // 2
            m = dense_mask if kvh == 0 else stream_mask
            ref = sdpa_one(q[b, h], k[b, m, kvh], v[b, m, kvh])
            np.testing.assert_allclose(out[b, h], ref, atol=1e-12)


def test_gather_tokens_against_a_per_token_walk_of_the_page_table():
    """Token t of sequence b lives at slot t mod PAGE of physical page page_table[b, t // PAGE]."""
    rng = np.random.default_rng(7)
    B, maxP, Hkv, d = 2, 5, 3, 4
    P = B * maxP
    pool = rng.standard_normal((P, Hkv, D.PAGE, d)).astype(np.float32)
    pt = rng.permutation(P).reshape(B, maxP)
    for b in range(B):
        for kvh in range(Hkv):
            toks = np.array([0, 1, D.PAGE - 1, D.PAGE, 2 * D.PAGE + 3, maxP * D.PAGE - 1])
            got = D.gather_tokens(pool, pt, b, kvh, toks)
            assert got.dtype == np.float64 and got.shape == (len(toks), d)
            for n, t in enumerate(toks):
                page, slot = divmod(int(t), D.PAGE)
                np.testing.assert_array_equal(got[n], pool[pt[b][page]][kvh][slot])
    assert D.gather_tokens(pool, pt, 0, 0, np.array([], dtype=np.int64)).shape == (0, d)
