"""Pins for the oracle's INT4 KV pages (a declared scheme: the pages name none).

* codes lie in [0, 15], the extremes of every group map to codes 0 and 15,
  and codes are monotone in the value within a group;
* dequantisation is within half a step (plus the float32 rounding of the fma)
  of the input;
* a group whose values are all equal dequantises exactly;
* the directed bf16 roundings of the summaries are checked by hand and
  against torch's bf16 conversion (bracketing, one step apart at most);
* the summaries of the dequantised keys bound every dequantised key;
* the test-side unpacker of the library's byte format (tests/int4_format.py,
  used by the GPU parity tests) hits the positions worked out by hand in
  tests/golden/int4_layout.json and is a bijection.
"""
import json
import os

import numpy as np
import pytest
import torch

import int4_format as F

import workloads as W
from oracle import quant as Q
from oracle import selection as Sel


def pool(seed=3, B=2, ctx=150, Hkv=2, d=64, lens=None):
    rng = np.random.default_rng(seed)
    k = torch.from_numpy(rng.standard_normal((B, ctx, Hkv, d)).astype(np.float32) * 3).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((B, ctx, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    n = (ctx + 63) // 64
    NP = B * n + 1
    pt = torch.from_numpy(rng.permutation(NP)[: B * n].reshape(B, n).astype(np.int32))
    pc = W.scatter_to_pages(k, v, pt, NP)
    lens = np.array([ctx] * B if lens is None else lens, np.int32)
    return pc.k_pages.float().numpy(), pc.v_pages.float().numpy(), pt.numpy(), lens


def test_storage_format_positions_match_the_hand_worked_page():
    """The test-side unpacker of the library's INT4 bytes (tests/int4_format.py)
    against positions worked out by hand from include/lserve.h's prose."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "int4_layout.json")))
    d = g["d"]
    kp = F.key_nibble_positions(d)
    for c, n in g["key_row"]["channel_to_nibble"].items():
        assert kp[int(c)] == n, c
    vp = F.value_nibble_positions(d)
    for u, c, n in g["value_page"]["token_channel_to_nibble"]:
        assert vp[u, c] == n, (u, c)
    kc = F.key_param_channels(d)
    for i, c in g["key_params"]["index_to_channel"].items():
        assert kc[int(i)] == c, i


def test_storage_format_is_a_bijection():
    """Every code of a key row / value page has its own nibble and every nibble
    holds one code; every channel's parameters sit at one index.  Unpacking
    bytes built nibble by nibble recovers the codes."""
    for d in (64, 128):
        kp = F.key_nibble_positions(d)
        assert sorted(kp.tolist()) == list(range(d))
        vp = F.value_nibble_positions(d)
        assert sorted(vp.ravel().tolist()) == list(range(64 * d))
        kc = F.key_param_channels(d)
        assert sorted(kc.tolist()) == list(range(d))
        rng = np.random.default_rng(d)
        codes = rng.integers(0, 16, size=(64, d)).astype(np.uint8)
        nib = np.zeros(64 * d, np.uint8)
        nib[vp.ravel()] = codes.ravel()
        packed = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
        np.testing.assert_array_equal(F.unpack_values(packed, d), codes)
        nib = np.zeros(d, np.uint8)
        nib[kp] = codes[0]
        np.testing.assert_array_equal(F.unpack_keys((nib[0::2] | (nib[1::2] << 4)).astype(np.uint8), d), codes[0])
        par = rng.standard_normal((2, d)).astype(np.float32)
        step, lo = F.unpack_key_params(par)
        np.testing.assert_array_equal(step[kc], par[0])
        np.testing.assert_array_equal(lo[kc], par[1])


def test_bf16_directed_rounding_by_hand():
    # bf16 keeps 8 significant bits: next to 1 the representable values are 1 +- k 2^-7
    x = np.array([1.0 + 2 ** -10, -1.0 - 2 ** -10, 1.5, -2.5, 2 ** -8 * 3.3, np.inf, -np.inf], np.float32)
    np.testing.assert_array_equal(Q.bf16_round_down(x),
                                  np.array([1.0, -1.0 - 2 ** -7, 1.5, -2.5, 2 ** -8 * 3.296875, np.inf, -np.inf],
                                           np.float32))
    np.testing.assert_array_equal(Q.bf16_round_up(x),
                                  np.array([1.0 + 2 ** -7, -1.0, 1.5, -2.5, 2 ** -8 * 3.3125, np.inf, -np.inf],
                                           np.float32))


def test_bf16_directed_rounding_brackets_and_is_tight():
    """Down <= x <= up, both bf16 (torch's own bf16 conversion leaves them
    unchanged), and they are equal or one bf16 step apart."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    dn, up = Q.bf16_round_down(x), Q.bf16_round_up(x)
    assert np.all(dn <= x) and np.all(x <= up)
    as_bf16 = lambda a: torch.from_numpy(a).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(as_bf16(dn), dn)
    np.testing.assert_array_equal(as_bf16(up), up)
    exact = dn == up
    np.testing.assert_array_equal(exact, as_bf16(x) == x)
    # no bf16 lies strictly between: same sign, so their top halves differ by one
    gap = np.abs(up.view(np.uint32).astype(np.int64) - dn.view(np.uint32).astype(np.int64))
    assert np.all(gap[~exact] == 0x10000)


def test_codes_range_extremes_monotone_and_error_bound():
    kp, vp, pt, L = pool(lens=[150, 97])
    qp = Q.quantize_pages(kp, vp, pt, L)
    kdeq, vdeq = qp.kdeq, qp.vdeq
    for b in range(2):
        for i in range(Sel.n_pages(L[b])):
            p, nv = pt[b, i], min(64, L[b] - 64 * i)
            for g in range(2):
                kc = qp.kcode[p, g, :nv]
                x = kp[p, g, :nv]
                assert kc.max() <= 15
                for c in range(x.shape[1]):           # keys: per channel
                    col = x[:, c]
                    if col.max() > col.min():
                        assert kc[col.argmin(), c] == 0 and kc[col.argmax(), c] == 15
                    order = np.argsort(col, kind="stable")
                    assert np.all(np.diff(kc[order, c].astype(int)) >= 0)
                step = qp.kstep[p, g]
                err = np.abs(kdeq[p, g, :nv] - x)
                # half a step, plus the float32 rounding of the fma
                rnd = np.maximum(np.abs(x), np.abs(kdeq[p, g, :nv])) * 2 ** -22
                assert np.all(err <= step[None, :] * 0.5 * (1 + 1e-5) + rnd + 1e-7)
                vc = qp.vcode[p, g, :nv]
                y = vp[p, g, :nv]
                for t in range(nv):                    # values: per token
                    if y[t].max() > y[t].min():
                        assert vc[t, y[t].argmin()] == 0 and vc[t, y[t].argmax()] == 15
                err = np.abs(vdeq[p, g, :nv] - y)
                rnd = np.maximum(np.abs(y), np.abs(vdeq[p, g, :nv])) * 2 ** -22
                assert np.all(err <= qp.vstep[p, g, :nv, None] * 0.5 * (1 + 1e-5) + rnd + 1e-7)


def test_constant_group_dequantises_exactly():
    kp, vp, pt, L = pool()
    kp[:] = 1.5
    vp[:] = -0.25
    qp = Q.quantize_pages(kp, vp, pt, L)
    kdeq, vdeq = qp.kdeq, qp.vdeq
    for b in range(2):
        for i in range(Sel.n_pages(L[b])):
            p, nv = pt[b, i], min(64, L[b] - 64 * i)
            assert np.all(kdeq[p, :, :nv] == 1.5) and np.all(vdeq[p, :, :nv] == -0.25)


def test_summaries_of_dequantised_keys_bound_them():
    kp, vp, pt, L = pool(lens=[150, 70])
    kind = np.array([0, 1], np.uint8)
    kdeq = Q.quantize_pages(kp, vp, pt, L).kdeq
    st = Q.quantized_stats(kdeq, pt, L, kind)
    for b in range(2):
        for t in range(L[b]):
            p, r = pt[b, t // 64], t % 64
            lp = r // 16
            assert np.all(st[p, 0, lp, 0] <= kdeq[p, 0, r]) and np.all(kdeq[p, 0, r] <= st[p, 0, lp, 1])
