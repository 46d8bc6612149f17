"""Pins for the oracle's INT4 KV pages (a declared scheme: the pages name none).

* codes lie in [0, 15], the extremes of every group map to codes 0 and 15,
  and codes are monotone in the value within a group;
* dequantisation is within one step (plus bf16 rounding) of the input;
* a group whose values are all equal dequantises exactly;
* the bf16 rounding of the dequantised values is round-to-nearest-even
  (checked by hand on ties);
* the summaries of the dequantised keys bound every dequantised key.
"""
import numpy as np
import torch

import workloads as W
from oracle import quant as Q
from oracle import selection as Sel


def pool(seed=3, B=2, ctx=150, Hkv=2, d=16, lens=None):
    rng = np.random.default_rng(seed)
    k = torch.from_numpy(rng.standard_normal((B, ctx, Hkv, d)).astype(np.float32) * 3).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((B, ctx, Hkv, d)).astype(np.float32)).to(torch.bfloat16)
    n = (ctx + 63) // 64
    NP = B * n + 1
    pt = torch.from_numpy(rng.permutation(NP)[: B * n].reshape(B, n).astype(np.int32))
    pc = W.scatter_to_pages(k, v, pt, NP)
    lens = np.array([ctx] * B if lens is None else lens, np.int32)
    return pc.k_pages.float().numpy(), pc.v_pages.float().numpy(), pt.numpy(), lens


def unpack(q):
    return np.stack([q & 15, q >> 4], axis=-1).reshape(*q.shape[:-1], -1)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 5 * 2 ** -9], np.float32)
    # ties go to the even 7-bit mantissa; 1 + 5/512 lies nearer 1 + 1/128 than 1 + 2/128
    np.testing.assert_array_equal(Q.bf16_round(x), np.array([1.0, 1.0 + 2 ** -6, -2.5, 1.0 + 2 ** -7], np.float32))


def test_codes_range_extremes_monotone_and_error_bound():
    kp, vp, pt, L = pool(lens=[150, 97])
    kq, kpar, vq, vpar, kdeq, vdeq = Q.quantize_pages(kp, vp, pt, L)
    for b in range(2):
        for i in range(Sel.n_pages(L[b])):
            p, nv = pt[b, i], min(64, L[b] - 64 * i)
            for g in range(2):
                kc = unpack(kq[p, g])[:nv]
                x = kp[p, g, :nv]
                assert kc.max() <= 15
                for c in range(x.shape[1]):           # keys: per channel
                    col = x[:, c]
                    if col.max() > col.min():
                        assert kc[col.argmin(), c] == 0 and kc[col.argmax(), c] == 15
                    order = np.argsort(col, kind="stable")
                    assert np.all(np.diff(kc[order, c].astype(int)) >= 0)
                step = kpar[p, g, 0]
                err = np.abs(kdeq[p, g, :nv] - x)
                assert np.all(err <= step[None, :] * 0.5 * (1 + 1e-5) + np.abs(x) * 2 ** -8 + 1e-6)
                vc = unpack(vq[p, g])[:nv]
                y = vp[p, g, :nv]
                for t in range(nv):                    # values: per token
                    if y[t].max() > y[t].min():
                        assert vc[t, y[t].argmin()] == 0 and vc[t, y[t].argmax()] == 15
                err = np.abs(vdeq[p, g, :nv] - y)
                assert np.all(err <= vpar[p, g, 0, :nv, None] * 0.5 * (1 + 1e-5) + np.abs(y) * 2 ** -8 + 1e-6)


def test_constant_group_dequantises_exactly():
    kp, vp, pt, L = pool()
    kp[:] = 1.5
    vp[:] = -0.25
    _, _, _, _, kdeq, vdeq = Q.quantize_pages(kp, vp, pt, L)
    for b in range(2):
        for i in range(Sel.n_pages(L[b])):
            p, nv = pt[b, i], min(64, L[b] - 64 * i)
            assert np.all(kdeq[p, :, :nv] == 1.5) and np.all(vdeq[p, :, :nv] == -0.25)


def test_summaries_of_dequantised_keys_bound_them():
    kp, vp, pt, L = pool(lens=[150, 70])
    kind = np.array([0, 1], np.uint8)
    _, _, _, _, kdeq, _ = Q.quantize_pages(kp, vp, pt, L)
    st = Q.quantized_stats(kdeq, pt, L, kind)
    for b in range(2):
        for t in range(L[b]):
            p, r = pt[b, t // 64], t % 64
            lp = r // 16
            assert np.all(st[p, 0, lp, 0] <= kdeq[p, 0, r]) and np.all(kdeq[p, 0, r] <= st[p, 0, lp, 1])
