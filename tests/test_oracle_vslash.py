"""Pins for the oracle's vertical-slash mask construction (oracle/vslash.py).

* tile masses against torch's softmax of the sampled rows (a library routine)
  summed over each tile, and every sampled row's masses sum to 1;
* the greedy on a hand-worked input (tests/golden/hand_examples.json): order of
  the candidates, sampled CRA after each, the candidates taken at three
  thresholds;
* the greedy against pure-Python brute force on random tiny inputs: the taken
  prefix is the shortest whose minimum retained mass (recounted tile by tile)
  reaches tau, and the mask holds exactly the tiles its candidates cover;
* tau = 1 keeps every causal tile; tau = 0 keeps only the diagonal;
* the sampled query tiles against their closed form.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import vslash as V

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


def hand_input():
    g = GOLD["vslash_greedy"]
    S = g["S"]
    q = np.zeros((1, S, 1, 2))
    q[0, :, 0, 0] = g["log_weight"]
    k = np.zeros((1, S, 1, 2))
    k[0, :64, 0, 0] = 1.0
    return q, k


def test_hand_example_order_and_cra():
    g = GOLD["vslash_greedy"]
    q, k = hand_input()
    tiles, r = V.tile_masses(q, k, 1, scale=1.0)
    order = V.candidate_order(tiles, r)
    assert [[c[0], c[1]] for c in order] == g["order"]
    taken, cras = V.greedy(tiles, r, 2.0)   # never reached: every candidate taken
    np.testing.assert_allclose(cras[:4], g["cra_after"], atol=1e-12)
    for tau in ("0.9", "0.95", "0.99"):
        taken, _ = V.greedy(tiles, r, float(tau))
        assert [list(t) for t in taken] == g[f"tau_{tau}_taken"], tau


def test_tile_masses_match_torch_softmax():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 320, 4, 16))
    k = rng.standard_normal((1, 320, 2, 16))
    tiles, r = V.tile_masses(q, k, 2, b=0, g=1)
    np.testing.assert_array_equal(tiles, [0, 2, 4])
    for s, qt in enumerate(tiles):
        i = 64 * qt + 63
        for h in range(2):
            logits = torch.from_numpy(q[0, i, 2 + h] @ k[0, : i + 1, 1].T / 4.0)
            w = torch.softmax(logits, dim=0).numpy()
            ref = np.array([w[64 * t: 64 * t + 64].sum() for t in range(qt + 1)])
            np.testing.assert_allclose(r[s, h, : qt + 1], ref, atol=1e-12)
            assert abs(r[s, h].sum() - 1) < 1e-12 and np.all(r[s, h, qt + 1:] == 0)


def brute_retained(tiles, r, taken):
    out = []
    for s, qt in enumerate(tiles):
        for h in range(r.shape[1]):
            tot = 0.0
            for kt in range(qt + 1):
                if any((kind == "column" and kt == idx) or (kind == "slash" and qt - kt == idx) for kind, idx in taken):
                    tot += r[s, h, kt]
            out.append(tot)
    return min(out)


@pytest.mark.parametrize("seed,tau,stride", [(1, 0.6, 1), (2, 0.8, 1), (3, 0.9, 2), (4, 0.5, 3)])
def test_greedy_brute_force(seed, tau, stride):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 384, 2, 8)) * 2
    k = rng.standard_normal((1, 384, 1, 8)) * 2
    tiles, r = V.tile_masses(q, k, stride)
    taken, cras = V.greedy(tiles, r, tau)
    order = [(c[0], c[1]) for c in V.candidate_order(tiles, r)]
    assert taken == order[: len(taken)]
    for m in range(1, len(taken) + 1):
        got = brute_retained(tiles, r, order[:m])
        assert abs(got - cras[m - 1]) < 1e-12
        if m < len(taken):
            assert got < tau
    assert cras[-1] >= tau or len(taken) == len(order)
    mask = V.mask_from(taken, 6)
    for qt in range(6):
        for kt in range(6):
            want = kt <= qt and any((kd == "column" and kt == ix) or (kd == "slash" and qt - kt == ix)
                                    for kd, ix in taken)
            assert mask[qt, kt] == want


def test_tau_extremes():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 256, 2, 8))
    k = rng.standard_normal((1, 256, 2, 8))
    kind = [0, 1]
    m1, cra1, _, _ = V.build_vslash_mask(q, k, kind, 1, 1.0)
    assert np.array_equal(m1[0, 0], np.tril(np.ones((4, 4), np.uint8)))
    assert abs(cra1[0, 0] - 1) < 1e-12
    assert not m1[0, 1].any()                     # streaming head: no mask
    m0, _, nc, ns = V.build_vslash_mask(q, k, kind, 1, 0.0)
    assert np.array_equal(m0[0, 0], np.eye(4, dtype=np.uint8)) and nc[0, 0] == 0 and ns[0, 0] == 1


@pytest.mark.parametrize("nQT,stride", [(1, 1), (7, 1), (7, 2), (7, 3), (8, 3), (5, 5), (4, 9), (64, 16)])
def test_sampled_tiles_closed_form(nQT, stride):
    """The last query tile is always sampled, then every stride-th tile below it."""
    t = V.sampled_tiles(nQT, stride)
    assert t[-1] == nQT - 1 and t[0] >= 0 and t[0] < stride
    assert len(t) == (nQT - 1) // stride + 1
    assert np.all(np.diff(t) == stride)
    if stride == 1:
        np.testing.assert_array_equal(t, np.arange(nQT))


def test_sampled_tiles_rejects_a_stride_below_one():
    with pytest.raises(ValueError):
        V.sampled_tiles(4, 0)
