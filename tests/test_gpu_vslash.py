"""GPU parity of the vertical-slash mask construction (lserve_build_vslash_mask)
against the oracle (oracle/vslash.py), through the C ABI.

Both sides take the same bf16 inputs; the oracle works in float64, the library
in float32 with fixed-order sums.  The mask decides integers from floating
point (which candidate ranks first, where the greedy stops), so it must equal
the oracle's exactly unless the oracle itself is within rounding of a decision:
two candidates ranked next to each other within 1e-5 relative, or the sampled
CRA at the stopping point within 1e-5 of tau.  Such cases are reported, not
accepted silently: the seeded inputs here are checked to be clear of them.
The sampled CRA must match to 1e-4 (fp32 sums of at most a few thousand tile
masses).
"""
import dataclasses

import numpy as np
import pytest
import torch

import workloads as W
from oracle import vslash as OV
from parity import f64

pytestmark = pytest.mark.gpu

U = pytest.importorskip("unified_sparse_attention_b200")


def decisions_clear(tiles, r, tau, taken, cras):
    order = OV.candidate_order(tiles, r)
    sc = np.array([c[2] for c in order[1:]])
    gaps = np.abs(np.diff(sc)) / np.maximum(np.abs(sc[:-1]), 1e-30)
    near_tie = np.any(gaps[: len(taken) + 1] < 1e-5)
    near_tau = any(abs(c - tau) < 1e-5 for c in cras)
    return not near_tie and not near_tau


@pytest.mark.parametrize("Hq,Hkv,d,S,stride,tau", [
    (4, 2, 64, 1024, 1, 0.9),
    (8, 2, 128, 1472, 3, 0.95),     # 23 query tiles: sampled tiles 22, 19, ..., 1
    (4, 4, 128, 768, 2, 0.8),       # MHA
    (16, 2, 64, 640, 1, 0.99),      # G = 8
])
def test_vslash_mask_matches_oracle(Hq, Hkv, d, S, stride, tau):
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=Hq, Hkv=Hkv, d=d, anchors=6)
    q, k, _ = W.prefill_inputs(w, S=S)
    kind = [0] * Hkv
    kind[-1] = 1                                   # one streaming head: all-zero mask
    hk = torch.tensor(kind, dtype=torch.uint8, device="cuda")
    bm, cra, ncol, nsla = U.lserve_build_vslash_mask(q.cuda(), k.cuda(), hk, stride, tau)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    ref_m, ref_cra, ref_nc, ref_ns = OV.build_vslash_mask(f64(q), f64(k), kind, stride, tau)
    for g in range(Hkv):
        if kind[g]:
            assert not bm[0, g].any()
            continue
        tiles, r = OV.tile_masses(f64(q), f64(k), stride, g=g)
        taken, cras = OV.greedy(tiles, r, tau)
        assert decisions_clear(tiles, r, tau, taken, cras), "seeded input sits on a decision boundary"
        np.testing.assert_array_equal(bm[0, g].cpu().numpy(), ref_m[0, g])
        assert ncol[0, g].item() == ref_nc[0, g] and nsla[0, g].item() == ref_ns[0, g]
        assert abs(cra[0, g].item() - ref_cra[0, g]) <= 1e-4


def test_vslash_mask_feeds_prefill_and_cra():
    """The mask is a valid lserve_prefill / lserve_cra input; its full CRA over
    every row is reported next to the sampled one (only the sampled rows are
    guaranteed to reach tau)."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=128, anchors=6)
    q, k, v = (t.cuda() for t in W.prefill_inputs(w, S=1024))
    hk = torch.tensor([0, 1], dtype=torch.uint8, device="cuda")
    bm, cra_s, _, _ = U.lserve_build_vslash_mask(q, k, hk, 1, 0.9)
    out = U.lserve_prefill(q, k, v, hk, 64, 256, bm)
    cra_full = U.lserve_cra(q, k, v, hk, 64, 256, bm)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    assert torch.isfinite(out.float()).all()
    assert cra_s[0, 0].item() >= 0.9
    assert 0.0 < cra_full[0, 0].item() <= 1.0 + 5e-3


def test_vslash_tau_extremes():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2, Hkv=1, d=64)
    q, k, _ = (t.cuda() for t in W.prefill_inputs(w, S=512))
    hk = torch.zeros(1, dtype=torch.uint8, device="cuda")
    bm, cra, nc, ns = U.lserve_build_vslash_mask(q, k, hk, 1, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(bm[0, 0].cpu(), torch.tril(torch.ones(8, 8, dtype=torch.uint8)))
    bm, cra, nc, ns = U.lserve_build_vslash_mask(q, k, hk, 1, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(bm[0, 0].cpu(), torch.eye(8, dtype=torch.uint8)) and nc.item() == 0 and ns.item() == 1
