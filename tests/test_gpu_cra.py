"""GPU parity of the CRA report (lserve_cra) against the oracle.

CRA (LServe + SampleAttention blog post, "CRA - The Accuracy Proxy", Fig. 4):
per query row the share of its causal softmax mass a sparse mask keeps, and
the minimum over the rows.  The GPU takes it from two LSE-only prefill passes,
so its error follows from the LSE bar (2e-3 absolute per pass):
|r - r_ref| <= r (exp(4e-3) - 1) < 5e-3.
"""
import dataclasses

import numpy as np
import pytest
import torch

import workloads as W
from oracle import cra as OC
from parity import f64

pytestmark = pytest.mark.gpu

U = pytest.importorskip("unified_sparse_attention_b200")

TOL = 5e-3


@pytest.mark.parametrize("Hq,Hkv,d,S,kind,sink,local,fill", [
    (4, 2, 64, 1024, [0, 1], 64, 256, 0.4),     # one dense head with a block mask, one streaming head
    (8, 2, 128, 768, [1, 0], 0, 100, 0.3),      # GQA 4, d 128
    (2, 2, 128, 640, [0, 0], 0, 0, 0.25),       # MHA (G = 1: two query tiles per work item), masks only
])
def test_cra_matches_oracle(Hq, Hkv, d, S, kind, sink, local, fill):
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=Hq, Hkv=Hkv, d=d, mask_columns=2, mask_band=2)
    dev = "cuda"
    q, k, v = W.prefill_inputs(w, S=S)
    bm = W.block_mask(w, S=S, fill=fill, B=q.shape[0])
    hk = torch.tensor(kind, dtype=torch.uint8)
    cra, ret = U.lserve_cra(q.to(dev), k.to(dev), v.to(dev), hk.to(dev), sink, local, bm.to(dev),
                            return_retained=True)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    ref = OC.retained_mass(f64(q), f64(k), f64(v), kind, sink, local, bm.numpy())
    got = f64(ret)
    assert np.all((got >= 0) & (got <= 1 + TOL))
    err = np.abs(got - ref).max()
    assert err <= TOL, f"retained mass max error {err:.3g}"
    np.testing.assert_allclose(f64(cra), ref.min(axis=2), atol=TOL)
    assert np.array_equal(f64(cra), got.min(axis=2))


def test_cra_is_one_when_nothing_is_dropped():
    w = W.WORKLOADS["tiny"]
    dev = "cuda"
    q, k, v = (t.to(dev) for t in W.prefill_inputs(w))
    hk = torch.zeros(w.Hkv, dtype=torch.uint8, device=dev)   # every head dense, no block mask
    cra = U.lserve_cra(q, k, v, hk, 0, 0, None)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    assert torch.all(cra == 1.0)   # the two passes are the same computation


def test_cra_tile_level_lambda():
    """The CRA of the tile-level Lambda reading: it keeps a superset of the
    token-level keys, so it retains at least as much."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=64)
    dev = "cuda"
    q, k, v = W.prefill_inputs(w, S=768)
    kind, sink, local = [1, 1], 30, 100
    hk = torch.tensor(kind, dtype=torch.uint8, device=dev)
    cra_t, ret_t = U.lserve_cra(q.to(dev), k.to(dev), v.to(dev), hk, sink, local, None, return_retained=True,
                                lambda_tiles=True)
    cra_e = U.lserve_cra(q.to(dev), k.to(dev), v.to(dev), hk, sink, local, None)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    ref = OC.retained_mass(f64(q), f64(k), f64(v), kind, sink, local, lambda_tiles=True)
    assert np.abs(f64(ret_t) - ref).max() <= TOL
    assert np.all(f64(cra_t) >= f64(cra_e) - TOL)
