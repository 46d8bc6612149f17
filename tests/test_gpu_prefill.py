"""GPU parity of block-sparse prefill (tile lists + attention) against the oracle.

All calls go through the C ABI (ctypes binding).  Inputs come from the seeded
generators and are handed unchanged to both sides.
"""
import dataclasses

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from parity import assert_attn_close, assert_lse_close, f64

pytestmark = pytest.mark.gpu

U = pytest.importorskip("unified_sparse_attention_b200")


def run_case(w, S, kind, sink, local, mask_fill=None, B=None, seed_mask=True, lambda_tiles=False):
    dev = "cuda"
    q, k, v = W.prefill_inputs(w, S=S, B=B)
    hk = torch.tensor(kind, dtype=torch.uint8)
    bm = None
    if mask_fill is not None:
        ww = dataclasses.replace(w, mask_columns=2, mask_band=2)
        bm = W.block_mask(ww, S=S, fill=mask_fill, B=q.shape[0])
    out, lse = U.lserve_prefill(q.to(dev), k.to(dev), v.to(dev), hk.to(dev), sink, local,
                                None if bm is None else bm.to(dev), return_lse=True, lambda_tiles=lambda_tiles)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    ref, ref_lse = OA.masked_attention(f64(q), f64(k), f64(v), kind, sink, local,
                                       None if bm is None else bm.numpy(), lambda_tiles=lambda_tiles)
    assert_attn_close(f64(out), ref, "prefill out")
    assert_lse_close(f64(lse), ref_lse, "prefill lse")
    return q, k, v, hk, bm, out


def test_tiny_workload_exact_config():
    w = W.WORKLOADS["tiny"]
    run_case(w, w.S, W.head_kind(w).tolist(), w.sink, w.local)


@pytest.mark.parametrize("sink,local", [(64, 256), (70, 130), (0, 1), (1, 0), (200, 64)])
def test_gqa4_d128_block_mask(sink, local):
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=8, Hkv=2, d=128)
    run_case(w, 1024, [0, 1], sink, local, mask_fill=0.4)


def test_mha_d128_batch2():
    w = dataclasses.replace(W.WORKLOADS["tiny"], B=2, Hq=4, Hkv=4, d=128)
    run_case(w, 512, [0, 1, 1, 0], 64, 256, B=2)


def test_gqa8_d64_masks():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=16, Hkv=2, d=64)
    run_case(w, 640, [1, 0], 0, 100, mask_fill=0.3)


def test_single_tile_and_empty_rows():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2, Hkv=2, d=128)
    run_case(w, 64, [0, 1], 0, 0)          # streaming head: sink=0, local=0 -> every row empty
    w2 = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2, Hkv=1, d=64)
    q, k, v = W.prefill_inputs(w2, S=256)
    bm = torch.zeros(1, 1, 4, 4, dtype=torch.uint8)
    bm[0, 0, 2, 0] = 1                      # q-tile 2 keeps only kt=0; tiles 0, 1, 3 keep nothing
    dev = "cuda"
    out, lse = U.lserve_prefill(q.to(dev), k.to(dev), v.to(dev), torch.zeros(1, dtype=torch.uint8, device=dev),
                                0, 0, bm.to(dev), return_lse=True)
    ref, ref_lse = OA.masked_attention(f64(q), f64(k), f64(v), [0], 0, 0, bm.numpy())
    assert_attn_close(f64(out), ref, "empty rows")
    assert_lse_close(f64(lse), ref_lse, "empty rows lse")


@pytest.mark.parametrize("mask_fill", [None, 0.35])
def test_tile_lists_bit_exact(mask_fill):
    w = dataclasses.replace(W.WORKLOADS["tiny"], B=2, Hq=8, Hkv=4, d=128, mask_columns=3, mask_band=2)
    S = 1472   # 23 tiles
    kind = [0, 1, 0, 1]
    bm = W.block_mask(w, S=S, fill=mask_fill, B=2) if mask_fill is not None else None
    hk = torch.tensor(kind, dtype=torch.uint8, device="cuda")
    off, cols = U.lserve_prefill_tile_lists(2, S, 8, 4, 128, hk, 70, 190,
                                            None if bm is None else bm.cuda())
    torch.cuda.synchronize()
    ref_off, ref_cols = OA.tile_lists(2, S, kind, 70, 190, None if bm is None else bm.numpy())
    np.testing.assert_array_equal(off.cpu().numpy(), ref_off)
    got = cols.cpu().numpy().view(np.uint16)[: ref_off[-1]].astype(np.int64)
    np.testing.assert_array_equal(got, ref_cols)


def test_skipped_tiles_are_never_read():
    """Poison (NaN) every KV tile the last query tile does not keep: its rows are unchanged."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=128, mask_columns=1, mask_band=1)
    S, kind, sink, local = 1024, [0, 1], 64, 200
    q, k, v = W.prefill_inputs(w, S=S)
    bm = W.block_mask(w, S=S, fill=0.3)
    dev = "cuda"
    hk = torch.tensor(kind, dtype=torch.uint8, device=dev)
    clean = U.lserve_prefill(q.to(dev), k.to(dev), v.to(dev), hk, sink, local, bm.to(dev))
    k2, v2 = k.clone(), v.clone()
    nq = S // 64
    for g in range(2):
        kept = OA.tile_kept(S, bool(kind[g]), sink, local, None if kind[g] else bm[0, g].numpy())[nq - 1]
        for kt in np.nonzero(~kept)[0]:
            k2[0, kt * 64:(kt + 1) * 64, g] = float("nan")
            v2[0, kt * 64:(kt + 1) * 64, g] = float("nan")
    pois = U.lserve_prefill(q.to(dev), k2.to(dev), v2.to(dev), hk, sink, local, bm.to(dev))
    torch.cuda.synchronize()
    last = slice(S - 64, S)
    assert torch.equal(clean[:, last], pois[:, last])
    assert torch.isfinite(pois[:, last].float()).all()


def test_repeated_calls_are_deterministic():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=8, Hkv=2, d=128)
    q, k, v = (t.cuda() for t in W.prefill_inputs(w, S=512))
    hk = torch.tensor([0, 1], dtype=torch.uint8, device="cuda")
    a = U.lserve_prefill(q, k, v, hk, 64, 256)
    b = U.lserve_prefill(q, k, v, hk, 64, 256)
    assert torch.equal(a, b)


@pytest.mark.parametrize("G,S", [(1, 960), (2, 512), (3, 704), (5, 448), (8, 384)])
def test_gqa_ratios_and_odd_tile_count(G, S):
    """Odd G (1, 3, 5) pairs query tiles of one head (an odd tile count leaves a
    half pair); even G pairs two heads of one query tile."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2 * G, Hkv=2, d=128)
    run_case(w, S, [0, 1], 64, 150, mask_fill=0.5)


def test_d64_mha_pairs_with_mask():
    w = dataclasses.replace(W.WORKLOADS["tiny"], B=2, Hq=2, Hkv=2, d=64)
    run_case(w, 832, [0, 1], 32, 97, mask_fill=0.3, B=2)


@pytest.mark.parametrize("G", [1, 2])
@pytest.mark.parametrize("sink,local", [(0, 64), (0, 65), (0, 66), (130, 127), (0, 4096), (5000, 0), (63, 1),
                                        (65, 129)])
def test_streaming_tile_runs_edges(G, sink, local):
    """Where the window's tile count steps (local 64 / 65 / 66), a window or sink
    covering the whole sequence, and an odd tile count (G = 1 pairs query tiles,
    so the last pair is ragged): the kernel's own tile runs for streaming and
    unmasked dense heads against the oracle's token-level kept sets."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2 * G, Hkv=2, d=64)
    run_case(w, 576, [1, 0], sink, local)


@pytest.mark.parametrize("G", [1, 4])
@pytest.mark.parametrize("sink,local", [(64, 256), (0, 65), (70, 130), (1, 0), (0, 4096)])
def test_tile_level_lambda(G, sink, local):
    """Tile-level Lambda (every causal key of every tile that meets the support):
    against the oracle's tile-level kept sets, next to a block-masked dense head."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2 * G, Hkv=2, d=128)
    run_case(w, 704, [1, 0], sink, local, mask_fill=0.4, lambda_tiles=True)


def test_tile_level_lambda_differs_from_token_level_only_at_the_edges():
    """With sink and window on tile boundaries plus one (local = 65) the two
    readings differ; with sink = 64 and a window covering whole tiles in both
    (local >= S) they are the same computation."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=64)
    q, k, v = (t.cuda() for t in W.prefill_inputs(w, S=512))
    hk = torch.tensor([1, 1], dtype=torch.uint8, device="cuda")
    a = U.lserve_prefill(q, k, v, hk, 64, 65)
    b = U.lserve_prefill(q, k, v, hk, 64, 65, lambda_tiles=True)
    assert not torch.equal(a, b)
    a = U.lserve_prefill(q, k, v, hk, 64, 4096)
    b = U.lserve_prefill(q, k, v, hk, 64, 4096, lambda_tiles=True)
    assert torch.equal(a, b)
