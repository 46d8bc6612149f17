"""GPU parity of the decode path (page summaries, bound scores, top-k, split-KV
paged attention + LSE merge) against the oracle, through the C ABI."""
import dataclasses

import numpy as np
import pytest
import torch

import workloads as W
from oracle import decode as OD
from oracle import selection as OS
from parity import assert_attn_close, assert_lse_close, check_selection, f64

pytestmark = pytest.mark.gpu

U = pytest.importorskip("unified_sparse_attention_b200")


def make(w, B, ctx, lens=None, NP=None):
    pc = W.decode_cache(w, B=B, ctx=ctx, seq_lens=lens, NP=NP)
    q = W.decode_query(w, B=B)
    return pc, q


def run_decode(w, B, ctx, budget, sink, local, lens=None, kind=None, NP=None):
    dev = "cuda"
    pc, q = make(w, B, ctx, lens, NP)
    kind = W.head_kind(w).tolist() if kind is None else kind
    hk = torch.tensor(kind, dtype=torch.uint8)
    kp, vp = pc.k_pages.to(dev), pc.v_pages.to(dev)
    pt, sl = pc.page_table.to(dev), pc.seq_lens.to(dev)
    stats = U.lserve_update_page_stats(kp, pt, sl, hk.to(dev))
    lse = torch.empty(B, w.Hq, dtype=torch.float32, device=dev)
    out, _, sel, sel_n = U.lserve_decode(q.to(dev), kp, vp, pt, sl, stats, hk.to(dev), sink, local, budget,
                                         lse=lse, return_selection=True)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    # oracle on the same bf16 inputs
    kp64, vp64, pt_np, L = f64(pc.k_pages), f64(pc.v_pages), pc.page_table.numpy(), pc.seq_lens.numpy()
    st_ref = OS.page_stats(kp64, pt_np, L, kind)
    np.testing.assert_array_equal(f64(stats), st_ref)          # bit-exact summaries
    q64 = f64(q)
    sel_ref, margin, scores = OS.select(q64, st_ref, pt_np, L, kind, budget, sink, local)
    sel_np, seln_np = sel.cpu().numpy(), sel_n.cpu().numpy()
    gpu_sel, ties = {}, 0
    for b in range(B):
        for g in range(w.Hkv):
            row = sel_np[b, g, : seln_np[b, g]]
            gpu_sel[(b, g)] = row
            if kind[g]:
                assert list(row) == list(sel_ref[(b, g)])
            else:
                n = OS.n_pages(L[b])
                ties += check_selection(row, OS.budget_pages(budget, L[b]), scores[b, g, :n])
            assert np.all(sel_np[b, g, seln_np[b, g]:] == -1)
    ref_out, ref_lse = OD.decode_attention(q64, kp64, vp64, pt_np, L, kind, gpu_sel, sink, local)
    assert_attn_close(f64(out), ref_out, "decode out")
    assert_lse_close(f64(lse), ref_lse, "decode lse")
    return dict(pc=pc, q=q, out=out, sel=gpu_sel, stats=stats, kind=kind, ties=ties)


def test_tiny_workload_exact_config():
    w = W.WORKLOADS["tiny"]
    r = run_decode(w, 1, w.ctx, w.token_budget, w.sink, w.local)
    dense = [g for g in range(w.Hkv) if r["kind"][g] == 0]
    assert all(len(r["sel"][(0, g)]) == 4 for g in dense)


@pytest.mark.parametrize("G,d", [(1, 128), (2, 64), (4, 128), (8, 128)])
def test_ragged_batch(G, d):
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2 * G, Hkv=2, d=d, dec_anchors=16)
    run_decode(w, 3, 1000, 512, 64, 100, lens=[1000, 333, 65], kind=[0, 1])


def test_more_heads_and_pages():
    w = dataclasses.replace(W.WORKLOADS["llama3_8b_decode_b16_64k"], dec_anchors=32)
    run_decode(w, 2, 8192 + 77, 1024, 64, 256)


def test_budget_covers_context_equals_dense():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=128)
    r = run_decode(w, 2, 700, 1 << 20, 64, 256, kind=[0, 0])
    for b in range(2):
        assert list(r["sel"][(b, 0)]) == list(range(11))


def test_single_token_and_empty_sequence():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=64)
    run_decode(w, 3, 130, 128, 0, 1, lens=[1, 130, 0], kind=[0, 1])


def test_unselected_pages_are_never_read():
    """Poison every pool row outside the attended token sets: the output is unchanged."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=8, Hkv=2, d=128, dec_anchors=8)
    r = run_decode(w, 2, 1500, 256, 64, 100, lens=[1500, 1210], kind=[0, 1])
    pc, q, kind = r["pc"], r["q"], r["kind"]
    kp, vp = pc.k_pages.clone(), pc.v_pages.clone()
    L = pc.seq_lens.tolist()
    for b in range(2):
        for g in range(2):
            toks = set(OD.token_set(L[b], bool(kind[g]), 64, 100, None if kind[g] else r["sel"][(b, g)]).tolist())
            for i in range(OS.n_pages(L[b])):
                p = int(pc.page_table[b, i])
                for row in range(64):
                    if i * 64 + row not in toks:
                        kp[p, g, row] = float("nan")
                        vp[p, g, row] = float("nan")
    dev = "cuda"
    out2 = U.lserve_decode(q.to(dev), kp.to(dev), vp.to(dev), pc.page_table.to(dev), pc.seq_lens.to(dev),
                           r["stats"], torch.tensor(kind, dtype=torch.uint8, device=dev), 64, 100, 256)
    torch.cuda.synchronize()
    assert torch.equal(out2, r["out"])


def test_incremental_page_stats():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=128)
    pc = W.decode_cache(w, B=1, ctx=1000)
    dev = "cuda"
    hk = torch.tensor([0, 0], dtype=torch.uint8, device=dev)
    kp, pt = pc.k_pages.to(dev), pc.page_table.to(dev)
    full = U.lserve_update_page_stats(kp, pt, pc.seq_lens.to(dev), hk)
    stale = full.clone()
    stale[pc.page_table[0, 10:].long().to(dev)] = 0
    U.lserve_update_page_stats(kp, pt, pc.seq_lens.to(dev), hk, stats=stale, first_logical_page=40)
    torch.cuda.synchronize()
    assert torch.equal(torch.nan_to_num(stale.float(), nan=7.0), torch.nan_to_num(full.float(), nan=7.0))


def test_out_of_range_page_id_is_reported_not_read():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2, Hkv=1, d=64)
    pc = W.decode_cache(w, B=1, ctx=256, NP=4)
    pt = pc.page_table.clone()
    pt[0, 2] = 1 << 20                       # outside the pool
    dev = "cuda"
    U.lserve_get_device_status()
    U.lserve_update_page_stats(pc.k_pages.to(dev), pt.to(dev), pc.seq_lens.to(dev),
                               torch.zeros(1, dtype=torch.uint8, device=dev))
    assert U.lserve_get_device_status() == 6
    assert U.lserve_get_device_status() == 0   # read clears it


# The attention grid deals all selected pages out evenly to its CTAs.  Forcing a
# small grid makes one CTA stream many pages (more than one 256-page chunk) and
# many units (more than the 128 one chunk window spans), and lets the grid
# exceed the page count elsewhere.
def test_one_cta_crosses_page_chunks(monkeypatch):
    monkeypatch.setenv("LSERVE_DECODE_GRID", "1")
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2, Hkv=1, d=64, dec_anchors=8)
    r = run_decode(w, 1, 20000, 300 * 64, 64, 100, kind=[0])
    assert len(r["sel"][(0, 0)]) == 300


@pytest.mark.parametrize("grid", ["1", "3", "7", "1000"])
def test_small_grid_spans_many_units(monkeypatch, grid):
    monkeypatch.setenv("LSERVE_DECODE_GRID", grid)
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=8, Hkv=4, d=64, dec_anchors=4)
    B = 40
    lens = [(37 * b) % 300 for b in range(B)]     # ragged, some sequences empty
    run_decode(w, B, 300, 128, 16, 70, lens=lens, kind=[0, 1, 0, 1])


@pytest.mark.parametrize("grid", ["2", "5"])
def test_small_grid_gqa_d128(monkeypatch, grid):
    monkeypatch.setenv("LSERVE_DECODE_GRID", grid)
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=16, Hkv=2, d=128, dec_anchors=16)
    run_decode(w, 3, 1000, 512, 64, 100, lens=[1000, 333, 65], kind=[0, 1])


def _reuse_setup(w, B, ctx, L0, budget, sink, local):
    """Cache holding ctx valid tokens per sequence; a selection step at lengths L0."""
    dev = "cuda"
    pc, q = make(w, B, ctx)
    kind = [g % 2 for g in range(w.Hkv)]   # dense and streaming heads alternate
    hk = torch.tensor(kind, dtype=torch.uint8, device=dev)
    kp, vp, pt = pc.k_pages.to(dev), pc.v_pages.to(dev), pc.page_table.to(dev)
    l0 = torch.tensor(L0, dtype=torch.int32, device=dev)
    stats = U.lserve_update_page_stats(kp, pt, l0, hk)
    out, _, sel, sel_n = U.lserve_decode(q.to(dev), kp, vp, pt, l0, stats, hk, sink, local, budget,
                                         return_selection=True)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    return pc, q, kind, hk, kp, vp, pt, l0, out, sel, sel_n


@pytest.mark.parametrize("G,d", [(4, 128), (1, 64)])
def test_reuse_at_the_same_lengths_is_bit_identical(G, d):
    w = dataclasses.replace(W.WORKLOADS["llama3_8b_32k"], Hq=4 * G, Hkv=4, d=d)
    B, ctx = 3, 5000
    pc, q, kind, hk, kp, vp, pt, l0, out, sel, sel_n = _reuse_setup(w, B, ctx, [ctx, 3000, 777], 1024, 64, 256)
    lse = torch.empty(B, w.Hq, dtype=torch.float32, device="cuda")
    again = U.lserve_decode_reuse(q.to("cuda"), kp, vp, pt, l0, hk, 64, 256, 1024, sel, sel_n, lse=lse)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    assert torch.equal(again, out)


def test_reuse_after_appending_tokens_matches_oracle():
    w = dataclasses.replace(W.WORKLOADS["llama3_8b_32k"], Hq=16, Hkv=4, d=128)
    B, ctx, sink, local, budget = 3, 6000, 64, 256, 1024
    L0, L1 = [5000, 2100, 700], [6000, 2170, 701]
    pc, q, kind, hk, kp, vp, pt, l0, _, sel, sel_n = _reuse_setup(w, B, ctx, L0, budget, sink, local)
    l1 = torch.tensor(L1, dtype=torch.int32, device="cuda")
    q1 = W.decode_query(w, B=B, step=1)   # the query of a later step
    lse = torch.empty(B, w.Hq, dtype=torch.float32, device="cuda")
    # the selection buffers double as outputs: dense rows stay, streaming rows follow the new lengths
    out = U.lserve_decode_reuse(q1.to("cuda"), kp, vp, pt, l1, hk, sink, local, budget, sel, sel_n, lse=lse,
                                sel_out=sel, sel_n_out=sel_n)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    sel_np, seln_np = sel.cpu().numpy(), sel_n.cpu().numpy()
    kept = {(b, g): sel_np[b, g, : seln_np[b, g]] for b in range(B) for g in range(w.Hkv)}
    ref_out, ref_lse = OD.reuse_decode(f64(q1), f64(pc.k_pages), f64(pc.v_pages), pc.page_table.numpy(),
                                       np.array(L1), kind, kept, sink, local)
    assert_attn_close(f64(out), ref_out, "reuse out")
    assert_lse_close(f64(lse), ref_lse, "reuse lse")
    for b in range(B):   # streaming rows were refreshed for the new lengths
        t = np.arange(L1[b])
        window = sorted(set((t[(t < sink) | (t >= L1[b] - local)] // 64).tolist()))
        for g in range(w.Hkv):
            if kind[g]:
                assert list(kept[(b, g)]) == window


def test_reuse_reports_a_page_index_outside_the_table():
    w = dataclasses.replace(W.WORKLOADS["llama3_8b_32k"], Hq=8, Hkv=2, d=128)
    B, ctx = 2, 3000
    pc, q, kind, hk, kp, vp, pt, l0, _, sel, sel_n = _reuse_setup(w, B, ctx, [ctx, ctx], 1024, 64, 256)
    dense = kind.index(0)
    bad = sel.clone()
    bad[0, dense, 0] = pt.shape[1] + 5            # not a page of the sequence's table
    U.lserve_decode_reuse(q.to("cuda"), kp, vp, pt, l0, hk, 64, 256, 1024, bad, sel_n)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 6   # LSERVE_ERR_DEVICE_BOUNDS
    assert U.lserve_get_device_status() == 0


@pytest.mark.parametrize("G,d", [(1, 128), (4, 128), (2, 64)])
def test_cross_mode_decode_equals_last_prefill_row(G, d):
    """The two CUDA paths agree: decoding the last prefill query against the
    prefill's own K/V (paged, pool rows outside the sequence NaN) with a budget
    covering the context (dense heads) or the same sink / local (streaming
    heads) gives the prefill's last output row."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2 * G, Hkv=2, d=d)
    S, sink, local = 640, 64, 150
    q, k, v = W.prefill_inputs(w, S=S)
    dev = "cuda"
    hk = torch.tensor([0, 1], dtype=torch.uint8, device=dev)
    pre = U.lserve_prefill(q.to(dev), k.to(dev), v.to(dev), hk, sink, local)
    pt = W.page_table(w, 1, S // 64, 16)
    pc = W.scatter_to_pages(k, v, pt, 16)
    kp, vp = pc.k_pages.to(dev), pc.v_pages.to(dev)
    ptd, sl = pc.page_table.to(dev), pc.seq_lens.to(dev)
    stats = U.lserve_update_page_stats(kp, ptd, sl, hk)
    out = U.lserve_decode(q[:, S - 1].contiguous().to(dev), kp, vp, ptd, sl, stats, hk, sink, local, S)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    assert_attn_close(f64(out[0]), f64(pre[0, S - 1]), "decode vs last prefill row")
