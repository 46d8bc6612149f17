"""lserve_decode_noalloc: the decode step for callers that may not allocate.

Serving loops with a memory budget fixed at start-up, and plugin hosts that
own every device allocation, cannot hand the library a workspace.  The
no-allocation entry point takes its scratch from a fixed array inside the
library instead.  This test calls it through the C ABI twice in a row -- the
second call finds the first call's leftovers in the shared array -- and checks
each result against lserve_decode with an ordinary workspace, within the
tolerance the other decode tests use.  It also checks that a batch too large
for the array is refused before anything runs.  All output buffers are
allocated here, by the test, before the calls.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import workloads as W
from parity import assert_attn_close, f64

pytestmark = pytest.mark.gpu

U = pytest.importorskip("unified_sparse_attention_b200")


def case(w, B, ctx, lens, kind, budget, seed_step):
    dev = "cuda"
    pc = W.decode_cache(w, B=B, ctx=ctx, seq_lens=lens)
    q = W.decode_query(w, B=B, step=seed_step).to(dev)
    hk = torch.tensor(kind, dtype=torch.uint8, device=dev)
    kp, vp, pt, sl = (t.to(dev) for t in (pc.k_pages, pc.v_pages, pc.page_table, pc.seq_lens))
    stats = U.lserve_update_page_stats(kp, pt, sl, hk)
    return (q, kp, vp, pt, sl, stats, hk, w.sink, w.local, budget)


def test_noalloc_decode_matches_workspace_decode_on_two_calls_in_a_row():
    w1 = dataclasses.replace(W.WORKLOADS["tiny"], Hq=8, Hkv=2, d=128, dec_anchors=16)
    w2 = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=4, d=64, dec_anchors=8)
    cases = [case(w1, 3, 2000, [2000, 777, 65], [0, 1], 512, 0),   # larger call first
             case(w2, 2, 700, [700, 129], [1, 0, 0, 1], 256, 1)]    # then a smaller one
    for args in cases:
        q = args[0]
        B, Hq, _ = q.shape
        Hkv = args[1].shape[1]
        kcap = U.lserve_decode_max_selected(B, Hq, Hkv, q.shape[2], args[1].shape[0], args[3].shape[1],
                                            args[7], args[8], args[9])
        ref = torch.empty_like(q)
        ref_sel = torch.empty(B, Hkv, kcap, dtype=torch.int32, device=q.device)
        ref_n = torch.empty(B, Hkv, dtype=torch.int32, device=q.device)
        U.lserve_decode(*args, out=ref, sel_out=ref_sel, sel_n=ref_n)
        out = torch.full_like(q, float("nan"))
        sel = torch.full((B, Hkv, kcap), -7, dtype=torch.int32, device=q.device)
        sel_n = torch.full((B, Hkv), -7, dtype=torch.int32, device=q.device)
        U.lserve_decode_noalloc(*args, out=out, sel_out=sel, sel_n=sel_n)
        torch.cuda.synchronize()
        assert U.lserve_get_device_status() == 0
        assert torch.equal(sel, ref_sel) and torch.equal(sel_n, ref_n)
        assert_attn_close(f64(out), f64(ref), "noalloc vs workspace decode")


def test_noalloc_narrows_its_grid_where_a_full_wave_would_not_fit():
    """G = 8, d = 128: a full wave's split partials alone need more than the
    array holds, so the call takes a narrower attention grid.  Same pages, same
    attention within the decode tolerance, for a batch of one and of three."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=16, Hkv=2, d=128, dec_anchors=16)
    for B, lens in ((1, [1500]), (3, [1500, 640, 64])):
        args = case(w, B, 1500, lens, [0, 1], 512, 2)
        q = args[0]
        Hkv = args[1].shape[1]
        kcap = U.lserve_decode_max_selected(B, 16, Hkv, 128, args[1].shape[0], args[3].shape[1],
                                            args[7], args[8], args[9])
        ref = torch.empty_like(q)
        ref_sel = torch.empty(B, Hkv, kcap, dtype=torch.int32, device=q.device)
        ref_n = torch.empty(B, Hkv, dtype=torch.int32, device=q.device)
        U.lserve_decode(*args, out=ref, sel_out=ref_sel, sel_n=ref_n)
        out = torch.full_like(q, float("nan"))
        sel = torch.full((B, Hkv, kcap), -7, dtype=torch.int32, device=q.device)
        sel_n = torch.full((B, Hkv), -7, dtype=torch.int32, device=q.device)
        U.lserve_decode_noalloc(*args, out=out, sel_out=sel, sel_n=sel_n)
        torch.cuda.synchronize()
        assert U.lserve_get_device_status() == 0
        assert torch.equal(sel, ref_sel) and torch.equal(sel_n, ref_n)
        assert_attn_close(f64(out), f64(ref), "noalloc (narrowed grid) vs workspace decode")


def test_noalloc_refuses_batches_larger_than_its_array():
    from unified_sparse_attention_b200 import binding as Bd
    lib = U.load_library()
    big = 1 << 20   # 16 sequences x 8 KV heads x 2^20-page rows of scores cannot fit in 16 MiB
    a = Bd.DecodeArgs(16, 32, 8, 128, big, big, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20,
                      64, 256, 4096, 0.0)
    assert lib.lserve_decode_workspace_size(ctypes.byref(a)) > Bd.NOALLOC_SCRATCH_BYTES
    rc = lib.lserve_decode_noalloc(ctypes.byref(a), ctypes.c_void_p(1 << 20), None, None, None, None)
    assert rc == 3
    assert "scratch" in U.lserve_last_error_string()
