"""Failure detection on the GPU without a fault: the decode kernel's bounded waits.

Every wait inside the decode attention kernel (on a stage's loads, on a free
stage, on the page resolver) gives up after LSERVE_WAIT_TIMEOUT_NS, records
LSERVE_ERR_DEVICE_TIMEOUT and lets the CTA leave after its copies in flight
have landed.  With LSERVE_DEBUG_STALL_DECODE set, the kernel's page resolver
publishes nothing -- a flag nobody sets -- so the issuer's and the consumers'
waits run out (with a 20 ms limit).  The status must say so, and the next call
without the hook must give the same result as before on the same context.
"""
import dataclasses

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

U = pytest.importorskip("unified_sparse_attention_b200")

LSERVE_ERR_DEVICE_TIMEOUT = 5


def test_decode_wait_limit_reports_timeout_and_context_survives(monkeypatch):
    w = dataclasses.replace(W.WORKLOADS["llama3_8b_32k"], dec_anchors=32)
    dev = "cuda"
    pc = W.decode_cache(w, device=dev, B=2, ctx=8192)
    q = W.decode_query(w, device=dev, B=2)
    hk = W.head_kind(w).to(dev)
    pt, sl = pc.page_table.to(dev), pc.seq_lens.to(dev)
    stats = U.lserve_update_page_stats(pc.k_pages, pt, sl, hk)
    args = (q, pc.k_pages, pc.v_pages, pt, sl, stats, hk, w.sink, w.local, 1024)
    ref = U.lserve_decode(*args)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0

    monkeypatch.setenv("LSERVE_WAIT_TIMEOUT_NS", "20000000")
    monkeypatch.setenv("LSERVE_DEBUG_STALL_DECODE", "1")
    U.lserve_decode(*args)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == LSERVE_ERR_DEVICE_TIMEOUT
    assert "bounded wait" in U.lserve_last_error_string()

    monkeypatch.delenv("LSERVE_DEBUG_STALL_DECODE")
    monkeypatch.delenv("LSERVE_WAIT_TIMEOUT_NS")
    again = U.lserve_decode(*args)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    assert torch.equal(again, ref)
