"""Failure detection on the GPU without a fault: the kernels' bounded waits.

Every wait inside the decode attention kernel and the tcgen05 prefill kernel
gives up after LSERVE_WAIT_TIMEOUT_NS, records LSERVE_ERR_DEVICE_TIMEOUT and
lets the CTA leave once its copies (and MMAs) in flight have landed.

* decode (bf16 and INT4 pages): with LSERVE_DEBUG_STALL_DECODE set, the page
  resolver publishes nothing -- a flag nobody sets -- so the issuer's and the
  consumers' waits run out;
* prefill: with LSERVE_DEBUG_STALL_PREFILL set, the producer hands out no work
  item, so the MMA and softmax warps' waits on the item ring run out.

Both with a 20 ms limit and nothing in flight.  The status must say so, and the
next call without the hook must give the same result as before on the same
context.
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


def test_decode_int4_wait_limit_reports_timeout_and_context_survives(monkeypatch):
    w = dataclasses.replace(W.WORKLOADS["llama3_8b_32k"], dec_anchors=32)
    dev = "cuda"
    pc = W.decode_cache(w, device=dev, B=2, ctx=8192)
    q = W.decode_query(w, device=dev, B=2)
    hk = W.head_kind(w).to(dev)
    pt, sl = pc.page_table.to(dev), pc.seq_lens.to(dev)
    kq, kpar, vq, vpar, st4 = U.lserve_quantize_pages_int4(pc.k_pages, pc.v_pages, pt, sl, hk)
    args = (q, kq, vq, kpar, vpar, pt, sl, st4, hk, w.sink, w.local, 1024)
    ref = U.lserve_decode_int4(*args)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0

    monkeypatch.setenv("LSERVE_WAIT_TIMEOUT_NS", "20000000")
    monkeypatch.setenv("LSERVE_DEBUG_STALL_DECODE", "1")
    U.lserve_decode_int4(*args)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == LSERVE_ERR_DEVICE_TIMEOUT
    assert "bounded wait" in U.lserve_last_error_string()

    monkeypatch.delenv("LSERVE_DEBUG_STALL_DECODE")
    monkeypatch.delenv("LSERVE_WAIT_TIMEOUT_NS")
    again = U.lserve_decode_int4(*args)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    assert torch.equal(again, ref)


def test_prefill_wait_limit_reports_timeout_and_context_survives(monkeypatch):
    w = W.WORKLOADS["tiny"]
    dev = "cuda"
    q, k, v = (t.to(dev) for t in W.prefill_inputs(w))
    hk = W.head_kind(w).to(dev)
    ref = U.lserve_prefill(q, k, v, hk, w.sink, w.local, None)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0

    monkeypatch.setenv("LSERVE_WAIT_TIMEOUT_NS", "20000000")
    monkeypatch.setenv("LSERVE_DEBUG_STALL_PREFILL", "1")
    U.lserve_prefill(q, k, v, hk, w.sink, w.local, None)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == LSERVE_ERR_DEVICE_TIMEOUT
    assert "bounded wait" in U.lserve_last_error_string()

    monkeypatch.delenv("LSERVE_DEBUG_STALL_PREFILL")
    monkeypatch.delenv("LSERVE_WAIT_TIMEOUT_NS")
    again = U.lserve_prefill(q, k, v, hk, w.sink, w.local, None)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    assert torch.equal(again, ref)
