"""GPU parity of the INT4 KV pages (quantiser and the decode step over INT4
pages) against the oracle, through the C ABI.

The quantiser's codes, steps, offsets and page summaries are integer or float32
decisions taken in float32 on both sides: bit-exact.  The decode step over INT4
pages is compared with the oracle's decode on the dequantised pools (the
oracle's own dequantisation), at the attention tolerances.  The library's bytes
are unpacked into the oracle's plain [token, channel] order first
(tests/int4_format.py, the storage format declared in include/lserve.h)."""
import dataclasses

import numpy as np
import pytest
import torch

import workloads as W
from oracle import decode as OD
from oracle import quant as OQ
from oracle import selection as OS
from parity import assert_attn_close, assert_lse_close, check_selection, f64
import int4_format as F

pytestmark = pytest.mark.gpu

U = pytest.importorskip("unified_sparse_attention_b200")


def quantize(pc, kind, first_page=0, bufs=None):
    dev = "cuda"
    NP, Hkv, P, d = pc.k_pages.shape
    if bufs is None:
        stats = torch.full((NP, Hkv, 4, 2, d), float("nan"), dtype=torch.bfloat16, device=dev)
        bufs = dict(stats=stats)
    r = U.lserve_quantize_pages_int4(pc.k_pages.to(dev), pc.v_pages.to(dev), pc.page_table.to(dev),
                                     pc.seq_lens.to(dev), torch.tensor(kind, dtype=torch.uint8, device=dev),
                                     first_page=first_page, **bufs)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    return dict(zip(("kq", "kpar", "vq", "vpar", "stats"), r))


def assert_quantiser_equal(g, qp, d):
    """The library's packed codes and parameters against the oracle's plain arrays, bit for bit."""
    np.testing.assert_array_equal(F.unpack_keys(g["kq"].cpu().numpy(), d), qp.kcode)
    np.testing.assert_array_equal(F.unpack_values(g["vq"].cpu().numpy(), d), qp.vcode)
    ks, klo = F.unpack_key_params(g["kpar"].cpu().numpy())
    np.testing.assert_array_equal(ks, qp.kstep)
    np.testing.assert_array_equal(klo, qp.klo)
    vs, vlo = F.unpack_value_params(g["vpar"].cpu().numpy())
    np.testing.assert_array_equal(vs, qp.vstep)
    np.testing.assert_array_equal(vlo, qp.vlo)


@pytest.mark.parametrize("d,lens", [(128, [1000, 333, 65]), (64, [130, 1, 640])])
def test_quantiser_bit_exact(d, lens):
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=d)
    pc = W.decode_cache(w, B=len(lens), ctx=max(lens), seq_lens=lens)
    kind = [0, 1]
    g = quantize(pc, kind)
    qp = OQ.quantize_pages(f64(pc.k_pages), f64(pc.v_pages), pc.page_table.numpy(), pc.seq_lens.numpy())
    assert_quantiser_equal(g, qp, d)
    st = OQ.quantized_stats(qp.kdeq, pc.page_table.numpy(), pc.seq_lens.numpy(), kind)
    np.testing.assert_array_equal(f64(g["stats"]), st)


def test_quantiser_first_page_keeps_earlier_pages():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=128)
    pc = W.decode_cache(w, B=2, ctx=900, seq_lens=[900, 520])
    kind = [0, 0]
    full = quantize(pc, kind)
    bufs = {k: torch.full_like(v, 7) if v.dtype != torch.bfloat16 else torch.full_like(v, 3.0)
            for k, v in full.items()}
    part = quantize(pc, kind, first_page=5, bufs=bufs)
    pt, L = pc.page_table.numpy(), pc.seq_lens.numpy()
    for b in range(2):
        for i in range(OS.n_pages(L[b])):
            p = int(pt[b, i])
            for name in ("kq", "vq", "kpar", "vpar", "stats"):
                got, ref = part[name][p], full[name][p]
                if i >= 5:
                    assert torch.equal(got, ref), (name, b, i)
                else:
                    assert torch.all(got == (3.0 if name == "stats" else 7)), (name, b, i)


def run_int4(w, B, ctx, budget, sink, local, lens=None, kind=None):
    dev = "cuda"
    pc = W.decode_cache(w, B=B, ctx=ctx, seq_lens=lens)
    q = W.decode_query(w, B=B)
    kind = W.head_kind(w).tolist() if kind is None else kind
    hk = torch.tensor(kind, dtype=torch.uint8, device=dev)
    g = quantize(pc, kind)
    pt, sl = pc.page_table.to(dev), pc.seq_lens.to(dev)
    lse = torch.empty(B, w.Hq, dtype=torch.float32, device=dev)
    out, _, sel, sel_n = U.lserve_decode_int4(q.to(dev), g["kq"], g["vq"], g["kpar"], g["vpar"], pt, sl,
                                              g["stats"], hk, sink, local, budget, lse=lse, return_selection=True)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    pt_np, L = pc.page_table.numpy(), pc.seq_lens.numpy()
    qp = OQ.quantize_pages(f64(pc.k_pages), f64(pc.v_pages), pt_np, L)
    kdeq, vdeq = qp.kdeq, qp.vdeq
    st_ref = OQ.quantized_stats(kdeq, pt_np, L, kind)
    q64 = f64(q)
    sel_ref, _, scores = OS.select(q64, st_ref, pt_np, L, kind, budget, sink, local)
    sel_np, seln_np = sel.cpu().numpy(), sel_n.cpu().numpy()
    gpu_sel = {}
    for b in range(B):
        for h in range(w.Hkv):
            row = sel_np[b, h, : seln_np[b, h]]
            gpu_sel[(b, h)] = row
            if kind[h]:
                assert list(row) == list(sel_ref[(b, h)])
            else:
                check_selection(row, OS.budget_pages(budget, L[b]), scores[b, h, : OS.n_pages(L[b])])
    ref_out, ref_lse = OD.decode_attention(q64, kdeq.astype(np.float64), vdeq.astype(np.float64), pt_np, L, kind,
                                           gpu_sel, sink, local)
    assert_attn_close(f64(out), ref_out, "int4 decode out")
    assert_lse_close(f64(lse), ref_lse, "int4 decode lse")
    return dict(pc=pc, q=q, out=out, lse=lse, kdeq=kdeq, vdeq=vdeq, stats=g["stats"], kind=kind, sel=gpu_sel)


@pytest.mark.parametrize("G,d", [(1, 128), (2, 64), (4, 128), (8, 128)])
def test_int4_decode_ragged_batch(G, d):
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2 * G, Hkv=2, d=d, dec_anchors=16)
    run_int4(w, 3, 1000, 512, 64, 100, lens=[1000, 333, 65], kind=[0, 1])


def test_int4_decode_gqa_many_pages():
    w = dataclasses.replace(W.WORKLOADS["llama3_8b_decode_b16_64k"], dec_anchors=32)
    run_int4(w, 2, 8192 + 77, 1024, 64, 256)


def test_int4_decode_single_token_and_empty_sequence():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=64)
    run_int4(w, 3, 130, 128, 0, 1, lens=[1, 130, 0], kind=[0, 1])


def test_int4_decode_matches_bf16_decode_on_dequantised_pools():
    """The bf16 path over pools holding the dequantised values, and the INT4
    path (steps folded into bf16(s q) and bf16(s p)), agree within the
    attention tolerance, and select the same pages (same summaries)."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=8, Hkv=2, d=128, dec_anchors=8)
    r = run_int4(w, 2, 1500, 256, 64, 100, lens=[1500, 1210], kind=[0, 1])
    dev = "cuda"
    pc = r["pc"]
    kd = torch.from_numpy(r["kdeq"]).to(torch.bfloat16).to(dev)
    vd = torch.from_numpy(r["vdeq"]).to(torch.bfloat16).to(dev)
    hk = torch.tensor(r["kind"], dtype=torch.uint8, device=dev)
    lse = torch.empty_like(r["lse"])
    out, _, sel, sel_n = U.lserve_decode(r["q"].to(dev), kd, vd, pc.page_table.to(dev), pc.seq_lens.to(dev),
                                         r["stats"], hk, 64, 100, 256, lse=lse, return_selection=True)
    torch.cuda.synchronize()
    for (b, h), row in r["sel"].items():
        assert list(sel[b, h, : sel_n[b, h]].cpu().numpy()) == list(row)
    assert_attn_close(f64(r["out"]), f64(out), "int4 vs bf16 on dequantised pools")
    assert_lse_close(f64(r["lse"]), f64(lse), "int4 vs bf16 lse")


def test_int4_decode_rejects_missing_params():
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=4, Hkv=2, d=128)
    pc = W.decode_cache(w, B=1, ctx=300)
    g = quantize(pc, [0, 1])
    lib = U.load_library()
    from unified_sparse_attention_b200.binding import DecodeArgs
    import ctypes
    q = W.decode_query(w, B=1).to("cuda")
    pt, sl = pc.page_table.to("cuda"), pc.seq_lens.to("cuda")
    hk = torch.tensor([0, 1], dtype=torch.uint8, device="cuda")
    a = DecodeArgs(1, 4, 2, 128, pc.k_pages.shape[0], pt.shape[1], q.data_ptr(), g["kq"].data_ptr(),
                   g["vq"].data_ptr(), pt.data_ptr(), sl.data_ptr(), g["stats"].data_ptr(), hk.data_ptr(), 64, 64,
                   256, 0.0)
    out = torch.empty_like(q)
    ws = torch.empty(int(lib.lserve_decode_workspace_size(ctypes.byref(a))), dtype=torch.uint8, device="cuda")
    st = lib.lserve_decode_int4(ctypes.byref(a), None, g["vpar"].data_ptr(), out.data_ptr(), None, None, None,
                                ws.data_ptr(), ws.numel(), None)
    assert st != 0 and "kpar" in U.lserve_last_error_string()


def test_int4_unattended_parameters_are_never_used():
    """NaN in the value steps/offsets of every row outside the attended token
    sets, and in the key steps/offsets of every page holding no attended token:
    the output is unchanged, bit for bit."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=8, Hkv=2, d=128, dec_anchors=8)
    r = run_int4(w, 2, 1500, 256, 64, 100, lens=[1500, 1210], kind=[0, 1])
    pc, kind = r["pc"], r["kind"]
    g = quantize(pc, kind)
    kpar, vpar = g["kpar"].cpu().clone(), g["vpar"].cpu().clone()
    L = pc.seq_lens.tolist()
    nan = float("nan")
    for b in range(2):
        for h in range(2):
            toks = set(OD.token_set(L[b], bool(kind[h]), 64, 100, None if kind[h] else r["sel"][(b, h)]).tolist())
            for i in range(OS.n_pages(L[b])):
                p = int(pc.page_table[b, i])
                rows = [row for row in range(64) if i * 64 + row not in toks]
                vpar[p, h, rows] = nan
                if len(rows) == 64:
                    kpar[p, h] = nan
    dev = "cuda"
    out2 = U.lserve_decode_int4(r["q"].to(dev), g["kq"], g["vq"], kpar.to(dev), vpar.to(dev), pc.page_table.to(dev),
                                pc.seq_lens.to(dev), g["stats"], torch.tensor(kind, dtype=torch.uint8, device=dev),
                                64, 100, 256)
    torch.cuda.synchronize()
    assert torch.equal(out2, r["out"])


def test_quantiser_ties_and_near_ties():
    """Groups built so that (x - lo) / s falls exactly on, or within float32
    rounding of, a half-integer: the codes (round half to even on the IEEE
    quotient) match the oracle bit for bit."""
    d, S = 64, 128
    k = torch.zeros(1, S, 2, d)
    v = torch.zeros(1, S, 2, d)
    t = torch.arange(64, dtype=torch.float32)
    c = torch.arange(d, dtype=torch.float32)
    # page 0: lo = 0, hi = 15, s = 1; values 0, 0.5, ..., 14.5 (exact ties at the odd halves)
    k[0, :64, :, :] = ((t[:, None] + c[None, :]) % 30 * 0.5)[:, None, :]
    k[0, 0, :, :], k[0, 1, :, :] = 0.0, 15.0
    v[0, :64, :, :] = ((t[:, None] + c[None, :]) % 30 * 0.5)[:, None, :]
    v[0, :64, :, 0], v[0, :64, :, 1] = 0.0, 15.0
    # page 1: lo = -1.5, hi = 0, s = fl(0.1); values -1.5 + 0.05 j, rounded to bf16 (near ties)
    k[0, 64:, :, :] = (-1.5 + 0.05 * ((t[:, None] * 7 + c[None, :]) % 31))[:, None, :]
    k[0, 64, :, :], k[0, 65, :, :] = -1.5, 0.0
    v[0, 64:, :, :] = (-1.5 + 0.05 * ((t[:, None] * 3 + c[None, :]) % 31))[:, None, :]
    v[0, 64:, :, 0], v[0, 64:, :, 1] = -1.5, 0.0
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    pt = torch.tensor([[1, 0]], dtype=torch.int32)
    pc = W.scatter_to_pages(k, v, pt, 2)
    kind = [0, 0]
    g = quantize(pc, kind)
    qp = OQ.quantize_pages(f64(pc.k_pages), f64(pc.v_pages), pc.page_table.numpy(), pc.seq_lens.numpy())
    assert_quantiser_equal(g, qp, d)
    st = OQ.quantized_stats(qp.kdeq, pc.page_table.numpy(), pc.seq_lens.numpy(), kind)
    np.testing.assert_array_equal(f64(g["stats"]), st)
    # the constructed groups do reach exact ties: some code is an even neighbour of x / s
    codes = qp.kcode[1, 0, 5]
    x = f64(pc.k_pages)[1, 0, 5]
    assert np.any((x % 1 == 0.5) & (codes % 2 == 0))


def test_int4_decode_reports_operands_past_fp16():
    """The folded operands are fp16: a key channel whose step times q leaves the fp16 range
    (|s q| > 65504) must be reported (LSERVE_ERR_DEVICE_BOUNDS), not turned into a silent
    non-finite output; the same call on ordinary keys reports nothing."""
    w = dataclasses.replace(W.WORKLOADS["tiny"], Hq=2, Hkv=2, d=128)
    dev = "cuda"
    pc = W.decode_cache(w, B=1, ctx=300)
    kind = [0, 1]
    q = W.decode_query(w, B=1).to(dev)
    pt, sl = pc.page_table.to(dev), pc.seq_lens.to(dev)
    hk = torch.tensor(kind, dtype=torch.uint8, device=dev)
    g = quantize(pc, kind)
    U.lserve_decode_int4(q, g["kq"], g["vq"], g["kpar"], g["vpar"], pt, sl, g["stats"], hk, 64, 64, 256)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 0
    # channel 5 of every key scaled so that its per-page step is ~1e5 (finite in bf16)
    big = pc.k_pages.clone()
    big[:, :, :, 5] = big[:, :, :, 5] * 3.0e5
    pc_big = dataclasses.replace(pc, k_pages=big)
    gb = quantize(pc_big, kind)
    qb = q.clone()
    qb[:, :, 5] = 1.0   # so that |s q| is the step itself, far past 65504
    U.lserve_decode_int4(qb, gb["kq"], gb["vq"], gb["kpar"], gb["vpar"], pt, sl, gb["stats"], hk, 64, 64, 256)
    torch.cuda.synchronize()
    assert U.lserve_get_device_status() == 6   # LSERVE_ERR_DEVICE_BOUNDS
