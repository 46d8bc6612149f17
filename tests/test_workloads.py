"""The seeded input generators: determinism, shapes, and the stated recipes."""
import numpy as np
import torch

import workloads as W


def test_deterministic_and_bf16():
    w = W.WORKLOADS["tiny"]
    a = W.prefill_inputs(w)
    b = W.prefill_inputs(w)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16
        assert torch.equal(x, y)
    q, k, v = a
    assert q.shape == (1, 1024, 4, 64) and k.shape == (1, 1024, 2, 64)


def test_head_kind_counts():
    for w in W.WORKLOADS.values():
        kind = W.head_kind(w)
        assert int(kind.sum()) == w.n_streaming and len(kind) == w.Hkv


def test_anchor_keys_present():
    w = W.WORKLOADS["tiny"]
    _, k, _ = W.prefill_inputs(w)
    u = W.anchor_dirs(w)
    proj = (k[0].float() * u[None]).sum(-1)          # [S, Hkv]
    top = proj.topk(8, dim=0).values
    assert float(top.min()) > 1.5                      # 3u added at 8 positions per KV head


def test_vertical_slash_density_readings():
    w = W.WORKLOADS["llama3_8b_prefill_128k_vslash"]
    n = w.S // 64
    causal = np.tril(np.ones((n, n), bool))
    for fill, lo, hi in ((W.FILL_30PCT, 0.29, 0.31), (0.05, 0.060, 0.070)):
        m = W.block_mask(w, fill=fill)[0, 0].numpy().astype(bool)
        dens = (m & causal).sum() / causal.sum()
        assert lo < dens < hi, dens
        band = np.array([m[i, i - 7:i + 1].all() for i in range(7, n)])
        assert band.all()


def test_page_table_is_permutation_and_scatter_is_layout_only():
    w = W.WORKLOADS["tiny"]
    _, k, v = W.prefill_inputs(w)
    pt = W.page_table(w, 1, 16, 16)
    assert sorted(pt[0].tolist()) == list(range(16))
    pc = W.scatter_to_pages(k, v, pt, 16)
    for t in (0, 63, 64, 500, 1023):
        assert torch.equal(pc.k_pages[pt[0, t // 64], :, t % 64], k[0, t])
        assert torch.equal(pc.v_pages[pt[0, t // 64], :, t % 64], v[0, t])


def test_decode_cache_ragged_tail_is_nan():
    w = W.WORKLOADS["tiny"]
    pc = W.decode_cache(w, B=2, ctx=200, seq_lens=[200, 70], NP=10)
    p = int(pc.page_table[1, 1])
    assert torch.isnan(pc.k_pages[p, :, 6:].float()).all()
    assert not torch.isnan(pc.k_pages[p, :, :6].float()).any()
