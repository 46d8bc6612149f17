#!/usr/bin/env python
"""Benchmark of the unified sparse-attention hot path on B200.

One step = one pass of the whole path on one GPU:
  * prefill: kept-tile lists + block-sparse causal attention at 128K tokens
    (Llama-3-8B layer shape, 4 streaming KV heads with sink 64 + local 256, 4
    dense KV heads with a seeded vertical-slash block mask at ~30 % tile density);
  * decode: incremental page-summary refresh of the newest logical page, then
    one sparse decode step -- bound scoring, top-k pages, split-KV paged
    attention and LSE merge -- for 4 sequences of 262,144 tokens (Llama-2-7B MHA
    shape, 16 dense + 16 streaming KV heads, budget 8,192 tokens).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Prints ONE JSON line on rank 0.  Multi-GPU runs are independent replicas
(the path has no exchange step); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "prefill attn ms & kept-tile TFLOPS at 128K; decode attn µs/step & HBM GB/s"
PREFILL_WL = "llama3_8b_prefill_128k_vslash"
DECODE_WL = "llama2_7b_mha"
L2_BYTES = 126 * 1024 * 1024


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) from one-pass ncu
# captures of single kernels of this script's default workloads (profiles/
# launch_list__bench_default.md): per launch of the prefill attention kernel, and
# per decode step (scoring, top-k + plan, paged attention, merge).  Reported only
# while the kernel sources hash as they did when the counters were taken.
TRAFFIC = {
    "prefill": {"bytes": 3580308224,
                "sources": ["prefill_tc.cuh", "tile_lists.cuh", "common.cuh", "lserve.cu"],
                "sha256": "ef6557d1c5dc32360d988c00841410d9348e121b19022ecef1c67280a53e08bf"},
    "decode": {"bytes": 821729792,
               "sources": ["select.cuh", "decode.cuh", "page_stats.cuh", "common.cuh", "lserve.cu"],
               "sha256": "315f552b689e827de55a67f81fcaf23efebac042beee7f01196f3b306ed86eba"},
}


def traffic(key, workload_is_default):
    """Counter-measured DRAM bytes for `key`, or None when the workload is not the
    captured one or the kernel sources changed since the capture."""
    t = TRAFFIC[key]
    if not workload_is_default:
        return None
    h = hashlib.sha256()
    for f in t["sources"]:
        path = os.path.join(ROOT, "unified_sparse_attention_b200", "csrc", f)
        if not os.path.exists(path):
            return None
        with open(path, "rb") as fh:
            h.update(fh.read())
    return t["bytes"] if h.hexdigest() == t["sha256"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, source="fallback")


# ------------------------------------------------------------------ workload

def kept_tile_counts(w, bm, kind):
    """Kept 64x64 tiles per KV head (dense: causal tiles the mask keeps; streaming:
    tiles meeting the Lambda support).  Pure bookkeeping for the FLOP count."""
    n = w.S // 64
    qt = torch.arange(n, device=bm.device if bm is not None else "cpu")[:, None]
    kt = torch.arange(n, device=qt.device)[None, :]
    causal = kt <= qt
    counts = []
    for g in range(w.Hkv):
        if kind[g]:
            mind = torch.clamp(64 * qt - 64 * kt - 63, min=0)
            keep = causal & ((64 * kt < w.sink) | (mind < w.local))
            counts.append(int(keep.sum()) * w.B)
        elif bm is not None:
            counts.append(sum(int((causal & (bm[b, g] != 0)).sum()) for b in range(w.B)))
        else:
            counts.append(int(causal.sum()) * w.B)
    return counts


def decode_bytes(w, kind, k_pages_per_seq, d):
    """Bytes the decode step must read/write (algorithmic, not what a kernel happens to touch)."""
    n_dense = sum(1 for x in kind if x == 0)
    n_stream = len(kind) - n_dense
    n_pages = (w.ctx + 63) // 64
    stats = w.dec_B * n_dense * n_pages * 4 * 2 * d * 2
    sel = w.dec_B * n_dense * k_pages_per_seq * 64 * d * 2 * 2
    stream_tok = min(w.ctx, w.sink + w.local)
    stream = w.dec_B * n_stream * stream_tok * d * 2 * 2
    q_out = 2 * w.dec_B * w.Hq * d * 2
    table = w.dec_B * n_pages * 4
    return dict(stats=stats, selected=sel, streaming=stream, q_out=q_out, table=table,
                total=stats + sel + stream + q_out + table)


def decode_bytes_int4(w, kind, k_pages_per_seq, d):
    """The same step over INT4 pages: a K or V row is d/2 bytes of codes; a page
    adds its key steps/offsets (2 d fp32) and value steps/offsets (2 x 64 fp32)."""
    b = decode_bytes(w, kind, k_pages_per_seq, d)
    n_dense = sum(1 for x in kind if x == 0)
    n_stream = len(kind) - n_dense
    page = 64 * d + 2 * d * 4 + 2 * 64 * 4
    sel = w.dec_B * n_dense * k_pages_per_seq * page
    stream_tok = min(w.ctx, w.sink + w.local)
    stream = w.dec_B * n_stream * (stream_tok * (d + 8) + -(-stream_tok // 64) * 2 * d * 4)
    total = b["stats"] + sel + stream + b["q_out"] + b["table"]
    return dict(stats=b["stats"], selected=sel, streaming=stream, q_out=b["q_out"], table=b["table"], total=total)


class Setup:
    def __init__(self, device, prefill_wl=PREFILL_WL, decode_wl=DECODE_WL):
        self.dev = device
        self.prefill_wl, self.decode_wl = prefill_wl, decode_wl
        self.wp = W.WORKLOADS[prefill_wl]
        self.wd = W.WORKLOADS[decode_wl]
        wp, wd = self.wp, self.wd
        self.kind_p = W.head_kind(wp)
        self.kind_d = W.head_kind(wd)
        self.q, self.k, self.v = W.prefill_inputs(wp, device=device)
        self.bm = W.block_mask(wp, device=device)
        self.hk_p = self.kind_p.to(device)
        self.tiles = kept_tile_counts(wp, self.bm, self.kind_p.tolist())
        G = wp.Hq // wp.Hkv
        self.prefill_flops = sum(self.tiles) * G * 4 * 64 * 64 * wp.d
        pc = W.decode_cache(wd, device=device)
        self.kp, self.vp = pc.k_pages, pc.v_pages
        self.pt, self.sl = pc.page_table.to(device), pc.seq_lens.to(device)
        self.hk_d = self.kind_d.to(device)
        self.qd = W.decode_query(wd, device=device)
        self.k_sel = min(wd.token_budget // 64, (wd.ctx + 63) // 64)
        self.dbytes = decode_bytes(wd, self.kind_d.tolist(), self.k_sel, wd.d)
        self.last_lp = (wd.ctx - 1) // 16


# -------------------------------------------------------------------- timing

class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        rows = [r.split(", ") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, pw, reasons, smax = [], [], set(), None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                clk, watts = float(r[1]), float(r[3])
                smax = float(r[2])
            except (ValueError, IndexError):
                continue
            if watts < 300.0:   # a sample outside the timed kernels (the GPU idles near 150 W)
                continue
            sm.append(clk)
            pw.append(watts)
            for nme, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(nme)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w": statistics.median(pw), "under_load": "samples above 300 W"}


def max_over_ranks(vals, dist=None, device="cpu"):
    """Element-wise max of the per-rank timings `vals` over all ranks (the job's
    time is its slowest rank's); the values themselves on a single rank."""
    if dist is None:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def flush_l2(buf):
    """Flush L2 between timed steps: write 2 x L2 of one half of `buf`, then read 2 x L2 of the
    other half, so that the written half's dirty lines are written back here, before the step,
    instead of inside it (that write-back alone is ~126 MB, about 19 µs of HBM time)."""
    n = buf.numel() // 2
    buf[:n].add_(1.0)
    buf[n:].sum()


def time_loop(fn, steps, warmup, stream, scratch=None, events_per_step=1):
    """Warm up, then time `steps` calls with CUDA events on `stream`; with `scratch`,
    L2 is flushed (flush_l2) between calls, outside the events."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if scratch is not None:
            flush_l2(scratch)
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def graphed(fn, warmup=2):
    """fn captured once into a CUDA graph (its kernels exactly as the C ABI launches them, programmatic
    dependencies included); returns the replay.  A serving loop captures its decode step so: the host then
    enqueues one graph per step instead of four kernels through Python, and the step's time is the GPU's."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):   # captured on torch's side stream; replayed on the current one
        fn()
    torch.cuda.synchronize()
    return g.replay


# ------------------------------------------------------------ other configs

def prefill_config(U, wl, dev, stream, steps, pk, fill=None, lambda_tiles=False, tensors=None):
    """One prefill workload: median ms per call, kept-tile TFLOP/s and fraction of the bf16 peak."""
    w = W.WORKLOADS[wl]
    q, k, v = tensors if tensors is not None else W.prefill_inputs(w, device=dev)
    bm = W.block_mask(w, device=dev, fill=fill) if (fill is not None or w.mask_fill is not None) else None
    kind = W.head_kind(w)
    hk = kind.to(dev)
    tiles = kept_tile_counts(w, bm, kind.tolist())
    flops = sum(tiles) * (w.Hq // w.Hkv) * 4 * 64 * 64 * w.d
    out = torch.empty_like(q)
    ws = torch.empty(U.lserve_prefill_workspace_size(w.B, w.S, w.Hq, w.Hkv, w.d), dtype=torch.uint8, device=dev)
    fn = lambda: U.lserve_prefill(q, k, v, hk, w.sink, w.local, bm, out=out, workspace=ws, lambda_tiles=lambda_tiles)
    ms = float(np.median(time_loop(fn, steps, 3, stream)))
    n = w.S // 64
    dense = [t for t, x in zip(tiles, kind.tolist()) if x == 0]
    density = sum(dense) / max(1, len(dense) * n * (n + 1) // 2 * w.B)
    tf = flops / (ms * 1e-3) / 1e12
    return {"prefill_ms": ms, "kept_tile_tflop": flops / 1e12, "tflops": tf, "frac_bf16_peak": tf / pk["bf16"],
            "dense_tile_density": density}


def decode_config(U, wl, dev, stream, steps, pk, scratch):
    """One decode workload: median µs per step (selection re-run), GB/s on the algorithmic bytes, fraction
    of HBM, and the same step with L2 flushed before it."""
    w = W.WORKLOADS[wl]
    kind = W.head_kind(w)
    pc = W.decode_cache(w, device=dev)
    pt, sl, hk = pc.page_table.to(dev), pc.seq_lens.to(dev), kind.to(dev)
    stats = U.lserve_update_page_stats(pc.k_pages, pt, sl, hk)
    qd = W.decode_query(w, device=dev)
    args = (qd, pc.k_pages, pc.v_pages, pt, sl, stats, hk, w.sink, w.local, w.token_budget)
    ws = torch.empty(U.lserve_decode_workspace_size(*args), dtype=torch.uint8, device=dev)
    out = torch.empty_like(qd)
    fn = lambda: U.lserve_decode(*args, out=out, workspace=ws)
    us_eager = float(np.median(time_loop(fn, steps, 3, stream))) * 1e3
    us_eager_fl = float(np.median(time_loop(fn, steps, 2, stream, scratch))) * 1e3
    replay = graphed(fn)
    us_graph = float(np.median(time_loop(replay, steps, 3, stream))) * 1e3
    us_graph_fl = float(np.median(time_loop(replay, steps, 2, stream, scratch))) * 1e3
    graph = us_graph < us_eager
    us, us_fl = (us_graph, us_graph_fl) if graph else (us_eager, us_eager_fl)
    k_sel = min(w.token_budget // 64, (w.ctx + 63) // 64)
    db = decode_bytes(w, kind.tolist(), k_sel, w.d)
    gbs = db["total"] / (us * 1e-6) / 1e9
    del pc, stats
    return {"decode_us_per_step": us, "decode_bytes": db["total"], "GBps": gbs, "frac_hbm": gbs / pk["hbm"],
            "decode_us_per_step_l2_flushed": us_fl,
            "frac_hbm_l2_flushed": db["total"] / (us_fl * 1e-6) / 1e9 / pk["hbm"],
            "decode_us_per_step_eager": us_eager, "decode_us_per_step_graph": us_graph,
            "decode_enqueue": "graph" if graph else "eager"}


def other_configs(U, setup, dev, stream, steps, pk, scratch, names):
    """The other workloads of the problem statement, and the next rows' features, measured in the same
    run (own inputs).  `names`: the entries to run (all by default)."""
    n = max(3, steps // 2)
    res = {}
    wp = setup.wp
    if "llama3_8b_32k" in names:
        c1 = prefill_config(U, "llama3_8b_32k", dev, stream, n, pk)
        c1.update(decode_config(U, "llama3_8b_32k", dev, stream, n, pk, scratch))
        c1["note"] = "B1 S32768 Hq32/Hkv8: 4 dense (unmasked) + 4 streaming KV heads; decode 1 sequence, " \
                     "budget 4096 (latency-bound: 13 MB per step)"
        res["llama3_8b_32k"] = c1
    if "llama3_8b_decode_b16_64k" in names:
        res["llama3_8b_decode_b16_64k"] = decode_config(U, "llama3_8b_decode_b16_64k", dev, stream, n, pk, scratch)
        res["llama3_8b_decode_b16_64k"]["note"] = "B16 ctx 65536 Hq32/Hkv8, 64 outlier-channel anchors, budget 4096"
        torch.cuda.empty_cache()
    if "llama2_7b_mha_prefill_64k" in names:
        c4 = prefill_config(U, "llama2_7b_mha", dev, stream, n, pk)
        c4["note"] = "B1 S65536 Hq=Hkv=32: 16 dense (unmasked) + 16 streaming KV heads"
        res["llama2_7b_mha_prefill_64k"] = c4
        torch.cuda.empty_cache()
    if "literal" in names and wp.name == "llama3_8b_prefill_128k_vslash":
        lit = prefill_config(U, "llama3_8b_prefill_128k_vslash_literal", dev, stream, n, pk,
                             tensors=(setup.q, setup.k, setup.v))
        lit["note"] = "the 128K recipe with the literal 5 % random fill (reading A)"
        res["llama3_8b_prefill_128k_vslash_literal"] = lit
    if "lambda_tiles" in names:
        # tile-level Lambda on the prefill workload: streaming heads keep whole tiles
        lt = prefill_config(U, wp.name, dev, stream, n, pk, tensors=(setup.q, setup.k, setup.v), lambda_tiles=True)
        res["lambda_tiles"] = {"workload": wp.name, "prefill_ms": lt["prefill_ms"], "tflops": lt["tflops"],
                               "note": "the prefill workload with tile-level Lambda on its streaming heads "
                                       "(compare prefill_ms of the main line)"}
    if "cra" in names:
        # CRA report of the prefill workload's mask: a causal and a sparse LSE-only pass, then the reduction
        fn = lambda: U.lserve_cra(setup.q, setup.k, setup.v, setup.hk_p, wp.sink, wp.local, setup.bm)
        ms = float(np.median(time_loop(fn, max(2, n // 2), 2, stream)))
        cra = fn()
        torch.cuda.synchronize()
        G = wp.Hq // wp.Hkv
        dense_q = [h for h in range(wp.Hq) if setup.kind_p[h // G] == 0]
        res["cra"] = {"workload": wp.name, "ms": ms, "cra_min_dense_heads": float(cra[0, dense_q].min()),
                      "cra_min_streaming_heads": float(cra[0, [h for h in range(wp.Hq) if h not in dense_q]].min()),
                      "note": "lserve_cra: one causal and one sparse LSE-only prefill pass and the reduction"}
    if "vslash" in names:
        # vertical-slash mask construction from sampled queries on the prefill workload's q/k
        stride, tau = 16, 0.95
        ws = torch.empty(U.lserve_vslash_workspace_size(wp.B, wp.S, wp.Hq, wp.Hkv, wp.d, stride), dtype=torch.uint8,
                         device=dev)
        bm_out = torch.empty(wp.B, wp.Hkv, wp.S // 64, wp.S // 64, dtype=torch.uint8, device=dev)
        fn = lambda: U.lserve_build_vslash_mask(setup.q, setup.k, setup.hk_p, stride, tau, block_mask=bm_out,
                                                workspace=ws)
        ms = float(np.median(time_loop(fn, n, 2, stream)))
        _, cra, ncol, nsla = fn()
        torch.cuda.synchronize()
        nt = wp.S // 64
        dense = [g for g in range(wp.Hkv) if setup.kind_p[g] == 0]
        causal = torch.tril(torch.ones(nt, nt, dtype=torch.bool, device=dev))
        dens = float(np.mean([float((bm_out[0, g].bool() & causal).sum()) / float(causal.sum()) for g in dense]))
        res["vslash_mask"] = {"workload": wp.name, "ms": ms, "sample_stride": stride, "tau": tau,
                              "dense_tile_density": dens, "sampled_cra_min": float(cra[0, dense].min()),
                              "columns": [int(ncol[0, g]) for g in dense],
                              "slashes": [int(nsla[0, g]) for g in dense],
                              "note": "lserve_build_vslash_mask: last row of every 16th query tile sampled, greedy "
                                      "columns/slashes until the sampled CRA reaches tau (N(0,1) keys give near-"
                                      "uniform attention, so little can be dropped)"}
    return res


OTHER_CONFIGS = ("llama3_8b_32k", "llama3_8b_decode_b16_64k", "llama2_7b_mha_prefill_64k", "literal",
                 "lambda_tiles", "cra", "vslash")


# ---------------------------------------------------------------- CPU oracle

def oracle_prefill_sample(setup, seconds=10.0, seed=0):
    """Time the fp64 oracle on sampled query rows of the prefill workload.
    Returns (rate in kept-tile TFLOP/s equivalent, rows, seconds)."""
    from oracle import attention as OA
    wp = setup.wp
    rng = np.random.default_rng(seed)
    kind = setup.kind_p.tolist()
    k = setup.k.float().cpu().numpy()
    v = setup.v.float().cpu().numpy()
    bm = setup.bm.cpu().numpy()
    n = wp.S // 64
    tiles_per_row = np.zeros((wp.Hkv, n), np.int64)
    for g in range(wp.Hkv):
        keep = OA.tile_kept(wp.S, bool(kind[g]), wp.sink, wp.local, None if kind[g] else bm[0, g])
        tiles_per_row[g] = keep.sum(axis=1)
    G = wp.Hq // wp.Hkv
    done_rows, flops, t_used = 0, 0.0, 0.0
    while t_used < seconds:
        rows = np.sort(rng.choice(wp.S, size=4, replace=False))
        qr = setup.q[:, torch.from_numpy(rows).to(setup.q.device)].float().cpu().numpy()
        t0 = time.perf_counter()
        OA.masked_attention(qr, k, v, kind, wp.sink, wp.local, bm, rows=rows, q_at_rows=True)
        t_used += time.perf_counter() - t0
        done_rows += len(rows)
        flops += sum(int(tiles_per_row[g, r // 64]) * G * 4 * 64 * wp.d for g in range(wp.Hkv) for r in rows)
    return flops / t_used / 1e12, done_rows, t_used


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


# ---------------------------------------------------------------------- main

def run_reference(args, rank, world):
    """Reference arm: the CPU oracle as it stands, on bounded samples of the same workload."""
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    setup = Setup(dev, args.prefill_wl, args.decode_wl)
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_prefill_sample(setup, seconds=per_step / 4, seed=100 + i)
    rates, secs, rows = [], 0.0, 0
    for i in range(args.steps):
        r, nr, t = oracle_prefill_sample(setup, seconds=per_step, seed=i)
        rates.append(r)
        secs += t
        rows += nr
    value = float(np.mean(rates))
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(1, args.steps) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": setup.wp.name, "seq_len": setup.wp.S, "kind": "oracle on sampled rows"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} query rows x {setup.wp.Hq} heads of the 128K prefill, "
                                   f"{secs:.1f} s of fp64 NumPy"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--other-configs", default="all",
                    help="comma list of the other workloads / features to measure (all, none, or names from "
                         "OTHER_CONFIGS)")
    ap.add_argument("--prefill-wl", default=PREFILL_WL, choices=sorted(W.WORKLOADS))
    ap.add_argument("--decode-wl", default=DECODE_WL, choices=sorted(W.WORKLOADS))
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))

    if args.impl == "reference":
        run_reference(args, rank, world)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return

    import unified_sparse_attention_b200 as U
    U.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    setup = Setup(dev, args.prefill_wl, args.decode_wl)
    wp, wd = setup.wp, setup.wd
    pk = peaks()

    out_p = torch.empty_like(setup.q)
    ws_p = torch.empty(U.lserve_prefill_workspace_size(wp.B, wp.S, wp.Hq, wp.Hkv, wp.d), dtype=torch.uint8,
                       device=dev)
    stats = U.lserve_update_page_stats(setup.kp, setup.pt, setup.sl, setup.hk_d)
    dargs = (setup.qd, setup.kp, setup.vp, setup.pt, setup.sl, stats, setup.hk_d, wd.sink, wd.local,
             wd.token_budget)
    ws_d = torch.empty(U.lserve_decode_workspace_size(*dargs), dtype=torch.uint8, device=dev)
    out_d = torch.empty_like(setup.qd)
    n = wp.S // 64
    ws_t = torch.empty_like(ws_p)

    def prefill():
        U.lserve_prefill(setup.q, setup.k, setup.v, setup.hk_p, wp.sink, wp.local, setup.bm, out=out_p,
                         workspace=ws_p)

    def tile_lists():
        U.lserve_prefill_tile_lists(wp.B, wp.S, wp.Hq, wp.Hkv, wp.d, setup.hk_p, wp.sink, wp.local, setup.bm)

    def decode():
        U.lserve_update_page_stats(setup.kp, setup.pt, setup.sl, setup.hk_d, stats=stats,
                                   first_logical_page=setup.last_lp)
        U.lserve_decode(*dargs, out=out_d, workspace=ws_d)

    def decode_only():
        U.lserve_decode(*dargs, out=out_d, workspace=ws_d)

    # selection reuse across decode steps: a step that keeps the dense heads'
    # pages of a selection step (no scoring, no summaries read)
    _, _, sel_d, seln_d = U.lserve_decode(*dargs, out=out_d, workspace=ws_d, return_selection=True)

    def decode_reuse():
        U.lserve_decode_reuse(setup.qd, setup.kp, setup.vp, setup.pt, setup.sl, setup.hk_d, wd.sink, wd.local,
                              wd.token_budget, sel_d, seln_d, out=out_d, workspace=ws_d)

    # INT4 pages: the decode pool quantised once (lserve_quantize_pages_int4), then
    # the same decode step over codes dequantised on chip
    kq, kpar, vq, vpar, stats4 = U.lserve_quantize_pages_int4(setup.kp, setup.vp, setup.pt, setup.sl, setup.hk_d)

    def quantize_pool():
        U.lserve_quantize_pages_int4(setup.kp, setup.vp, setup.pt, setup.sl, setup.hk_d, kq=kq, kpar=kpar, vq=vq,
                                     vpar=vpar, stats=stats4)

    def decode_int4():
        U.lserve_decode_int4(setup.qd, kq, vq, kpar, vpar, setup.pt, setup.sl, stats4, setup.hk_d, wd.sink,
                             wd.local, wd.token_budget, out=out_d, workspace=ws_d)

    def step():
        prefill()
        decode()

    # Every step reads far more than L2 holds (prefill: q, k, v; decode: page
    # summaries + selected pages), so the timed loops do not flush L2 between
    # steps; the decode step is also timed with a flush (a 252 MB write, then a 252 MB read that
    # takes the written lines' write-back out of the step) for reference.
    scratch = torch.zeros(4 * L2_BYTES // 4, dtype=torch.float32, device=dev)   # 2 x L2 written + 2 x L2 read
    prefill_in_bytes = sum(t.numel() * t.element_size() for t in (setup.q, setup.k, setup.v))
    big = prefill_in_bytes > L2_BYTES and setup.dbytes["total"] > L2_BYTES
    fl = None if big else scratch   # smaller (profiling) workloads are flushed instead
    # component timings (same launches, timed separately)
    t_tiles = time_loop(tile_lists, max(3, args.steps // 2), 2, stream, fl)
    t_prefill = time_loop(prefill, args.steps, args.warmup, stream, fl)
    # decode steps: one CUDA-graph replay of the captured C-ABI call per step (see graphed()); the
    # eager figure (Python enqueue of each call inside the timed region) is reported beside it
    t_decode_eager = time_loop(decode_only, args.steps, args.warmup, stream, fl)
    t_decode_eager_fl = time_loop(decode_only, args.steps, 2, stream, scratch)
    t_reuse_eager = time_loop(decode_reuse, args.steps, args.warmup, stream, fl)
    t_int4_eager = time_loop(decode_int4, args.steps, args.warmup, stream, fl)
    g_decode, g_reuse, g_int4 = graphed(decode_only), graphed(decode_reuse), graphed(decode_int4)
    t_decode_graph = time_loop(g_decode, args.steps, args.warmup, stream, fl)
    t_decode_graph_fl = time_loop(g_decode, args.steps, 2, stream, scratch)
    t_reuse_graph = time_loop(g_reuse, args.steps, args.warmup, stream, fl)
    t_int4_graph = time_loop(g_int4, args.steps, args.warmup, stream, fl)
    # the faster enqueue of the same kernels, chosen per measurement on its unflushed median
    dec_graph = np.median(t_decode_graph) < np.median(t_decode_eager)
    t_decode, t_decode_flushed = (t_decode_graph, t_decode_graph_fl) if dec_graph else \
        (t_decode_eager, t_decode_eager_fl)
    t_reuse = min(t_reuse_graph, t_reuse_eager, key=np.median)
    t_int4 = min(t_int4_graph, t_int4_eager, key=np.median)
    t_quant = time_loop(quantize_pool, 2, 1, stream)   # once per page in a server: off the step
    names = OTHER_CONFIGS if args.other_configs == "all" else \
        tuple(x for x in args.other_configs.split(",") if x and x != "none")
    extra = other_configs(U, setup, dev, stream, args.steps, pk, scratch, names) if names else None

    # the timed steps
    clocks = Clocks(local_rank)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_step = time_loop(step, args.steps, 0, stream, fl)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    assert U.lserve_get_device_status() == 0, "kernel reported an error"

    ms_step = float(np.mean(t_step))
    ms_prefill = float(np.median(t_prefill))
    ms_tiles = float(np.median(t_tiles))
    ms_attn = max(1e-6, ms_prefill - ms_tiles)
    us_decode = float(np.median(t_decode)) * 1e3
    us_reuse = float(np.median(t_reuse)) * 1e3
    us_int4 = float(np.median(t_int4)) * 1e3
    ms_step, ms_prefill, us_decode, us_reuse, us_int4 = max_over_ranks(
        [ms_step, ms_prefill, us_decode, us_reuse, us_int4], dist, dev)
    int4_bytes = decode_bytes_int4(wd, setup.kind_d.tolist(), setup.k_sel, wd.d)
    # quantiser: K and V of every held (page, head) read once; codes, steps/offsets and
    # (dense heads) summaries written
    held = sum((int(L) + 63) // 64 for L in setup.sl.tolist())   # pages the sequences hold
    n_dense_d = sum(1 for x in setup.kind_d.tolist() if x == 0)
    quant_bytes = held * (wd.Hkv * (2 * 64 * wd.d * 2 + 64 * wd.d + 2 * wd.d * 4 + 2 * 64 * 4)
                          + n_dense_d * 4 * 2 * wd.d * 2)
    reuse_bytes = setup.dbytes["total"] - setup.dbytes["stats"]

    tflops_prefill = setup.prefill_flops / (ms_prefill * 1e-3) / 1e12
    tflops_attn = setup.prefill_flops / (ms_attn * 1e-3) / 1e12
    gbps_decode = setup.dbytes["total"] / (us_decode * 1e-6) / 1e9
    value = world * setup.prefill_flops / (ms_prefill * 1e-3) / 1e12

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (setup.q, setup.k, setup.v))
        hbm_ = setup.bm.cpu().pin_memory()
        hqd = setup.qd.cpu().pin_memory()
        ho = torch.empty(setup.q.shape, dtype=torch.bfloat16).pin_memory()
        hod = torch.empty(setup.qd.shape, dtype=torch.bfloat16).pin_memory()
        dq, dk, dv, dbm, dqd = (torch.empty_like(t) for t in (setup.q, setup.k, setup.v, setup.bm, setup.qd))

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            dbm.copy_(hbm_, non_blocking=True)
            dqd.copy_(hqd, non_blocking=True)
            U.lserve_prefill(dq, dk, dv, setup.hk_p, wp.sink, wp.local, dbm, out=out_p, workspace=ws_p)
            U.lserve_update_page_stats(setup.kp, setup.pt, setup.sl, setup.hk_d, stats=stats,
                                       first_logical_page=setup.last_lp)
            U.lserve_decode(dqd, *dargs[1:], out=out_d, workspace=ws_d)
            ho.copy_(out_p, non_blocking=True)
            hod.copy_(out_d, non_blocking=True)

        t_e2e = time_loop(e2e_step, max(3, args.steps // 2), 2, stream, fl)
        ms_e2e = float(np.mean(t_e2e))
        ms_e2e = max_over_ranks([ms_e2e], dist, dev)[0]
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hbm_, hqd))
        d2h = ho.numel() * 2 + hod.numel() * 2
        e2e = {"value": world * setup.prefill_flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "note": "prefill TFLOP/s over the whole step (prefill + decode) incl. H2D of q,k,v,mask,"
                       "decode q and D2H of both outputs; the KV page pool stays resident"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, rows, secs = oracle_prefill_sample(setup, seconds=10.0)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{rows} query rows x {wp.Hq} heads of the 128K prefill ({secs:.1f} s fp64 NumPy), "
                         f"rate scaled by each row's kept-tile FLOPs"}

    n_dense = sum(1 for g in range(wp.Hkv) if setup.kind_p[g] == 0)
    dense_density = (sum(setup.tiles[g] for g in range(wp.Hkv) if setup.kind_p[g] == 0)
                     / max(1, n_dense * n * (n + 1) / 2))
    launches_per_step = 4 + 1 + 4   # tile count/scan/fill + attention; stats refresh; score/top-k+plan/attention/merge
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{wp.name} prefill (B{wp.B} S{wp.S} Hq{wp.Hq} Hkv{wp.Hkv} d{wp.d}, dense-head tile "
                               f"density {dense_density:.3f}) + {wd.name} decode (B{wd.dec_B} ctx{wd.ctx} Hq{wd.Hq} "
                               f"Hkv{wd.Hkv} d{wd.d}, budget {wd.token_budget})",
                   "l2": (f"no flush: inputs larger than L2 ({L2_BYTES / 2**20:.0f} MiB) -- prefill reads "
                          f"{prefill_in_bytes / 1e9:.2f} GB of q/k/v, decode {setup.dbytes['total'] / 1e6:.0f} MB "
                          f"per step") if big else "flushed between steps (a 252 MB write, then a 252 MB read)",
                   "parallelism": f"replicas x{world}"},
        "prefill_ms": ms_prefill, "prefill_attention_ms": ms_attn, "tile_lists_ms": ms_tiles,
        "prefill_tflops": tflops_prefill, "kept_tile_tflop": setup.prefill_flops / 1e12,
        "decode_us_per_step": us_decode, "decode_GBps": gbps_decode, "decode_bytes": setup.dbytes,
        "decode_us_per_step_l2_flushed": float(np.median(t_decode_flushed)) * 1e3,
        "decode_us_per_step_eager": float(np.median(t_decode_eager)) * 1e3,
        "decode_us_per_step_graph": float(np.median(t_decode_graph)) * 1e3,
        "decode_timing": "the same four kernels enqueued two ways: eager (the Python C-ABI call inside the timed "
                         "region, launches chained by programmatic dependent launch) and one CUDA-graph replay "
                         "of the captured call; decode_us_per_step (and the flushed, reuse and INT4 figures) "
                         f"take the faster: {'graph' if dec_graph else 'eager'} here",
        "decode_reuse": {"us_per_step": us_reuse, "bytes": reuse_bytes,
                         "GBps": reuse_bytes / (us_reuse * 1e-6) / 1e9,
                         "frac_hbm": reuse_bytes / (us_reuse * 1e-6) / 1e9 / pk["hbm"],
                         "cadence4_us_per_step": (us_decode + 3 * us_reuse) / 4,
                         "note": "selection reused across decode steps: the dense heads keep the pages of a "
                                 "selection step (no scoring, no summaries read); cadence4 = one selection step "
                                 "and three reuse steps"},
        "decode_int4": {"us_per_step": us_int4, "bytes": int4_bytes["total"],
                        "GBps": int4_bytes["total"] / (us_int4 * 1e-6) / 1e9,
                        "frac_hbm": int4_bytes["total"] / (us_int4 * 1e-6) / 1e9 / pk["hbm"],
                        "speedup_vs_bf16": us_decode / us_int4,
                        "quantize_pool_ms": float(np.median(t_quant)),
                        "quantize_pool_bytes": quant_bytes,
                        "quantize_GBps": quant_bytes / (float(np.median(t_quant)) * 1e-3) / 1e9,
                        "note": "decode step over INT4 pages (codes + fp32 steps/offsets, dequantised on chip); "
                                "pool quantised once before timing"},
        "roofline": {"bound": "tensor", "kernel": "prefill attention", "achieved": tflops_prefill,
                     "peak": pk["bf16"], "unit": "TFLOP/s", "frac": tflops_prefill / pk["bf16"],
                     "traffic": traffic("prefill", wp.name == PREFILL_WL), "traffic_unit": "bytes per launch",
                     "algorithmic_bytes_note": "compulsory: q, k, v, mask read once, out and lse written once",
                     "peak_source": pk["source"] + " bf16 burst",
                     "peak_sustained": pk["bf16_sust"], "frac_sustained": tflops_prefill / pk["bf16_sust"],
                     "peak_note": "frac uses the burst peak; in loops this kernel runs at the 1 kW power cap "
                                  "(about 1.7 GHz, sw_power_cap), where the sustained cuBLAS figure applies",
                     "achieved_note": "kept-tile FLOPs / whole lserve_prefill time (the on-device tile-list "
                                      "build included)"},
        "roofline_decode": {"bound": "hbm", "kernel": "decode step (score, top-k + plan, paged attention, merge)",
                            "achieved": gbps_decode, "peak": pk["hbm"], "unit": "GB/s",
                            "frac": gbps_decode / pk["hbm"],
                            "traffic": traffic("decode", wd.name == DECODE_WL), "traffic_unit": "bytes per step",
                            "algorithmic_bytes": setup.dbytes["total"], "peak_source": pk["source"]},
        "other_configs": extra,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
