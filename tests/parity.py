"""Shared comparison helpers for the GPU parity tests (imported by tests only).

Tolerances for attention outputs (bf16 inputs, fp32 accumulation, bf16 output)
against the fp64 oracle: max |err| <= 1e-2 and ||err||_2 / ||ref||_2 <= 5e-3.
LSE (fp32 on the GPU): |err| <= 2e-3.  Page summaries: bit-exact.  Page sets:
exact except inside the tie band (oracle scores within 1e-5 relative of the
k-th score), where only the tied pages may differ and the count must match.
"""
from __future__ import annotations

import numpy as np
import torch

ATOL_OUT = 1e-2
RTOL_L2 = 5e-3
ATOL_LSE = 2e-3
TIE_REL = 1e-5


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def attn_errors(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref)) or 1.0
    rel_l2 = float(np.linalg.norm(got - ref)) / denom
    return max_abs, rel_l2


def assert_attn_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs, rel_l2 = attn_errors(got, ref)
    assert max_abs <= ATOL_OUT and rel_l2 <= RTOL_L2, f"{what}: max_abs={max_abs:.3g} rel_l2={rel_l2:.3g}"
    return max_abs, rel_l2


def assert_lse_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: -inf pattern differs"
    assert np.all(np.isneginf(got[~fin])), f"{what}: empty rows must give -inf"
    if fin.any():
        e = float(np.abs(got[fin] - ref[fin]).max())
        assert e <= ATOL_LSE, f"{what}: lse max_abs={e:.3g}"


def check_selection(sel_gpu, k: int, scores_ref: np.ndarray):
    """Tie-aware comparison of one (b, kvh) page set.  Returns True if a tie was present."""
    sel_gpu = [int(x) for x in sel_gpu]
    assert len(sel_gpu) == k, f"selected {len(sel_gpu)} pages, expected {k}"
    assert sel_gpu == sorted(sel_gpu) and len(set(sel_gpu)) == k, "selection must be ascending and unique"
    n = len(scores_ref)
    if k >= n:
        assert sel_gpu == list(range(n))
        return False
    if k == 0:
        return False
    order = np.lexsort((np.arange(n), -scores_ref))
    t = scores_ref[order[k - 1]]
    band = TIE_REL * max(abs(t), np.finfo(np.float64).tiny)
    must = set(np.nonzero(scores_ref > t + band)[0].tolist())
    never = set(np.nonzero(scores_ref < t - band)[0].tolist())
    s = set(sel_gpu)
    assert must <= s, f"missed pages {sorted(must - s)[:8]} clearly above the k-th score"
    assert not (s & never), f"selected pages {sorted(s & never)[:8]} clearly below the k-th score"
    oracle_set = set(np.sort(order[:k]).tolist())
    return s != oracle_set or abs(scores_ref[order[k - 1]] - scores_ref[order[k]]) <= band
