"""Planted mistakes: each plausible slip in the oracle must fail at least one pin.

Every case swaps one oracle function (on the CPU, through monkeypatch) for a
copy with a single deliberate error -- an off-by-one window, a dropped or
swapped term, a wrong tie rule, a missing scale -- and checks that the named
pin test then fails.  This is what makes the pins a check on the oracle and
not a restatement of it.
"""
import numpy as np
import pytest

import test_oracle_attention as TA
import test_oracle_decode as TD
import test_oracle_quant as TQ
import test_oracle_selection as TS
from oracle import attention as A
from oracle import cra as CR
from oracle import decode as D
from oracle import quant as Q
from oracle import selection as Sel
from oracle import vslash as VS
import test_oracle_vslash as TV

_kept = A.kept_mask
_bounds = Sel.logical_bounds
_masked = A.masked_attention


def kept_window_off_by_one(rows, S, streaming, sink, local, tm, lambda_tiles=False):
    i = np.asarray(rows)[:, None]
    j = np.arange(S)[None, :]
    if streaming:
        return (j <= i) & ((j < sink) | (i - j <= local))
    return _kept(rows, S, streaming, sink, local, tm, lambda_tiles)


def kept_sink_inclusive(rows, S, streaming, sink, local, tm, lambda_tiles=False):
    i = np.asarray(rows)[:, None]
    j = np.arange(S)[None, :]
    if streaming:
        return (j <= i) & ((j <= sink) | (i - j < local))
    return _kept(rows, S, streaming, sink, local, tm, lambda_tiles)


def kept_mask_transposed(rows, S, streaming, sink, local, tm, lambda_tiles=False):
    i = np.asarray(rows)[:, None]
    j = np.arange(S)[None, :]
    if not streaming and tm is not None:
        return (j <= i) & (np.asarray(tm)[j // 64, i // 64] != 0)
    return _kept(rows, S, streaming, sink, local, tm, lambda_tiles)


def kept_tile_lambda_drops_causal(rows, S, streaming, sink, local, tm, lambda_tiles=False):
    i = np.asarray(rows)[:, None]
    j = np.arange(S)[None, :]
    if streaming and lambda_tiles:   # whole kept tiles, the diagonal one included past the query
        qt, kt = i // 64, j // 64
        return (kt <= qt) & ((64 * kt < sink) | (np.maximum(64 * qt - 64 * kt - 63, 0) < local))
    return _kept(rows, S, streaming, sink, local, tm, lambda_tiles)


def vslash_covered_wrong_side(kind, idx, qt, kt):
    return kt <= qt and ((kind == "column" and kt == idx) or (kind == "slash" and kt - qt == idx))


def vslash_order_no_forced_diagonal(tiles, r):
    order = _vs_order(tiles, r)
    return sorted(order, key=lambda c: (-c[2], 0 if c[0] == "column" else 1, c[1]))


def bounds_kmax_only(q, stats, page_table, seq_len, b, h, G):
    st = np.array(stats, dtype=np.float64)
    st[..., 0, :] = st[..., 1, :]
    return _bounds(q, st, page_table, seq_len, b, h, G)


def bounds_min_instead_of_max(q, stats, page_table, seq_len, b, h, G):
    q = np.asarray(q, dtype=np.float64)
    out = _bounds(q, stats, page_table, seq_len, b, h, G)
    kvh = h // G
    for i in range(out.shape[0]):
        for l in range(4):
            if np.isfinite(out[i, l]):
                s = stats[page_table[b][i], kvh, l]
                out[i, l] = np.minimum(q[b, h] * s[1], q[b, h] * s[0]).sum()
    return out


def topk_ties_high(scores_row, k):
    s = np.asarray(scores_row, dtype=np.float64)
    order = np.lexsort((-np.arange(len(s)), -s))
    return np.sort(order[:k]), np.inf


def token_set_drops_current(seq_len, streaming, sink, local, pages=None):
    t = _token_set(seq_len, streaming, sink, local, pages)
    return t[t < seq_len - 1]


def masked_no_scale(q, k, v, head_kind, sink, local, block_mask=None, scale=None, rows=None, row_chunk=256):
    return _masked(q, k, v, head_kind, sink, local, block_mask, 1.0, rows, row_chunk)


def page_stats_ignores_length(k_pages, page_table, seq_lens, head_kind, first_logical_page=0, stats=None):
    full = [64 * ((int(L) + 63) // 64) for L in seq_lens]
    return _stats(k_pages, page_table, full, head_kind, first_logical_page, stats)


_stats = Sel.page_stats
_token_set = D.token_set


def cra_mean_not_min(q, k, v, head_kind, sink, local, block_mask=None, scale=None, rows=None, lambda_tiles=False):
    return CR.retained_mass(q, k, v, head_kind, sink, local, block_mask, scale, rows, lambda_tiles).mean(axis=2)


def retained_inverted(q, k, v, head_kind, sink, local, block_mask=None, scale=None, rows=None, lambda_tiles=False):
    return 1.0 / _retained(q, k, v, head_kind, sink, local, block_mask, scale, rows, lambda_tiles)


_retained = CR.retained_mass
_vs_order = VS.candidate_order


def codes_truncate(x, lo, s):
    with np.errstate(divide="ignore", invalid="ignore"):
        c = np.floor(((x - lo).astype(np.float32) / s).astype(np.float32))
    c = np.where(s > 0, c, 0.0)
    return np.clip(c, 0, 15).astype(np.uint8)


def step_sixteen_levels(lo, hi):
    return ((hi - lo) / np.float32(16.0)).astype(np.float32)


def dequant_drops_offset(code, s, lo):
    return (code.astype(np.float64) * s.astype(np.float64)).astype(np.float32)




CASES = [
    ("window off by one", A, "kept_mask", kept_window_off_by_one,
     lambda: TA.test_streaming_equals_sdpa_with_lambda_mask(0, 64)),
    ("sink inclusive", A, "kept_mask", kept_sink_inclusive,
     lambda: TA.test_streaming_equals_sdpa_with_lambda_mask(3, 1)),
    ("block mask transposed", A, "kept_mask", kept_mask_transposed,
     TA.test_block_mask_equals_sdpa_with_expanded_mask),
    ("tile-level Lambda drops the causal mask", A, "kept_mask", kept_tile_lambda_drops_causal,
     lambda: TA.test_tile_level_lambda_brute_force(64, 256)),
    ("no softmax scale", A, "masked_attention", masked_no_scale,
     lambda: TA.test_all_tiles_kept_equals_dense_causal(2)),
    ("bound drops kmin", Sel, "logical_bounds", bounds_kmax_only,
     lambda: TS.test_bound_dominates_every_dot_product(1)),
    ("bound takes min", Sel, "logical_bounds", bounds_min_instead_of_max,
     TS.test_bound_hand_example),
    ("ties to higher index", Sel, "topk_pages", topk_ties_high,
     lambda: TS.test_topk_brute_force_with_ties(0)),
    ("decode drops current token", D, "token_set", token_set_drops_current,
     lambda: TD.test_full_budget_equals_dense_decode(None)),
    ("stats ignore sequence length", Sel, "page_stats", page_stats_ignores_length,
     TS.test_stats_closed_form_on_contiguous_keys),
    ("CRA takes the mean", CR, "cra", cra_mean_not_min, TD.test_cra_is_one_without_dropping_and_matches_weight_sums),
    ("retained mass inverted", CR, "retained_mass", retained_inverted,
     TD.test_cra_is_one_without_dropping_and_matches_weight_sums),
    ("vslash slash offset from the wrong side", VS, "covered", vslash_covered_wrong_side,
     TV.test_hand_example_order_and_cra),
    ("vslash diagonal not forced first", VS, "candidate_order", vslash_order_no_forced_diagonal,
     TV.test_hand_example_order_and_cra),
    ("INT4 codes truncated", Q, "_codes", codes_truncate, TQ.test_codes_range_extremes_monotone_and_error_bound),
    ("INT4 step over 16 levels", Q, "_step", step_sixteen_levels,
     TQ.test_codes_range_extremes_monotone_and_error_bound),
    ("INT4 dequantisation drops the offset", Q, "dequant", dequant_drops_offset,
     TQ.test_constant_group_dequantises_exactly),
    ("INT4 summaries rounded to nearest", Q, "bf16_round_down", Q.bf16_round,
     TQ.test_summaries_of_dequantised_keys_bound_them),
]


@pytest.mark.parametrize("name,mod,attr,bad,pin", CASES, ids=[c[0] for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, mod, attr, bad, pin):
    monkeypatch.setattr(mod, attr, bad)
    if mod is Sel and attr == "page_stats":
        monkeypatch.setattr(TS.Sel, attr, bad)
    with pytest.raises(AssertionError):
        pin()
