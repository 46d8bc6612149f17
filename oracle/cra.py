"""Cumulative residual attention (CRA) of a sparse mask.

Test infrastructure only (see the package docstring).

Source: LServe + SampleAttention blog post, "CRA - The Accuracy Proxy" and
Fig. 4: for every query, the share of its full (causal, unmasked) softmax mass
that the sparse mask keeps; CRA is the minimum of that share over the queries.

    r_i  = sum_{j in K(i)} softmax_j(scale * q_i . k_j  |  j <= i)
    CRA  = min_i r_i

Computed here as exp(lse_sparse(i) - lse_causal(i)), which is the same ratio.
"""
from __future__ import annotations

import numpy as np

from .attention import masked_attention


def retained_mass(q, k, v, head_kind, sink, local, block_mask=None, scale=None, rows=None, lambda_tiles=False):
    """float64[B, Hq, R]: per query row the retained share of its causal softmax mass."""
    dense_kind = np.zeros(len(head_kind), dtype=np.uint8)
    _, lse_full = masked_attention(q, k, v, dense_kind, 0, 0, None, scale, rows)
    _, lse_sparse = masked_attention(q, k, v, head_kind, sink, local, block_mask, scale, rows,
                                     lambda_tiles=lambda_tiles)
    return np.exp(lse_sparse - lse_full)


def cra(q, k, v, head_kind, sink, local, block_mask=None, scale=None, rows=None, lambda_tiles=False):
    """float64[B, Hq]: minimum over query rows of the retained mass."""
    return retained_mass(q, k, v, head_kind, sink, local, block_mask, scale, rows, lambda_tiles).min(axis=2)
