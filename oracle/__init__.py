"""Plain, slow, CPU-only reference of the unified sparse-attention path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (the CUDA library and its Python binding) never calls into it and
fails loudly when its compiled library is missing; nothing here shares code,
tables or constants with the CUDA side.

Everything is NumPy float64.  Inputs are the same bf16 tensors the GPU sees,
up-cast exactly to float64.  Each function follows the plain definition of what
the method computes; where the pages leave a step open the reading taken is
stated in the function's docstring.

Sources (page title, section / figure):

* mlsanity, "LServe: Efficient Long-sequence LLM Serving with Unified Sparse
  Attention" -- Abstract (block-wise skipping, streaming heads, constant number
  of KV pages, hierarchical page selection by query-centric similarity);
  "Builds on" (Quest: Query-Aware Sparsity; PagedAttention; DuoAttention).
* LServe + SampleAttention blog post -- "LServe - Prefill Phase" and Fig. 1
  (whole-tile skipping, Lambda-shaped streaming support), "LServe - Decode
  Phase" and Fig. 2 (per-page summary score, top-k pages, token-level attention
  inside the selected pages), "CRA - The Accuracy Proxy" and Fig. 4.

Modules:

* ``attention``  masked causal softmax attention (prefill), kept-tile lists
* ``selection``  key min/max page summaries, upper-bound page scores,
                 hierarchical (logical -> physical) max, top-k pages
* ``decode``     token-level attention over the selected pages (or the
                 streaming heads' sink + local tokens)
* ``cra``        cumulative residual attention of a mask

Pinned by ``tests/test_oracle_*.py`` against brute force, closed forms,
library routines and invariants (see each test's docstring).
"""
from . import attention, selection, decode, cra  # noqa: F401
