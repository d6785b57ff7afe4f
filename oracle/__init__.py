"""fp64 CPU oracle of the MSA forward pass: test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may use it; the product path never imports it.
"""
from .msa_oracle import (  # noqa: F401
    attend, attend_row, block_maxima_row, block_scores, dense_causal_gqa, forward,
    index_scores_row, pooled_select, select, select_row, selection_metrics,
)
