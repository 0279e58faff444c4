"""Plain fp64 CPU oracle for branch attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product package may import, call or
link this package; only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg (and its reference arm) use it.  It shares no code with the CUDA
path.

Every function follows "Online Draft Co-Training" (arXiv 2609.07108) as
summarised on the paper pages:
  * technical-contribution / method-detail sections: a branch query is split
    into a causal main-sequence part and a rank-local branch part, merged by
    l = log(e^{l_m} + e^{l_b}), O = e^{l_m - l} O_m + e^{l_b - l} O_b;
  * core-innovation section: packed, load-balanced zigzag sharding with the
    branch K/V kept on the anchor's shard.
Parity pins for every function live in tests/test_oracle_*.py.
"""
from .branch_attention import (  # noqa: F401
    Derived, derive, visible_keys, dense_mask, forward_dense, backward_dense,
    lse_merge, split_forward, zigzag_chunks, zigzag_forward, rows_forward,
    rows_backward_dq, keys_backward, keys_backward_both, useful_pairs, to64, visible_counts, zero_query_dv, round_bf16,
)
from .plan import plan, row_intervals, PLAN_BM, PLAN_BN  # noqa: F401
